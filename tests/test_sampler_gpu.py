"""GPU parity of the layered flow sampler (block stack x Euler steps) against
the float64 oracle's sampler loop, from the same seeded weights, modulation
and initial latents."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import H3Sampler, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("w,n_layers,n_steps", [(S.WORKLOADS["tiny"], 50, 8), (RAGGED, 4, 2)],
                         ids=["tiny_50x8", "ragged_4x2"])
def test_sampler_against_oracle(w, n_layers, n_steps):
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, n_layers, n_steps)
    dev = torch.device("cuda", 0)
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in st["blocks"]]
    smp = H3Sampler(w, inp, blocks, device=dev)
    text = to_dev_bf16(inp["text"], dev)
    lv = torch.from_numpy(st["lat_video"]).to(dev)
    la = torch.from_numpy(st["lat_audio"]).to(dev)
    lv_bf, la_bf = lv.to(torch.bfloat16), la.to(torch.bfloat16)
    mod_all = torch.from_numpy(st["mod_all"]).to(dev)
    smp.run(text, lv, la, lv_bf, la_bf, mod_all, n_steps)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    assert torch.equal(lv_bf, lv.to(torch.bfloat16)) and torch.equal(la_bf, la.to(torch.bfloat16))
    r, pos = oracle_ranges_and_pos(w)
    rv, ra = O.sample(inp["text"], st["lat_video"], st["lat_audio"], inp, st["blocks"], st["mod_all"], r, pos, w.H,
                      n_steps)
    gv, ga = to_np(lv), to_np(la)
    # the latents' total change over the sampler (the part the model decides)
    check_close(gv - st["lat_video"], rv - st["lat_video"], "video latent change")
    check_close(ga - st["lat_audio"], ra - st["lat_audio"], "audio latent change")
    check_close(gv, rv, "video latent")
    check_close(ga, ra, "audio latent")


@pytest.mark.parametrize("qk_e4m3", [False, True], ids=["qk_bf16", "qk_e4m3"])
def test_sampler_e4m3_against_oracle(qk_e4m3):
    """The sampler with e4m3 block GEMMs (and, qk_e4m3, e4m3 q, k into
    attention) against the oracle's sampler loop with the e4m3 block (weights
    quantised per output channel on both sides from the same bf16 values; the
    row quantiser is bit-exact)."""
    from oracle import h3_oracle_fp8 as F8
    w, n_layers, n_steps = RAGGED, 2, 2
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, n_layers, n_steps)
    dev = torch.device("cuda", 0)
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in st["blocks"]]
    smp = H3Sampler(w, inp, blocks, device=dev, e4m3=True, qk_e4m3=qk_e4m3)
    text = to_dev_bf16(inp["text"], dev)
    lv = torch.from_numpy(st["lat_video"]).to(dev)
    la = torch.from_numpy(st["lat_audio"]).to(dev)
    lv_bf, la_bf = lv.to(torch.bfloat16), la.to(torch.bfloat16)
    mod_all = torch.from_numpy(st["mod_all"]).to(dev)
    smp.run(text, lv, la, lv_bf, la_bf, mod_all, n_steps)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    r, pos = oracle_ranges_and_pos(w)
    q8 = [{n: F8.quantize_weight(b[n]) for n in ("Wqkv", "Wo", "Wgu", "Wd")} for b in st["blocks"]]
    sv, sa = O.sigma_schedule(n_steps, 12.0), O.sigma_schedule(n_steps, 3.0)
    rv = st["lat_video"].astype(np.float64)
    ra = st["lat_audio"].astype(np.float64)
    T, Hl, Wl, _ = rv.shape
    ch, na, _ = ra.shape
    for s in range(n_steps):
        x = O.embed(inp["text"], O.round_to_bf16(rv), O.round_to_bf16(ra), inp["W_text"], inp["W_vid"], inp["W_aud"], r)
        for b, Wb in enumerate(st["blocks"]):
            x = F8.block_forward_e4m3(x, st["mod_all"][s][b], r, pos, *q8[b]["Wqkv"], Wb["qn_w"], Wb["kn_w"],
                                      *q8[b]["Wo"], *q8[b]["Wgu"], *q8[b]["Wd"], w.H, qk_e4m3=qk_e4m3)
        vv, va = O.head_unpack(x, r, inp["W_vhead"], inp["W_ahead"], T, Hl, Wl, ch, na)
        rv = O.euler_step(rv, vv, sv[s], sv[s + 1])
        ra = O.euler_step(ra, va, sa[s], sa[s + 1])
    gv, ga = to_np(lv), to_np(la)
    # the e4m3 block's delta bound (see test_fp8_gpu) for the latents' change
    bound = 0.5 if qk_e4m3 else 0.35
    check_close(gv - st["lat_video"], rv - st["lat_video"], "video latent change", bound, 2.5e-2)
    check_close(ga - st["lat_audio"], ra - st["lat_audio"], "audio latent change", bound, 2.5e-2)
    check_close(gv, rv, "video latent")
    check_close(ga, ra, "audio latent")


def test_full_width_two_block_stack_one_step_sampled_rows():
    """Two full-width blocks and one Euler step (sigma 1 -> 0) on the 768sq_2s
    workload (7,904 packed tokens), through the sampler's calls.  The oracle
    runs the first block on every row (the second block's attention reads all
    of its output), then the second block, the head and the Euler update on
    sampled rows; the test compares the latent entries that those rows
    produce (a video token's 2 x 2 x 24 latent values, an audio token's 64)."""
    w, n_layers, n_steps = S.WORKLOADS["768sq_2s"], 2, 1
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, n_layers, n_steps)
    dev = torch.device("cuda", 0)
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in st["blocks"]]
    smp = H3Sampler(w, inp, blocks, device=dev)
    text = to_dev_bf16(inp["text"], dev)
    lv = torch.from_numpy(st["lat_video"]).to(dev)
    la = torch.from_numpy(st["lat_audio"]).to(dev)
    lv_bf, la_bf = lv.to(torch.bfloat16), la.to(torch.bfloat16)
    mod_all = torch.from_numpy(st["mod_all"]).to(dev)
    smp.run(text, lv, la, lv_bf, la_bf, mod_all, n_steps)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    del blocks, smp
    r, pos = oracle_ranges_and_pos(w)
    L = r["L"]
    T, Hl, Wl, _ = st["lat_video"].shape
    ch, na, _ = st["lat_audio"].shape
    x = O.embed(inp["text"], O.round_to_bf16(st["lat_video"]), O.round_to_bf16(st["lat_audio"]), inp["W_text"],
                inp["W_vid"], inp["W_aud"], r)
    b0, b1 = st["blocks"]
    x = O.block_forward(x, st["mod_all"][0][0], r, pos, n_heads=w.H, **b0)
    sa_, ca_ = r["start"][O.AUDIO], r["count"][O.AUDIO]
    sv_, cv_ = r["start"][O.VIDEO], r["count"][O.VIDEO]
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([rng.choice(np.arange(sa_, sa_ + ca_), 6, replace=False),
                                     rng.choice(np.arange(sv_, sv_ + cv_), 18, replace=False),
                                     [sa_, sa_ + ca_ - 1, sv_, L - 1]]))
    x2, _ = O.block_forward_rows(x, st["mod_all"][0][1], r, pos, rows, n_heads=w.H, **b1)
    # the head is row-local: run it on a stream that holds only the sampled
    # rows, then keep the latent entries those rows produce
    xs = np.zeros((L, w.D))
    xs[rows] = x2
    vv, va = O.head_unpack(xs, r, inp["W_vhead"], inp["W_ahead"], T, Hl, Wl, ch, na)
    rv = O.euler_step(st["lat_video"], vv, 1.0, 0.0)
    ra = O.euler_step(st["lat_audio"], va, 1.0, 0.0)
    src = np.zeros(L, bool)
    src[rows] = True
    sel_v = O.unpatchify(np.repeat(src[sv_:sv_ + cv_, None], 96, axis=1), T, Hl, Wl)
    sel_a = src[sa_:sa_ + ca_].reshape(ch, na)
    assert sel_v.sum() > 0 and sel_a.sum() > 0
    gv, ga = to_np(lv), to_np(la)
    for name, g, ref, lat0 in (("video", gv[sel_v], rv[sel_v], st["lat_video"][sel_v]),
                               ("audio", ga[sel_a], ra[sel_a], st["lat_audio"][sel_a])):
        check_close(g - lat0, ref - lat0, f"{name} latent change (sampled tokens)")
        check_close(g, ref, f"{name} latent (sampled tokens)")


def test_sampler_checkpoint_resume_is_bit_exact(tmp_path):
    """Stopping after two of four steps, saving the state, loading it into
    fresh tensors and resuming gives the uninterrupted run's latents bit for
    bit."""
    w, n_layers, n_steps = RAGGED, 2, 4
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, n_layers, n_steps)
    dev = torch.device("cuda", 0)
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in st["blocks"]]
    smp = H3Sampler(w, inp, blocks, device=dev)
    text = to_dev_bf16(inp["text"], dev)
    mod_all = torch.from_numpy(st["mod_all"]).to(dev)

    def fresh():
        lv = torch.from_numpy(st["lat_video"]).to(dev)
        la = torch.from_numpy(st["lat_audio"]).to(dev)
        return lv, la, lv.to(torch.bfloat16), la.to(torch.bfloat16)

    lv, la, lvb, lab = fresh()
    smp.run(text, lv, la, lvb, lab, mod_all, n_steps)
    lv2, la2, lvb2, lab2 = fresh()
    smp.run(text, lv2, la2, lvb2, lab2, mod_all, n_steps, end_step=2)
    path = str(tmp_path / "sampler_state.npz")
    H3Sampler.save_state(path, 2, lv2, la2)
    del lv2, la2, lvb2, lab2
    s0, lv3, la3, lvb3, lab3 = H3Sampler.load_state(path, dev)
    assert s0 == 2
    smp.run(text, lv3, la3, lvb3, lab3, mod_all, n_steps, start_step=s0)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    assert torch.equal(lv3, lv) and torch.equal(la3, la)
