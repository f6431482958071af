"""GPU parity: every C-ABI call against the float64 oracle.

Both sides always start from the same seeded, bf16-rounded inputs; no oracle
input is ever taken from the CUDA path.  Each call is tested on its own
(seeded inputs for that call) and the whole step end to end (seeded raw
latents and features in, oracle recomputes everything).  Integer, byte and
index work is compared bit-exactly; floating point within the block tolerance
of parity_util.check_close unless a test states a tighter bound.
"""
import dataclasses
import functools

import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import H3BlockStep, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu

WORKLOADS = [S.WORKLOADS["tiny"], RAGGED]
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


@functools.lru_cache(maxsize=1)
def _inputs(w, weights=True):
    return S.make_inputs(w, weights=weights)


def _setup(w, weights=True):
    inp = _inputs(w, weights)
    st = H3BlockStep(w, weights=inp if weights else None)
    text, video, audio = (to_dev_bf16(inp[k], st.device) for k in ("text", "video", "audio"))
    mod = torch.from_numpy(inp["mod"]).to(st.device)
    return inp, st, text, video, audio, mod


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def _rows_stream(w, rng, L, Lp, D, std=1.0, bf16=False):
    """Seeded [L_pad, D] activations, zero padding rows."""
    a = np.zeros((Lp, D), np.float32)
    a[:L] = rng.standard_normal((L, D), dtype=np.float32) * np.float32(std)
    return S.bf16_round(a) if bf16 else a


# ---------------------------------------------------------------- A1 + A2

@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_embed_pack_bit_exact_packing_and_projection(w):
    inp, st, text, video, audio, mod = _setup(w)
    st.embed(text, video, audio)
    torch.cuda.synchronize()
    r, pos = oracle_ranges_and_pos(w)
    assert st.ranges.as_dict() == r
    L = r["L"]
    assert np.array_equal(to_np(st.patches), O.patchify(inp["video"]))                 # integer gather
    assert np.array_equal(st.pos.cpu().numpy()[:L], pos.astype(np.float32))           # fp32 of oracle values
    assert np.all(st.pos.cpu().numpy()[L:] == 0)
    mids = st.mod_ids.cpu().numpy()
    assert np.array_equal(mids[:L], O.modality_of_rows(r).astype(np.uint8))
    assert np.all(mids[L:] == 255)
    x = to_np(st.x)
    ref = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    check_close(x[:L], ref, "embed x", 1e-4, 1e-5)          # fp32 accumulation of exact bf16 products
    assert np.all(x[L:] == 0)


# ---------------------------------------------------------------- each call on seeded inputs

@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_ln_modulate_seeded(w):
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(31 + w.index)
    x = _rows_stream(w, rng, L, Lp, w.D) * 3.0 + 0.5
    x[L:] = 0
    mod = (rng.standard_normal((3, 6, w.D)) * 0.1).astype(np.float32)
    d, rg = h3.make_dims(w.D, w.H, w.F), h3.h3_make_ranges(*r["count"])
    xm = torch.empty(Lp, w.D, dtype=torch.bfloat16, device=DEV)
    for br in (h3.H3_MSA, h3.H3_MLP):
        h3.h3_adaln_norm_modulate(d, rg, _f32(x), _f32(mod), br, xm)
        g = to_np(xm)
        # bf16 output: rounding alone is up to 2^-8 |y|, ~0.018 RMS at the
        # 4.5-sigma tail of a Gaussian-like output, so the block bound applies
        check_close(g[:L], O.adaln_modulate(x[:L], mod, r, br), f"ln_modulate branch {br}", 3e-2, 3e-3)
        assert np.all(g[L:] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_qkv_qknorm_mrope_seeded(w):
    inp, st, text, video, audio, mod = _setup(w)
    st.embed(text, video, audio)                       # GPU positions for the GPU side
    r, pos = oracle_ranges_and_pos(w)                  # oracle positions for the oracle side
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(41 + w.index)
    xm = _rows_stream(w, rng, L, Lp, w.D, bf16=True)
    st.xm.copy_(to_dev_bf16(xm, DEV))
    h3.h3_qkv_qknorm_mrope(st.dims, st.ranges, st.xm, st.W["Wqkv"], st.W["qn_w"], st.W["kn_w"], st.pos,
                           st.q, st.k, st.v)
    ref = O.qkv_qknorm_mrope(xm[:L], inp["Wqkv"], inp["qn_w"], inp["kn_w"], pos, w.H)
    for name, g, o in zip("qkv", (st.q, st.k, st.v), ref):
        gg = to_np(g)
        check_close(gg[:, :L, :].transpose(1, 0, 2), o, name, 3e-2, 3e-3)      # bf16 output (see LN test)
        assert np.all(gg[:, L:, :] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_attention_seeded(w):
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(51 + w.index)
    q, k, v = (S.bf16_round(rng.standard_normal((w.H, Lp, 128), dtype=np.float32)) for _ in range(3))
    for a in (q, k, v):
        a[:, L:, :] = 0
    d, rg = h3.make_dims(w.D, w.H, w.F), h3.h3_make_ranges(*r["count"])
    o = torch.empty(Lp, w.I, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, to_dev_bf16(q, DEV), to_dev_bf16(k, DEV), to_dev_bf16(v, DEV), o)
    g = to_np(o)
    ref = O.attention(*(a[:, :L, :].transpose(1, 0, 2) for a in (q, k, v)))
    # Block tolerance: rounding P and o to bf16 alone (float64 emulation on
    # the CPU) gives up to 0.024 * RMS at L = 128.
    check_close(g[:L], ref, "attention")
    assert np.all(g[L:] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_gated_residual_seeded(w):
    inp = _inputs(w)
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(61 + w.index)
    x = _rows_stream(w, rng, L, Lp, w.D)
    o = _rows_stream(w, rng, L, Lp, w.I, bf16=True)
    d, rg = h3.make_dims(w.D, w.H, w.F), h3.h3_make_ranges(*r["count"])
    xg = _f32(x)
    h3.h3_gated_residual(d, rg, xg, to_dev_bf16(o, DEV), to_dev_bf16(inp["Wo"], DEV), _f32(inp["mod"]), h3.H3_MSA)
    g = to_np(xg)
    ref = O.gated_residual(x[:L], o[:L], inp["Wo"], inp["mod"], r)
    check_close(g[:L] - x[:L], ref - x[:L], "gated residual delta", 1e-3, 1e-4)   # fp32 accumulate, no rounding
    assert np.all(g[L:] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_ffn_swiglu_seeded(w):
    inp = _inputs(w)
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(71 + w.index)
    x = _rows_stream(w, rng, L, Lp, w.D)
    xm = _rows_stream(w, rng, L, Lp, w.D, bf16=True)
    d, rg = h3.make_dims(w.D, w.H, w.F), h3.h3_make_ranges(*r["count"])
    xg = _f32(x)
    ws = torch.empty(Lp, w.F, dtype=torch.bfloat16, device=DEV)
    h3.h3_ffn_swiglu(d, rg, xg, to_dev_bf16(xm, DEV), to_dev_bf16(inp["Wgu"], DEV), to_dev_bf16(inp["Wd"], DEV),
                     _f32(inp["mod"]), ws)
    g = to_np(xg)
    ref = O.ffn_swiglu(x[:L], xm[:L], inp["Wgu"], inp["Wd"], inp["mod"], r)
    check_close(g[:L] - x[:L], ref - x[:L], "ffn delta")      # SiLU*up rounded to bf16
    assert np.all(g[L:] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_head_unpack_seeded(w):
    inp = _inputs(w)
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(81 + w.index)
    x = _rows_stream(w, rng, L, Lp, w.D)
    d, rg = h3.make_dims(w.D, w.H, w.F), h3.h3_make_ranges(*r["count"])
    hn = torch.empty(Lp, w.D, dtype=torch.bfloat16, device=DEV)
    vv = torch.empty(w.T_lat, w.H_lat, w.W_lat, w.C_lat, device=DEV)
    va = torch.empty(w.audio_channels, w.n_audio, w.C_audio, device=DEV)
    h3.h3_head_unpack(d, rg, _f32(x), to_dev_bf16(inp["W_vhead"], DEV), to_dev_bf16(inp["W_ahead"], DEV),
                      tuple(vv.shape), tuple(va.shape), hn, vv, va)
    rv, ra = O.head_unpack(x[:L], r, inp["W_vhead"], inp["W_ahead"], w.T_lat, w.H_lat, w.W_lat, w.audio_channels,
                           w.n_audio)
    check_close(to_np(vv), rv, "video head", 3e-2, 3e-3)       # bf16 normalised input (see LN test)
    check_close(to_np(va), ra, "audio head", 3e-2, 3e-3)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_head_euler_fused(w):
    """h3_head_euler (the Euler step in the head GEMMs' epilogues) equals
    h3_head_unpack followed by h3_euler_step on each latent bit for bit,
    writes the bf16 copies of the updated latents, and matches the oracle's
    head + Euler step (each modality on its own shifted schedule)."""
    inp = _inputs(w)
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(83 + w.index)
    x = _rows_stream(w, rng, L, Lp, w.D)
    lv0 = rng.standard_normal((w.T_lat, w.H_lat, w.W_lat, w.C_lat)).astype(np.float32)
    la0 = rng.standard_normal((w.audio_channels, w.n_audio, w.C_audio)).astype(np.float32)
    d, rg = h3.make_dims(w.D, w.H, w.F), h3.h3_make_ranges(*r["count"])
    sv = h3.h3_sigma_schedule(8, 12.0)
    sa = h3.h3_sigma_schedule(8, 3.0)
    Wv, Wa = to_dev_bf16(inp["W_vhead"], DEV), to_dev_bf16(inp["W_ahead"], DEV)
    hn = torch.empty(Lp, w.D, dtype=torch.bfloat16, device=DEV)
    shapes = ((w.T_lat, w.H_lat, w.W_lat, w.C_lat), (w.audio_channels, w.n_audio, w.C_audio))
    for s in (0, 5):
        lv, la = _f32(lv0), _f32(la0)
        lv16 = torch.full(lv.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
        la16 = torch.full(la.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
        h3.h3_head_euler(d, rg, _f32(x), Wv, Wa, *shapes, hn, lv, la, (sv[s], sv[s + 1]), (sa[s], sa[s + 1]),
                         lv16, la16)
        # unfused reference path through the library
        vv, va = torch.empty_like(lv), torch.empty_like(la)
        h3.h3_head_unpack(d, rg, _f32(x), Wv, Wa, *shapes, hn, vv, va)
        lv_ref, la_ref = _f32(lv0), _f32(la0)
        h3.h3_euler_step(lv_ref, vv, sv[s], sv[s + 1])
        h3.h3_euler_step(la_ref, va, sa[s], sa[s + 1])
        torch.cuda.synchronize()
        assert torch.equal(lv, lv_ref) and torch.equal(la, la_ref)
        assert torch.equal(lv16, lv.to(torch.bfloat16)) and torch.equal(la16, la.to(torch.bfloat16))
        rv, ra = O.head_unpack(x[:L], r, inp["W_vhead"], inp["W_ahead"], w.T_lat, w.H_lat, w.W_lat,
                               w.audio_channels, w.n_audio)
        ov = O.euler_step(lv0, rv, np.float64(np.float32(sv[s])), np.float64(np.float32(sv[s + 1])))
        oa = O.euler_step(la0, ra, np.float64(np.float32(sa[s])), np.float64(np.float32(sa[s + 1])))
        # the latent change (the head's contribution) at the head's bound
        check_close(to_np(lv) - lv0, ov - lv0, f"video latent change, step {s}", 3e-2, 3e-3)
        check_close(to_np(la) - la0, oa - la0, f"audio latent change, step {s}", 3e-2, 3e-3)
    # without bf16 copies (NULL) the latents are the same
    lv, la = _f32(lv0), _f32(la0)
    h3.h3_head_euler(d, rg, _f32(x), Wv, Wa, *shapes, hn, lv, la, (sv[5], sv[6]), (sa[5], sa[6]))
    torch.cuda.synchronize()
    assert torch.equal(lv, lv_ref) and torch.equal(la, la_ref)


def test_euler_and_schedule_seeded():
    rng = np.random.default_rng(91)
    lat = rng.standard_normal(1000003).astype(np.float32)        # odd length: vector body + scalar tail
    vel = rng.standard_normal(1000003).astype(np.float32)
    for shift in (12.0, 3.0):
        sig = np.array(h3.h3_sigma_schedule(8, shift), np.float32)
        assert np.array_equal(sig, O.sigma_schedule(8, shift).astype(np.float32))
        for i in (0, 3, 7):
            g = _f32(lat)
            h3.h3_euler_step(g, _f32(vel), float(sig[i]), float(sig[i + 1]))
            ref = O.euler_step(lat, vel, np.float64(sig[i]), np.float64(sig[i + 1]))
            check_close(to_np(g), ref, f"euler shift {shift} step {i}", 1e-6, 1e-7)
    g = _f32(lat)
    h3.h3_euler_step(g, _f32(vel), 0.7, 0.0)                    # sigma 0.7 -> 0: the clean latent
    check_close(to_np(g), O.clean_latent(lat, vel, np.float64(np.float32(0.7))), "clean latent", 1e-6, 1e-7)


# ---------------------------------------------------------------- end to end

@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_step_end_to_end_against_oracle(w):
    """Raw seeded latents and features in; the oracle recomputes packing,
    projections, the block, the head and the Euler step from the same
    inputs."""
    inp, st, text, video, audio, mod = _setup(w)
    r, pos = oracle_ranges_and_pos(w)
    L = r["L"]
    rng = np.random.default_rng(101 + w.index)
    lat_v = rng.standard_normal(st.v_video.shape).astype(np.float32)
    lat_a = rng.standard_normal(st.v_audio.shape).astype(np.float32)
    gv, ga = _f32(lat_v), _f32(lat_a)
    sv, sa = O.sigma_schedule(8, 12.0), O.sigma_schedule(8, 3.0)
    st.embed(text, video, audio)
    st.block(mod)
    x2 = to_np(st.x)[:L]
    st.head()
    st.euler(gv, ga, (float(sv[2]), float(sv[3])), (float(sa[2]), float(sa[3])))
    x0 = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    ref = O.block_forward(x0, inp["mod"], r, pos, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"], inp["Wgu"],
                          inp["Wd"], w.H)
    check_close(x2, ref, "block output")
    # The branch delta is checked too, so that the residual cannot mask a
    # branch error.  Its max bound follows from the bf16 operands: rounding
    # xm, q/k/v, P, o and the SwiGLU product to bf16 at exactly the points this
    # path does, in float64 on the CPU, already gives max|err| = 0.030 *
    # RMS(delta) on the ragged workload (mean rel 3.1e-3); 5e-2 leaves room
    # for fp32 accumulation order and ex2.approx.
    check_close(x2 - x0, ref - x0, "block delta", max_rel_rms=5e-2)
    vv, va = O.head_unpack(ref, r, inp["W_vhead"], inp["W_ahead"], w.T_lat, w.H_lat, w.W_lat, w.audio_channels,
                           w.n_audio)
    check_close(to_np(st.v_video), vv, "video velocity")
    check_close(to_np(st.v_audio), va, "audio velocity")
    ev = O.euler_step(lat_v, vv, np.float32(sv[2]), np.float32(sv[3]))
    ea = O.euler_step(lat_a, va, np.float32(sa[2]), np.float32(sa[3]))
    check_close(to_np(gv), ev, "video latent after Euler")
    check_close(to_np(ga), ea, "audio latent after Euler")


def test_zero_modulation_block_is_bit_exact_identity():
    w = S.WORKLOADS["tiny"]
    inp, st, text, video, audio, mod = _setup(w)
    st.embed(text, video, audio)
    x0 = st.x.clone()
    st.block(torch.zeros_like(mod))
    torch.cuda.synchronize()
    assert torch.equal(st.x, x0)
    r, _ = oracle_ranges_and_pos(w)
    for m in range(3):                   # gate 0 on one modality: exactly that range unchanged
        st.x.copy_(x0)
        m2 = mod.clone()
        m2[m, 2] = 0
        m2[m, 5] = 0
        st.block(m2)
        torch.cuda.synchronize()
        s, c = r["start"][m], r["count"][m]
        assert torch.equal(st.x[s:s + c], x0[s:s + c])
        for mm in (mm for mm in range(3) if mm != m):
            s2, c2 = r["start"][mm], r["count"][mm]
            assert bool((st.x[s2:s2 + c2] != x0[s2:s2 + c2]).any(dim=1).all())


def test_block_is_deterministic():
    inp, st, text, video, audio, mod = _setup(RAGGED)
    outs = []
    for _ in range(2):
        st.embed(text, video, audio)
        st.block(mod)
        st.head()
        torch.cuda.synchronize()
        outs.append((st.x.clone(), st.v_video.clone(), st.v_audio.clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_attention_edge_lengths():
    """L = 1 (one key: output = v), one full tile, one tile + 1, an odd number
    of query tiles (the last CTA's second tile is a duplicate, not stored)."""
    H = 4
    for L in (1, 127, 128, 129, 3 * 128 + 5):
        d = h3.make_dims(320, H, 896)
        rg = h3.h3_make_ranges(L, 0, 0)
        Lp = rg.L_pad
        rng = np.random.default_rng(L)
        qkv = [S.bf16_round(rng.standard_normal((H, Lp, 128), dtype=np.float32)) for _ in range(3)]
        o = torch.empty(Lp, H * 128, dtype=torch.bfloat16, device=DEV)
        h3.h3_attention(d, rg, *(to_dev_bf16(a, DEV) for a in qkv), o)
        got = to_np(o)
        ref = O.attention(*(a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in qkv))
        check_close(got[:L], ref, f"attention L={L}")
        assert np.all(got[L:] == 0)
        if L == 1:
            assert np.allclose(got[0], qkv[2][:, 0, :].reshape(-1), rtol=1e-2, atol=1e-2)


@pytest.mark.parametrize("kind", ["ramp", "spike_last", "spike_second_half"])
def test_attention_reference_moves(kind):
    """Scores that grow along the keys, far past the first key tile's row max:
    the kernel's reference (the first tile's max) must move, with O and the
    running sums rescaled, in either 64-key half of a tile.  ramp: key norms
    grow 7x over the sequence; spike_last: the last (partial) key tile scaled
    30x (p would overflow fp32 against the old reference); spike_second_half:
    keys [64, 128) of an interior tile scaled 30x (the first half's PV is
    already issued when the second half moves the reference)."""
    H, L = 4, 1000
    d = h3.make_dims(320, H, 896)
    rg = h3.h3_make_ranges(L, 0, 0)
    Lp = rg.L_pad
    rng = np.random.default_rng({"ramp": 1, "spike_last": 2, "spike_second_half": 3}[kind])
    q, k, v = (rng.standard_normal((H, Lp, 128), dtype=np.float32) for _ in range(3))
    if kind == "ramp":
        k *= (1 + 6 * np.arange(Lp, dtype=np.float32) / L)[None, :, None]
    elif kind == "spike_last":
        k[:, (L - 1) // 128 * 128:] *= 30
    else:
        k[:, 3 * 128 + 64: 4 * 128] *= 30
    q, k, v = (S.bf16_round(a) for a in (q, k, v))
    for a in (q, k, v):
        a[:, L:, :] = 0
    o = torch.empty(Lp, H * 128, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, *(to_dev_bf16(a, DEV) for a in (q, k, v)), o)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    got = to_np(o)
    ref = O.attention(*(a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in (q, k, v)))
    check_close(got[:L], ref, f"attention ({kind})")
    assert np.all(got[L:] == 0)


def _normalised(rng, H, Lp, w):
    """Rows as the QKV call writes them: RMS-normalised, scaled by the norm
    weight w, rounded to bf16."""
    x = rng.standard_normal((H, Lp, 128))
    return S.bf16_round((x / np.sqrt((x * x).mean(-1, keepdims=True) + 1e-6) * w).astype(np.float32))


@pytest.mark.parametrize("L", [1, 64, 127, 128, 129, 3 * 128 + 5, 1000])
def test_attention_split_normalised(L):
    """Normalised q, k with their norm weights: the split-softmax kernel
    (exponentials against the static bound, each row over two warps), down to
    one key, a half-empty key tile and an odd query-tile count."""
    H = 4
    d = h3.make_dims(320, H, 896)
    rg = h3.h3_make_ranges(L, 0, 0)
    Lp = rg.L_pad
    rng = np.random.default_rng(700 + L)
    qn = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    kn = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    q, k = _normalised(rng, H, Lp, qn), _normalised(rng, H, Lp, kn)
    v = S.bf16_round(rng.standard_normal((H, Lp, 128), dtype=np.float32))
    for a in (q, k, v):
        a[:, L:, :] = 0
    o = torch.full((Lp, H * 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, *(to_dev_bf16(a, DEV) for a in (q, k, v)), o, qn_w=to_dev_bf16(qn, DEV),
                    kn_w=to_dev_bf16(kn, DEV))
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    got = to_np(o)
    ref = O.attention(*(a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in (q, k, v)))
    check_close(got[:L], ref, f"split attention L={L}")
    assert np.all(got[L:] == 0)


@pytest.mark.parametrize("kind", ["far_above", "far_below", "wide_bound"])
def test_attention_split_falls_back(kind):
    """Norm weights given but the bound does not hold, or is too wide: the
    CTAs concerned are recomputed by the general kernel and the result is the
    oracle's.  far_above: some keys 30x longer than normalised rows (scores
    far above the bound); far_below: every key opposite to every query and 10x
    longer (every p would flush to 0); wide_bound: norm weights near 2.5
    (scores up to +-100 in log2 units, past the fp32 range of the exponentials
    against the bound)."""
    H, L = 4, 1000
    d = h3.make_dims(320, H, 896)
    rg = h3.h3_make_ranges(L, 0, 0)
    Lp = rg.L_pad
    rng = np.random.default_rng({"far_above": 11, "far_below": 12, "wide_bound": 13}[kind])
    scale = 2.5 if kind == "wide_bound" else 1.0
    qn = S.bf16_round((scale * (1 + 0.05 * rng.standard_normal(128))).astype(np.float32))
    kn = S.bf16_round((scale * (1 + 0.05 * rng.standard_normal(128))).astype(np.float32))
    q, k = _normalised(rng, H, Lp, qn), _normalised(rng, H, Lp, kn)
    if kind == "far_above":
        k[:, 3 * 128 + 64: 4 * 128] = S.bf16_round(30 * k[:, 3 * 128 + 64: 4 * 128])
    elif kind == "far_below":
        q[:] = q[:, :1, :]
        k[:] = S.bf16_round((-10 * q[:, :1, :]).astype(np.float32))
    v = S.bf16_round(rng.standard_normal((H, Lp, 128), dtype=np.float32))
    for a in (q, k, v):
        a[:, L:, :] = 0
    o = torch.empty(Lp, H * 128, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, *(to_dev_bf16(a, DEV) for a in (q, k, v)), o, qn_w=to_dev_bf16(qn, DEV),
                    kn_w=to_dev_bf16(kn, DEV))
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    got = to_np(o)
    ref = O.attention(*(a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in (q, k, v)))
    check_close(got[:L], ref, f"split attention fallback ({kind})")
    assert np.all(got[L:] == 0)


# ---------------------------------------------------------------- full sizes, sampled outputs

FULL = [S.WORKLOADS["768sq_2s"], S.WORKLOADS["768x1344_5s"]]


def _sample_rows(L, k, seed):
    edge = [0, 1, L // 2, L - 2, L - 1]
    rows = np.unique(np.concatenate([S.random_rows(L, k, seed), edge]))
    return rows[rows < L]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_block_sampled_rows(w):
    """The bench's workloads at full width in the bench's launch configuration:
    GPU embed + block; the oracle computes sampled output rows from the same
    raw inputs (K/V for every token, per head)."""
    inp, st, text, video, audio, mod = _setup(w)
    r, pos = oracle_ranges_and_pos(w)
    L = r["L"]
    st.embed(text, video, audio)
    st.block(mod)
    torch.cuda.synchronize()
    rows = _sample_rows(L, 12, seed=w.index)
    x2 = to_np(st.x[torch.from_numpy(rows).to(DEV)])
    x0 = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    ref, _ = O.block_forward_rows(x0, inp["mod"], r, pos, rows, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"],
                                  inp["Wgu"], inp["Wd"], w.H)
    check_close(x2, ref, f"{w.name} block output rows")
    check_close(x2 - x0[rows], ref - x0[rows], f"{w.name} block delta rows", max_rel_rms=5e-2)


@pytest.mark.parametrize("L,H", [(7904, 56), (32160, 8), (124016, 2)], ids=["768sq_2s", "768x1344_5s", "768x1792_15s"])
def test_full_length_attention_sampled_rows(L, H):
    """Attention at each workload's packed length (fewer heads at the longer
    lengths: heads are independent CTAs), sampled query rows against all keys."""
    d = h3.make_dims(5376, H, 14336)
    rg = h3.h3_make_ranges(L, 0, 0)
    Lp = rg.L_pad
    rng = np.random.default_rng(L)
    # normalised q, k with their norm weights (the split-softmax kernel, as the
    # block runs it)
    qn = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    kn = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    qkv = [_normalised(rng, H, Lp, qn), _normalised(rng, H, Lp, kn),
           S.bf16_round(rng.standard_normal((H, Lp, 128), dtype=np.float32))]
    for a in qkv:
        a[:, L:, :] = 0
    o = torch.empty(Lp, H * 128, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, *(to_dev_bf16(a, DEV) for a in qkv), o, qn_w=to_dev_bf16(qn, DEV),
                    kn_w=to_dev_bf16(kn, DEV))
    rows = _sample_rows(L, 48, seed=L)
    got = to_np(o[torch.from_numpy(rows).to(DEV)])
    q, k, v = (a[:, :L, :].transpose(1, 0, 2) for a in qkv)
    ref = O.attention_rows(q[rows], k, v)
    check_close(got, ref, f"attention L={L} rows")
    if Lp > L:
        assert float(o[L:].float().abs().max()) == 0.0


# The 15 s workload's token layout (512 text, 2 x 600 audio, 91 x 24 x 56
# video tokens: L = 124,016, L_pad = 124,032, 969 query tiles, so the last
# attention CTA holds one tile) at the tiny widths, so that the oracle can
# follow sampled rows through the whole block at that length.
LONG_TINY = dataclasses.replace(S.WORKLOADS["768x1792_15s"], name="768x1792_15s_tiny_width", index=30, D=320, H=4,
                                F=896, D_text=256)


def test_long_sequence_block_tiny_width_sampled_rows():
    """The whole block (embed, LN + modulate, QKV + RMSNorm + RoPE,
    attention over 124,016 tokens, gated out-projection, SwiGLU FFN) at the
    longest packed length with the tiny widths; the oracle follows sampled
    rows (K and V of every token, per head), including the first and last
    rows of every modality range and rows of the last, single-tile CTA."""
    w = LONG_TINY
    inp, st, text, video, audio, mod = _setup(w)
    r, pos = oracle_ranges_and_pos(w)
    L = r["L"]
    assert L == 124016 and r["L_pad"] // 128 % 2 == 1
    st.embed(text, video, audio)
    x0_gpu = to_np(st.x[:L])
    st.block(mod)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    edges = [s + c - 1 for s, c in zip(r["start"], r["count"])] + list(r["start"]) + [L - 128, L - 3]
    rows = np.unique(np.concatenate([_sample_rows(L, 24, seed=1792), edges]))
    x0 = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    check_close(x0_gpu[rows], x0[rows], "embedded rows", 1e-4, 1e-5)
    ref, _ = O.block_forward_rows(x0, inp["mod"], r, pos, rows, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"],
                                  inp["Wgu"], inp["Wd"], w.H)
    x2 = to_np(st.x[torch.from_numpy(rows).to(DEV)])
    check_close(x2, ref, "124k-token block output rows")
    check_close(x2 - x0[rows], ref - x0[rows], "124k-token block delta rows", max_rel_rms=5e-2)


def test_full_length_qkv_sampled_rows():
    """QKV + Q/K RMSNorm + RoPE at the longest packed length (124,016 tokens,
    969 row tiles), sampled rows, real positions of that workload."""
    w = S.WORKLOADS["768x1792_15s"]
    inp = _inputs(w)
    r, pos = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    st = H3BlockStep(w, weights=inp)
    st.embed(*(to_dev_bf16(inp[k], st.device) for k in ("text", "video", "audio")))
    rng = np.random.default_rng(1793)
    rows = _sample_rows(L, 24, seed=1793)
    xm_rows = S.bf16_round(rng.standard_normal((len(rows), w.D), dtype=np.float32))
    st.xm.zero_()
    st.xm[torch.from_numpy(rows).to(DEV)] = to_dev_bf16(xm_rows, DEV)
    h3.h3_qkv_qknorm_mrope(st.dims, st.ranges, st.xm, st.W["Wqkv"], st.W["qn_w"], st.W["kn_w"], st.pos,
                           st.q, st.k, st.v)
    ref = O.qkv_qknorm_mrope(xm_rows, inp["Wqkv"], inp["qn_w"], inp["kn_w"], pos[rows], w.H)
    ridx = torch.from_numpy(rows).to(DEV)
    for name, g, o in zip("qkv", (st.q, st.k, st.v), ref):
        gg = to_np(g[:, ridx, :]).transpose(1, 0, 2)
        check_close(gg, o, f"{name} rows at L={L}", 3e-2, 3e-3)               # bf16 output (see LN test)


def test_device_status_clean_after_work():
    assert h3.h3_device_status() == 0
