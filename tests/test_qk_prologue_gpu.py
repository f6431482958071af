"""Q/K RMSNorm + 3-D RoPE in attention's prologue: h3_qkv_qknorm_mrope
without H3_QK_NORM_ROPE_IN_QKV writes q, k raw, and h3_attention without it
normalises and rotates each Q tile once and each K tile as it lands
("MiniMax-H3: native joint audio-video generation" §3.2: per-head RMSNorm,
then the positional encoding, then attention).

Against the oracle: the raw projections against the plain product, the
prologue attention on seeded raw q, k, v against the oracle's rmsnorm +
rope + attention of the same values, and the QKV (raw) -> attention
(prologue) path against the oracle's block path from the same xm; the two
placements on the GPU against each other.

Both placements keep the normalised, rotated q and k in bf16 (the epilogue
in global memory, the prologue in shared memory, the tensor cores' operand
type), and the prologue placement also stores the raw q, k in bf16 between
the two calls.  The oracle takes the same bf16 roundings (O.round_to_bf16)
at those points: near-uniform softmax rows average many values of v, so
their output RMS is small against the rounding of a score, and without them
the attention-level comparison measures bf16 storage, not the kernels."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import H3BlockStep, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
WORKLOADS = [S.WORKLOADS["tiny"], RAGGED]


def _dims(w):
    return h3.make_dims(w.D, w.H, w.F, rope=w.rope_split)


def _pos_dev(pos, Lp):
    p = np.zeros((Lp, 3), np.float32)
    p[:len(pos)] = pos
    return torch.from_numpy(p).to(DEV)


def _raw_qkv(rng, H, L, Lp, scale=1.0):
    """Raw q, k, v rows (bf16-rounded, zero past L) as [H][L_pad][128]."""
    out = []
    for _ in range(3):
        a = S.bf16_round((scale * rng.standard_normal((H, Lp, 128))).astype(np.float32))
        a[:, L:, :] = 0
        out.append(a)
    return out


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_qkv_raw_projection(w):
    """Without the flag the QKV call writes xm Wqkv^T, split into heads, as
    bf16; qn_w, kn_w and pos are not needed."""
    inp = S.make_inputs(w)
    r, _ = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(61 + w.index)
    xm = np.zeros((Lp, w.D), np.float32)
    xm[:L] = S.bf16_round(rng.standard_normal((L, w.D)).astype(np.float32))
    d, rg = _dims(w), h3.h3_make_ranges(*r["count"])
    q, k, v = (torch.empty(w.H, Lp, 128, dtype=torch.bfloat16, device=DEV) for _ in range(3))
    h3.h3_qkv_qknorm_mrope(d, rg, to_dev_bf16(xm, DEV), to_dev_bf16(inp["Wqkv"], DEV), None, None, None, q, k, v,
                           flags=0)
    raw = xm[:L].astype(np.float64) @ inp["Wqkv"].astype(np.float64).T      # [L, 3 I]
    I = w.H * 128
    for part, g in enumerate((q, k, v)):
        ref = raw[:, part * I:(part + 1) * I].reshape(L, w.H, 128)
        gg = to_np(g)
        check_close(gg[:, :L, :].transpose(1, 0, 2), ref, "qkv"[part] + " raw", 3e-2, 3e-3)
        assert np.all(gg[:, L:, :] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_attention_prologue_on_raw_rows(w):
    """Raw seeded q, k (scale 3, so the norm matters), the norm weights and
    the workload's positions: the prologue kernel against rmsnorm, rope and
    attention in the oracle."""
    inp = S.make_inputs(w)
    r, pos = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(71 + w.index)
    q, k, v = _raw_qkv(rng, w.H, L, Lp, scale=3.0)
    d, rg = _dims(w), h3.h3_make_ranges(*r["count"])
    o = torch.empty(Lp, w.H * 128, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, to_dev_bf16(q, DEV), to_dev_bf16(k, DEV), to_dev_bf16(v, DEV), o,
                    qn_w=to_dev_bf16(inp["qn_w"], DEV), kn_w=to_dev_bf16(inp["kn_w"], DEV), pos=_pos_dev(pos, Lp),
                    flags=0)
    assert h3.h3_device_status() == 0
    qo, ko, vo = (a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in (q, k, v))
    R = O.round_to_bf16
    qn = R(O.rope(O.rmsnorm(qo, inp["qn_w"]), pos, w.rope_split))
    kn = R(O.rope(O.rmsnorm(ko, inp["kn_w"]), pos, w.rope_split))
    ref = O.attention(qn, kn, vo)
    got = to_np(o)
    check_close(got[:L], ref, "prologue attention")
    assert np.all(got[L:] == 0)


@pytest.mark.parametrize("L", [1, 127, 129, 3 * 128 + 5, 1000])
def test_attention_prologue_edge_lengths(L):
    """Edge lengths (one token, a partial tile, an odd tile count, one query
    tile in the last CTA) with seeded integer (t, h, w) positions."""
    H = 4
    d = h3.make_dims(320, H, 896)
    rg = h3.h3_make_ranges(L, 0, 0)
    Lp = rg.L_pad
    rng = np.random.default_rng(81 + L)
    pos = rng.integers(0, 64, size=(L, 3)).astype(np.float64)
    q, k, v = _raw_qkv(rng, H, L, Lp, scale=2.0)
    qw = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    kw = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    o = torch.empty(Lp, H * 128, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, to_dev_bf16(q, DEV), to_dev_bf16(k, DEV), to_dev_bf16(v, DEV), o,
                    qn_w=to_dev_bf16(qw, DEV), kn_w=to_dev_bf16(kw, DEV), pos=_pos_dev(pos, Lp), flags=0)
    assert h3.h3_device_status() == 0
    qo, ko, vo = (a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in (q, k, v))
    R = O.round_to_bf16
    ref = O.attention(R(O.rope(O.rmsnorm(qo, qw), pos)), R(O.rope(O.rmsnorm(ko, kw), pos)), vo)
    got = to_np(o)
    check_close(got[:L], ref, f"prologue attention L={L}")
    assert np.all(got[L:] == 0)


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_block_path_both_placements(w):
    """QKV + attention from the same xm with the norm and RoPE in the QKV
    epilogue and in attention's prologue: each against the oracle's path
    (qkv_qknorm_mrope, attention), and the two against each other (they
    differ only by the bf16 rounding of the raw q, k)."""
    inp = S.make_inputs(w)
    st = H3BlockStep(w, device=DEV, weights=inp)
    st.embed(*(to_dev_bf16(inp[kk], DEV) for kk in ("text", "video", "audio")))
    r, pos = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    rng = np.random.default_rng(91 + w.index)
    xm = np.zeros((Lp, w.D), np.float32)
    xm[:L] = S.bf16_round(rng.standard_normal((L, w.D)).astype(np.float32))
    st.xm.copy_(to_dev_bf16(xm, DEV))
    outs = {}
    for name, flags in (("epilogue", h3.H3_QK_NORM_ROPE_IN_QKV), ("prologue", 0)):
        h3.h3_qkv_qknorm_mrope(st.dims, st.ranges, st.xm, st.W["Wqkv"], st.W["qn_w"], st.W["kn_w"], st.pos,
                               st.q, st.k, st.v, flags=flags)
        h3.h3_attention(st.dims, st.ranges, st.q, st.k, st.v, st.o, qn_w=st.W["qn_w"], kn_w=st.W["kn_w"],
                        pos=st.pos, flags=flags)
        assert h3.h3_device_status() == 0
        outs[name] = to_np(st.o).copy()
    R = O.round_to_bf16
    # epilogue placement: q, k normalised and rotated from the fp32
    # accumulator, stored in bf16; v stored in bf16
    qr, kr, vr = O.qkv_qknorm_mrope(xm[:L], inp["Wqkv"], inp["qn_w"], inp["kn_w"], pos, w.H, split=w.rope_split)
    refs = {"epilogue": O.attention(R(qr), R(kr), R(vr))}
    # prologue placement: raw q, k stored in bf16, then normalised and
    # rotated, then stored in bf16 again (shared memory)
    I = w.H * 128
    raw = R(O.linear(xm[:L], inp["Wqkv"]))
    q_raw, k_raw = (raw[:, p * I:(p + 1) * I].reshape(L, w.H, 128) for p in (0, 1))
    refs["prologue"] = O.attention(R(O.rope(O.rmsnorm(q_raw, inp["qn_w"]), pos, w.rope_split)),
                                   R(O.rope(O.rmsnorm(k_raw, inp["kn_w"]), pos, w.rope_split)), R(vr))
    for name, g in outs.items():
        check_close(g[:L], refs[name], f"attention output, norm + RoPE in the {name}")
        assert np.all(g[L:] == 0)
    # the two placements differ by the extra bf16 storage of the raw q, k:
    # a score moves by up to ~2^-9 of |q| |k| / sqrt(128), which the
    # near-uniform rows carry into an output of small RMS
    check_close(outs["prologue"][:L], outs["epilogue"][:L].astype(np.float64), "prologue vs epilogue placement",
                max_rel_rms=0.1)


def test_full_length_prologue_sampled_rows():
    """The prologue kernel at the longest packed length (124,016 tokens, 2
    heads, the 15 s workload's positions), sampled query rows against the
    oracle over all keys."""
    w = S.WORKLOADS["768x1792_15s"]
    H = 2
    r, pos = oracle_ranges_and_pos(w)
    L, Lp = r["L"], r["L_pad"]
    d = h3.make_dims(5376, H, 14336, rope=w.rope_split)
    rg = h3.h3_make_ranges(*r["count"])
    rng = np.random.default_rng(L + 9)
    q, k, v = _raw_qkv(rng, H, L, Lp, scale=2.0)
    qw = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    kw = S.bf16_round((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    o = torch.empty(Lp, H * 128, dtype=torch.bfloat16, device=DEV)
    h3.h3_attention(d, rg, to_dev_bf16(q, DEV), to_dev_bf16(k, DEV), to_dev_bf16(v, DEV), o,
                    qn_w=to_dev_bf16(qw, DEV), kn_w=to_dev_bf16(kw, DEV), pos=_pos_dev(pos, Lp), flags=0)
    assert h3.h3_device_status() == 0
    rows = np.unique(np.concatenate([S.random_rows(L, 48, seed=L + 9), [0, 1, L // 2, L - 2, L - 1]]))
    got = to_np(o[torch.from_numpy(rows).to(DEV)])
    qo, ko, vo = (a[:, :L, :].transpose(1, 0, 2).astype(np.float64) for a in (q, k, v))
    R = O.round_to_bf16
    qn = R(O.rope(O.rmsnorm(qo[rows], qw), pos[rows], w.rope_split))
    kn = R(O.rope(O.rmsnorm(ko, kw), pos, w.rope_split))
    ref = O.attention_rows(qn, kn, vo)
    check_close(got, ref, "prologue attention L=124016 rows")
    assert float(o[L:].float().abs().max()) == 0.0


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_block_with_prologue_placement(w):
    """The whole block with the norm and RoPE in attention's prologue
    (h3_block_forward and the pipeline with flags 0) against the oracle's
    block: the block bound on the output, the branch-delta bound of the
    default placement on its delta."""
    inp = S.make_inputs(w)
    st = H3BlockStep(w, device=DEV, weights=inp)
    st.qk_flags = 0
    st.embed(*(to_dev_bf16(inp[kk], DEV) for kk in ("text", "video", "audio")))
    mod = torch.from_numpy(inp["mod"]).to(DEV)
    r, pos = oracle_ranges_and_pos(w)
    L = r["L"]
    x0_dev = st.x.clone()
    st.block(mod)
    assert h3.h3_device_status() == 0
    x_pipe = to_np(st.x)[:L]
    # the same block through the C-ABI block call with flags 0
    st.x.copy_(x0_dev)
    h3.h3_block_forward(st.dims, st.ranges, st.x, mod, st.pos, h3.block_weights(st.W),
                        h3.block_buffers(st.xm, st.q, st.k, st.v, st.o, st.ws), flags=0)
    assert h3.h3_device_status() == 0
    assert np.array_equal(to_np(st.x)[:L], x_pipe)
    x0 = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    ref = O.block_forward(x0, inp["mod"], r, pos, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"], inp["Wgu"],
                          inp["Wd"], w.H)
    check_close(x_pipe, ref, "block output, prologue placement")
    check_close(x_pipe - x0, ref - x0, "block delta, prologue placement", max_rel_rms=5e-2)
