"""Float64 CPU oracle of the FP8 (e4m3) GEMM path.  TEST INFRASTRUCTURE ONLY.

Only tests/, the graft smoke entry and the bench's CPU-baseline leg may import
this module.  It shares no code with the CUDA library.

The pages say only that the community ships FP8 / INT4 quantisations of the
trunk ("H3's omni-modal ambition" (0539edu.com), the ecosystem paragraph);
they fix no format.  This module states the scheme the FP8 path computes:

  * e4m3 as defined by the OCP 8-bit floating point specification (OFP8):
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field
    0 holds the subnormals m/8 * 2^-6; the all-ones pattern S.1111.111 is
    NaN and there is no infinity, so the largest finite magnitude is
    1.75 * 2^8 = 448.
  * Encoding rounds to the nearest representable value, ties to the even
    code (mantissa LSB 0), after saturating |x| to 448; the code's sign bit
    is the input's sign bit (so -0 and negative values that round to zero
    give 0x80).
  * Row scaling: for a row r of an [M, K] matrix, amax = max |r|;
    rscale = fp32(448 / amax) and scale = fp32(amax / 448) (both IEEE fp32
    divisions); codes = e4m3(fp32(r * rscale)); a zero row has rscale =
    scale = 0.  The float decisions are taken in fp32 on both sides.
  * Activations are scaled per token (row of A), weights per output channel
    (row of the [out, in] weight), and an FP8 GEMM is
    out[m, n] = scale_a[m] * scale_b[n] * sum_k dec(qa[m, k]) dec(qb[n, k]),
    after which the bf16 path's epilogues apply unchanged.
  * Optionally (H3_QK_E4M3) q and k reach attention as e4m3 codes with one
    static scale each, taken from the bound that RMSNorm then RoPE put on a
    head row: every element is at most sqrt(128) max|w| in magnitude (w the
    norm weight), so s = fp32(fp32(sqrt(128) * max|w|) / 448) and
    code = e4m3(fp32(x * fp32(448 / fp32(sqrt(128) * max|w|)))), in fp32
    arithmetic with sqrt(128) as the fp32 constant 11.3137085.  Attention
    then sees S = s_q s_k sum dec(q) dec(k).

Parity pins (tests/test_oracle_fp8_pins.py): the value table against the
closed form of every code; encoding against a brute-force nearest search and
against torch's float8_e4m3fn conversion; saturation; ties; the row-scaling
invariants (the row max maps to code 0x7e, reconstruction error within half
an e4m3 step); the FP8 GEMM against the float64 product of decoded values
written out as an explicit triple loop on a tiny case.
"""
from __future__ import annotations

import numpy as np

from . import h3_oracle as O

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of an e4m3 code (OFP8); NaN for S.1111.111."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """float64 value of every code 0..255 (NaN at 0x7f and 0xff)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


_POS = None  # values of codes 0..126 (all finite non-negative values, ascending)


def _pos_values() -> np.ndarray:
    global _POS
    if _POS is None:
        _POS = e4m3_table()[:127].copy()
    return _POS


def e4m3_encode(x) -> np.ndarray:
    """Round-to-nearest-even, saturating encoding of x (any float array).

    The nearest representable magnitude is found by search over the 127
    finite non-negative values; a tie goes to the even code."""
    x = np.asarray(x, dtype=np.float64)
    pos = _pos_values()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(pos, a, side="left")  # first value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - pos[lo]
    d_hi = pos[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a == pos[hi], hi, code).astype(np.uint8)  # exact hits
    # the sign bit is the input's sign bit (a negative value that rounds to
    # zero, and -0, give the negative zero 0x80)
    code = np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)
    return code


def e4m3_decode(codes) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, dtype=np.uint8)]


def quantize_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 quantisation of a 2-D array (values taken as fp32).

    Returns (codes uint8 [M, K], scale float32 [M]) with
    dec(codes[r]) * scale[r] ~= x[r].  Rows are processed in blocks only to
    bound memory; every row follows the definition above on its own."""
    x32 = np.asarray(x, dtype=np.float32)
    M = x32.shape[0]
    codes = np.zeros(x32.shape, dtype=np.uint8)
    scale = np.zeros(M, dtype=np.float32)
    if x32.size == 0:
        return codes, scale
    for r0 in range(0, M, 1024):
        blk = x32[r0:r0 + 1024]
        amax = np.max(np.abs(blk), axis=1).astype(np.float32)
        nz = amax > 0
        safe = np.where(nz, amax, np.float32(1)).astype(np.float32)
        rscale = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(0)).astype(np.float32)
        scale[r0:r0 + len(blk)] = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(0))
        y = (blk * rscale[:, None]).astype(np.float32)
        c = e4m3_encode(y)
        c[~nz] = 0  # zero row: scale 0, codes 0
        codes[r0:r0 + len(blk)] = c
    return codes, scale


def dequantize_rows(codes, scale) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]


def gemm_e4m3(qa, sa, qb, sb) -> np.ndarray:
    """out[m, n] = sa[m] sb[n] sum_k dec(qa[m, k]) dec(qb[n, k]), float64."""
    return np.asarray(sa, np.float64)[:, None] * (e4m3_decode(qa) @ e4m3_decode(qb).T) * \
        np.asarray(sb, np.float64)[None, :]


# --------------------------------------------------------------------------
# The block's GEMM calls with e4m3 operands (epilogues as in the bf16 path)
# --------------------------------------------------------------------------

def quantize_weight(W) -> tuple[np.ndarray, np.ndarray]:
    """Per-output-channel quantisation of an [out, in] weight."""
    return quantize_rows(W)


QK_SQRT128 = np.float32(11.3137085)


def qk_code_scale(w) -> tuple[np.float32, np.float32]:
    """(inverse scale, scale) of the e4m3 codes of q or k rows normalised
    with weight w (see the module docstring), in fp32."""
    m = np.float32(np.max(np.abs(np.asarray(w, np.float32))))
    if m == 0:
        # an all-zero weight makes every element 0: codes 0 and scale 0
        # (the scaling of F2 for a zero row)
        return np.float32(0.0), np.float32(0.0)
    d = np.float32(QK_SQRT128 * m)
    return np.float32(np.float32(448.0) / d), np.float32(d / np.float32(448.0))


def quantize_qk(x, w) -> np.ndarray:
    """e4m3 codes of x (q or k rows after RMSNorm with weight w and RoPE):
    e4m3(fp32(x * inv))."""
    inv, _ = qk_code_scale(w)
    return e4m3_encode((np.asarray(x, np.float64) * np.float64(inv)).astype(np.float32))


def dequantize_qk(codes, w) -> np.ndarray:
    _, s = qk_code_scale(w)
    return e4m3_decode(codes) * np.float64(s)


def qkv_qknorm_mrope_e4m3(xq, xs, Wq, Ws, qn_w, kn_w, pos, n_heads, head_dim=128, split=(32, 48, 48)):
    """QKV from e4m3 operands, then the bf16 path's per-head Q/K RMSNorm and
    3-D RoPE on the fp32 accumulator."""
    return O.qkv_qknorm_mrope(dequantize_rows(xq, xs), dequantize_rows(Wq, Ws), qn_w, kn_w, pos, n_heads,
                              head_dim, split)


def gated_residual_e4m3(x, oq, os_, Wq, Ws, mod, ranges, rows=None):
    """x + gate_msa[m] * (o Wo^T) with e4m3 o and Wo."""
    return np.asarray(x, np.float64) + O.gate_rows(mod, ranges, O.MSA, rows) * gemm_e4m3(oq, os_, Wq, Ws)


def swiglu_hidden_e4m3(xq, xs, Wguq, Wgus) -> np.ndarray:
    """SiLU(gate) * up from the e4m3 gate/up GEMM (Wgu = [gate; up]), float64."""
    F = Wguq.shape[0] // 2
    gu = gemm_e4m3(xq, xs, Wguq, Wgus)
    return O.silu(gu[:, :F]) * gu[:, F:]


def ffn_down_e4m3(x, hq, hs, Wdq, Wds, mod, ranges, rows=None):
    """x + gate_mlp[m] * (h Wd^T) with e4m3 h and Wd."""
    return np.asarray(x, np.float64) + O.gate_rows(mod, ranges, O.MLP, rows) * gemm_e4m3(hq, hs, Wdq, Wds)


def block_forward_e4m3(x, mod, ranges, pos, Wqkv_q, Wqkv_s, qn_w, kn_w, Wo_q, Wo_s, Wgu_q, Wgu_s, Wd_q, Wd_s,
                       n_heads, head_dim=128, split=(32, 48, 48), return_parts=False, qk_e4m3=False):
    """The block with its four GEMMs in e4m3.  Quantisation points: the two
    modulated LayerNorm outputs (from their fp32 values), the attention
    output and the SwiGLU hidden state (from the bf16 tensors the path
    stores), and with qk_e4m3 q and k (static scales, from their fp32
    values).  Attention itself stays in the bf16 path's form."""
    x = np.asarray(x, np.float64)
    xm1 = O.adaln_modulate(x, mod, ranges, O.MSA)
    xq1, xs1 = quantize_rows(xm1)
    q, k, v = qkv_qknorm_mrope_e4m3(xq1, xs1, Wqkv_q, Wqkv_s, qn_w, kn_w, pos, n_heads, head_dim, split)
    if qk_e4m3:
        q = dequantize_qk(quantize_qk(q, qn_w), qn_w)
        k = dequantize_qk(quantize_qk(k, kn_w), kn_w)
    o = O.attention(q, k, v)
    oq, os_ = quantize_rows(O.round_to_bf16(o))
    x1 = gated_residual_e4m3(x, oq, os_, Wo_q, Wo_s, mod, ranges)
    xm2 = O.adaln_modulate(x1, mod, ranges, O.MLP)
    xq2, xs2 = quantize_rows(xm2)
    h = swiglu_hidden_e4m3(xq2, xs2, Wgu_q, Wgu_s)
    hq, hs = quantize_rows(O.round_to_bf16(h))
    x2 = ffn_down_e4m3(x1, hq, hs, Wd_q, Wd_s, mod, ranges)
    if return_parts:
        return x2, {"xm1": xm1, "o": o, "x1": x1, "xm2": xm2, "h": h}
    return x2
