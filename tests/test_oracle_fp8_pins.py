"""Pins of the FP8 (e4m3) oracle against the OCP OFP8 definition, a brute-force
search, torch's float8_e4m3fn conversion and closed forms (CPU only)."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle_fp8 as F


def test_value_table_closed_form():
    t = F.e4m3_table()
    # OFP8 e4m3: bias 7, largest finite 1.75 * 2^8, smallest normal 2^-6,
    # smallest subnormal 2^-9, S.1111.111 is NaN, no infinities
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9
    assert t[0x38] == 1.0 and t[0x40] == 2.0 and t[0x3C] == 1.5
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and np.signbit(t[0x80])
    assert np.isinf(t).sum() == 0
    assert np.isfinite(t).sum() == 254
    pos = t[:127]
    assert np.all(np.diff(pos) > 0)
    # spacing: 2^-9 below 2^-6 (subnormals and the first binade), then doubling per binade
    assert np.allclose(np.diff(pos[:16]), 2.0 ** -9)
    for e in range(1, 15):
        binade = pos[8 * e: 8 * e + 8]
        assert np.allclose(np.diff(binade), 2.0 ** (e - 7) / 8)
    for c in range(128):  # the sign bit only negates
        assert (np.isnan(t[c]) and np.isnan(t[c + 128])) or t[c + 128] == -t[c]


def _brute_force_encode(x):
    """Nearest finite e4m3 value by exhaustive search; ties to the even code;
    saturation to +-448; the sign bit of x kept."""
    t = F.e4m3_table()
    out = []
    for v in np.asarray(x, np.float64).ravel():
        a = min(abs(v), 448.0)
        best, best_d = None, None
        for c in range(127):
            d = abs(t[c] - a)
            if best is None or d < best_d or (d == best_d and c % 2 == 0 and best % 2 == 1):
                best, best_d = c, d
        if np.signbit(v):
            best |= 0x80
        out.append(best)
    return np.array(out, dtype=np.uint8).reshape(np.shape(x))


def test_encode_matches_brute_force():
    rng = np.random.default_rng(7)
    t = F.e4m3_table()
    pos = t[:127]
    mids = (pos[:-1] + pos[1:]) / 2  # every tie
    x = np.concatenate([
        rng.standard_normal(2000) * 30, rng.standard_normal(500) * 0.01, mids, -mids, pos, -pos,
        np.array([0.0, -0.0, 448.0, 449.0, 464.0, 500.0, 1e30, -1e30, 2.0 ** -12]),
    ])
    assert np.array_equal(F.e4m3_encode(x), _brute_force_encode(x))


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    pos = F.e4m3_table()[:127]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    x = np.concatenate([rng.uniform(-448, 448, 20000).astype(np.float32),
                        (rng.standard_normal(20000) * 0.05).astype(np.float32), mids, -mids,
                        np.array([-0.0, 0.0, -1e-9, 2.0 ** -10], np.float32)])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(x), ref)


def test_saturation():
    assert list(F.e4m3_encode([448.0, 1e4, -1e4, 464.0, 479.0])) == [0x7E, 0x7E, 0xFE, 0x7E, 0x7E]


def test_quantize_rows_invariants():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((16, 300)) * rng.uniform(1e-3, 1e3, (16, 1))).astype(np.float32)
    x[5] = 0.0
    codes, scale = F.quantize_rows(x)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32
    assert scale[5] == 0 and not codes[5].any()
    dec = F.dequantize_rows(codes, scale)
    for r in range(16):
        if r == 5:
            continue
        amax = np.max(np.abs(x[r]))
        # the row's largest magnitude lands on the largest code
        assert (codes[r] & 0x7F).max() == 0x7E
        assert scale[r] == np.float32(amax) / np.float32(448.0)
        # within half a step: 2^-4 relative in the normal range, 2^-10 code
        # units below it, plus the fp32 rounding of the two scale factors
        err = np.abs(dec[r] - x[r].astype(np.float64))
        bound = np.maximum(np.abs(x[r]) * 2.0 ** -4, 2.0 ** -10 * scale[r]) * (1 + 1e-6) + 1e-6 * np.abs(x[r])
        assert np.all(err <= bound)


def test_gemm_triple_loop():
    rng = np.random.default_rng(5)
    qa = rng.integers(0, 256, (3, 7)).astype(np.uint8)
    qb = rng.integers(0, 256, (4, 7)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x10  # no NaN codes
    qb[(qb & 0x7F) == 0x7F] = 0x22
    sa = np.array([0.5, 2.0, 0.125], np.float32)
    sb = np.array([1.0, 0.25, 4.0, 3.0], np.float32)
    out = F.gemm_e4m3(qa, sa, qb, sb)
    for m in range(3):
        for n in range(4):
            acc = 0.0
            for k in range(7):
                acc += F.e4m3_value(int(qa[m, k])) * F.e4m3_value(int(qb[n, k]))
            assert out[m, n] == pytest.approx(float(sa[m]) * float(sb[n]) * acc, rel=1e-12, abs=1e-300)


def test_qk_codes_static_scale():
    """q / k codes with the static scale from the norm weight: the scale is
    fp32(sqrt(128) max|w|) / 448; the bound that RMSNorm then RoPE give a head
    row (every element at most sqrt(128) max|w|) lands on the largest code
    without passing it; every finite code of the scale's grid round-trips;
    and dequantised values are within half a step of a 3-bit mantissa."""
    rng = np.random.default_rng(11)
    w = (1 + 0.1 * rng.standard_normal(128)).astype(np.float32)
    w[17] = -1.6  # the bound uses |w|
    inv, s = F.qk_code_scale(w)
    assert s == np.float32(np.float32(np.float32(11.3137085) * np.float32(1.6)) / np.float32(448.0))
    assert abs(float(inv) * float(s) - 1.0) < 1e-6
    # extreme row: all of the row's energy in one element, |x| = sqrt(128) max|w|
    x = np.zeros((1, 128))
    x[0, 5] = -np.sqrt(128.0) * 1.6
    c = F.quantize_qk(x, w)
    assert c[0, 5] == 0xFE                       # -448
    # rows that RMSNorm (weight w) and a rotation of pairs produce stay within the bound
    r = rng.standard_normal((256, 128))
    r = r / np.sqrt((r ** 2).mean(1, keepdims=True)) * w.astype(np.float64)
    ang = rng.uniform(-np.pi, np.pi, (256, 64))
    a, b = r[:, 0::2], r[:, 1::2]
    rot = np.empty_like(r)
    rot[:, 0::2], rot[:, 1::2] = a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)
    assert np.all(np.abs(rot) <= np.sqrt(128.0) * 1.6 + 1e-12)
    dec = F.dequantize_qk(F.quantize_qk(rot, w), w)
    assert np.all(np.abs(F.e4m3_decode(F.quantize_qk(rot, w))) <= 448.0)
    err = np.abs(dec - rot)
    assert np.all(err <= np.maximum(np.abs(rot) * 2.0 ** -4, 2.0 ** -10 * float(s)) * (1 + 1e-6) + 1e-7)
    # every finite code of the grid round-trips exactly
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = F.e4m3_decode(codes) * np.float64(s)
    assert np.array_equal(F.quantize_qk(vals, w) & 0x7F, codes & 0x7F)


def test_qk_codes_zero_norm_weight():
    """An all-zero norm weight (every q or k element 0) takes the zero-row
    rule of the row scaling: inverse scale 0 and scale 0, so its codes are 0
    and dequantise to 0, with no 0 * inf anywhere."""
    inv, s = F.qk_code_scale(np.zeros(128, np.float32))
    assert inv == 0.0 and s == 0.0
    x = np.zeros((3, 128))
    x[1, 7] = -0.0
    c = F.quantize_qk(x, np.zeros(128, np.float32))
    assert np.all((c & 0x7F) == 0)
    assert np.all(F.dequantize_qk(c, np.zeros(128, np.float32)) == 0)
