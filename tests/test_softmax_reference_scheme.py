"""The attention kernel's online-softmax algorithm, modelled in float64 on
the CPU, equals the exact softmax-weighted sum (to 1e-12) on score patterns
that exercise every branch.  The algorithm, per query row over key tiles of
128 keys in two halves of 64:

  * the reference m is the first key tile's row max (log2 units);
  * each half's p = 2^(s - m) is accepted while its sum stays <= 2^16;
  * otherwise m moves to max(m, the half's own max), the running sum l and
    the accumulator o (which hold every earlier half, including the tile's
    first half when the second one moves m) are rescaled by 2^(m_old - m_new),
    and the half is redone;
  * o / l at the end.

This pins the scheme itself (no GPU): a dropped rescale, a rescale of the
wrong partial sums or a reference taken from the wrong half fails here."""
import numpy as np
import pytest

LIMIT = 2.0 ** 16


def kernel_scheme(s_log2, v, tile=128):
    """s_log2 [n_keys] scores already in log2 units, v [n_keys, d]."""
    n = len(s_log2)
    m = s_log2[:tile].max()
    l = 0.0
    o = np.zeros(v.shape[1])
    moves = 0
    for t0 in range(0, n, tile):
        hsum = [0.0, 0.0]
        hacc = [np.zeros(v.shape[1]), np.zeros(v.shape[1])]
        for hf in range(2):
            lo, hi = t0 + 64 * hf, min(t0 + 64 * hf + 64, n)
            if lo >= hi:
                continue
            p = np.exp2(s_log2[lo:hi] - m)
            if t0 > 0 and not (p.sum() <= LIMIT):
                m_new = max(m, s_log2[lo:hi].max())
                a = np.exp2(m - m_new)
                m = m_new
                moves += 1
                l *= a
                o *= a
                if hf == 1:          # the first half was taken against the old reference
                    hsum[0] *= a
                    hacc[0] *= a
                p = np.exp2(s_log2[lo:hi] - m)
            hsum[hf] = p.sum()
            hacc[hf] = p @ v[lo:hi]
        l += hsum[0] + hsum[1]
        o += hacc[0] + hacc[1]
    return o / l, moves


def exact(s_log2, v):
    p = np.exp2(s_log2 - s_log2.max())
    return (p / p.sum()) @ v


@pytest.mark.parametrize("kind", ["normal", "ramp", "spike_first_half", "spike_second_half", "descending",
                                  "huge_late", "partial_tail"])
def test_scheme_equals_exact_softmax(kind):
    rng = np.random.default_rng({"normal": 1, "ramp": 2, "spike_first_half": 3, "spike_second_half": 4,
                                 "descending": 5, "huge_late": 6, "partial_tail": 7}[kind])
    n = 1000 if kind != "partial_tail" else 3 * 128 + 5
    s = rng.standard_normal(n) * 2.0
    if kind == "ramp":
        s += np.linspace(0, 60, n)            # the reference moves many times
    elif kind == "spike_first_half":
        s[3 * 128 + 10] += 90.0               # moves it in a first half
    elif kind == "spike_second_half":
        s[3 * 128 + 100] += 90.0              # moves it in a second half (first half already taken)
    elif kind == "descending":
        s += np.linspace(60, 0, n)            # the first tile holds the max: never moves
    elif kind == "huge_late":
        s[-3] += 500.0                        # would overflow fp32 against the old reference
    elif kind == "partial_tail":
        s[-2] += 40.0                         # the move happens in the partial last tile
    v = rng.standard_normal((n, 16))
    got, moves = kernel_scheme(s, v)
    np.testing.assert_allclose(got, exact(s, v), rtol=1e-12, atol=1e-12)
    if kind in ("ramp", "spike_first_half", "spike_second_half", "huge_late", "partial_tail"):
        assert moves > 0
    if kind in ("normal", "descending"):
        assert moves == 0
