"""Loops-only twin of the oracle's block arithmetic.  TEST INFRASTRUCTURE ONLY.

Plain Python loops over scalars (no matmul operator, no einsum, no NumPy
reductions) so that an axis, transpose or broadcasting slip in the vectorised
oracle shows up as a mismatch.  Meant for micro sizes (tens of tokens).  It
restates the same readings as h3_oracle (see its header) and cites the same
passages: "MiniMax-H3: native joint audio-video generation" (note.shouss.top)
§3, §3.1, §3.2 for the block, "MiniMax-H3 paper reading" (gojay.top) §7.4
for the 3-D RoPE.
"""
from __future__ import annotations

import math


def _mat(x):
    return [[float(v) for v in row] for row in x]


def _linear(x, W):
    out = []
    for row in x:
        o = []
        for wrow in W:
            acc = 0.0
            for a, b in zip(row, wrow):
                acc += a * b
            o.append(acc)
        out.append(o)
    return out


def _modality(r, ranges):
    for m in range(3):
        s, c = ranges["start"][m], ranges["count"][m]
        if s <= r < s + c:
            return m
    raise ValueError(r)


def _ln_mod(x, mod, ranges, branch, eps=1e-6):
    out = []
    for r, row in enumerate(x):
        n = len(row)
        mu = 0.0
        for v in row:
            mu += v
        mu /= n
        var = 0.0
        for v in row:
            var += (v - mu) * (v - mu)
        var /= n
        inv = 1.0 / math.sqrt(var + eps)
        m = _modality(r, ranges)
        shift, scale = mod[m][3 * branch], mod[m][3 * branch + 1]
        out.append([(v - mu) * inv * (1.0 + scale[d]) + shift[d] for d, v in enumerate(row)])
    return out


def _rms(vec, w, eps=1e-6):
    ss = 0.0
    for v in vec:
        ss += v * v
    inv = 1.0 / math.sqrt(ss / len(vec) + eps)
    return [v * inv * w[d] for d, v in enumerate(vec)]


def _rope(vec, p, split, theta=10000.0):
    out = list(vec)
    base = 0
    for axis, d in enumerate(split):
        for i in range(d // 2):
            ang = p[axis] * theta ** (-2.0 * i / d)
            c, s = math.cos(ang), math.sin(ang)
            a, b = vec[base + 2 * i], vec[base + 2 * i + 1]
            out[base + 2 * i] = a * c - b * s
            out[base + 2 * i + 1] = a * s + b * c
        base += d
    return out


def block_forward_loops(x, mod, ranges, pos, Wqkv, qn_w, kn_w, Wo, Wgu, Wd, n_heads,
                        head_dim=128, split=(32, 48, 48)):
    """Same block as h3_oracle.block_forward, scalar loops only."""
    x = _mat(x)
    mod = [[[float(v) for v in vec] for vec in m] for m in mod]
    pos = _mat(pos)
    L, D = len(x), len(x[0])
    I = n_heads * head_dim
    xm = _ln_mod(x, mod, ranges, 0)
    qkv = _linear(xm, _mat(Wqkv))
    qn_w = [float(v) for v in qn_w]
    kn_w = [float(v) for v in kn_w]
    q = [[None] * n_heads for _ in range(L)]
    k = [[None] * n_heads for _ in range(L)]
    v = [[None] * n_heads for _ in range(L)]
    for r in range(L):
        for h in range(n_heads):
            lo = h * head_dim
            q[r][h] = _rope(_rms(qkv[r][lo:lo + head_dim], qn_w), pos[r], split)
            k[r][h] = _rope(_rms(qkv[r][I + lo:I + lo + head_dim], kn_w), pos[r], split)
            v[r][h] = qkv[r][2 * I + lo:2 * I + lo + head_dim]
    scale = 1.0 / math.sqrt(head_dim)
    o = [[0.0] * I for _ in range(L)]
    for h in range(n_heads):
        for r in range(L):
            s = []
            for c in range(L):
                acc = 0.0
                for d in range(head_dim):
                    acc += q[r][h][d] * k[c][h][d]
                s.append(acc * scale)
            mx = max(s)
            e = [math.exp(t - mx) for t in s]
            tot = 0.0
            for t in e:
                tot += t
            for d in range(head_dim):
                acc = 0.0
                for c in range(L):
                    acc += e[c] * v[c][h][d]
                o[r][h * head_dim + d] = acc / tot
    attn = _linear(o, _mat(Wo))
    x1 = []
    for r in range(L):
        g = mod[_modality(r, ranges)][2]
        x1.append([x[r][d] + g[d] * attn[r][d] for d in range(D)])
    xm2 = _ln_mod(x1, mod, ranges, 1)
    Wgu = _mat(Wgu)
    F = len(Wgu) // 2
    gate = _linear(xm2, Wgu[:F])
    up = _linear(xm2, Wgu[F:])
    hmid = [[(a / (1.0 + math.exp(-a))) * b for a, b in zip(gr, ur)] for gr, ur in zip(gate, up)]
    f = _linear(hmid, _mat(Wd))
    x2 = []
    for r in range(L):
        g = mod[_modality(r, ranges)][5]
        x2.append([x1[r][d] + g[d] * f[r][d] for d in range(D)])
    return x2
