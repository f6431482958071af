"""Pins of the float64 oracle to facts fixed outside the oracle itself.

Each test ties one oracle function to a value the pages print (golden file),
a closed form, an invariant, or an independent library routine, so that a
dropped term, a wrong sign or index, or a transposed operand fails here.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

from oracle import h3_oracle as O
from oracle import h3_loops
from omni_modal_diffusion_b200 import synthetic as S


def _pin_close(a, b, tol):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if b.ndim == 0:
        b = np.full_like(a, b)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, err


# ---------------------------------------------------------------- A1 shapes

def test_config_widths_from_pages(golden):
    D = int(golden["hidden"])
    assert int(golden["heads"]) * int(golden["head_dim"]) == int(golden["attention_inner"])
    assert int(golden["attention_inner"]) != D
    # modulation consumed as [3 modalities][6][D]: 18 D features (96768 at D=5376)
    per_mod = int(golden["adaln_out_features_per_modality"])
    assert int(golden["modalities"]) * per_mod * D == 96768
    w = S.WORKLOADS["768sq_2s"]
    assert (w.D, w.H, w.head_dim, w.I, w.F, w.D_text) == (
        D, int(golden["heads"]), int(golden["head_dim"]), int(golden["attention_inner"]),
        int(golden["ffn_inner"]), int(golden["text_input_dim"]))


def test_adaln_producer_width_matches_page_parameter_counts(golden):
    """Reading G22: each block's AdaLN producer is one linear from a D/2-wide
    conditioning vector to the 18 D modulation features.  That width is the
    one that reproduces the pages' counts: 50 blocks x 18 D x D/2 = 13.0 B
    parameters in the AdaLN branch, and with the blocks' attention and FFN
    weights (19.3 B) the 33 B total and the ~20 B deployed without it."""
    D, blocks = int(golden["hidden"]), int(golden["blocks"])
    I, F = int(golden["attention_inner"]), int(golden["ffn_inner"])
    adaln = blocks * 18 * D * (D // 2)
    trunk = blocks * (D * 3 * I + I * D + 2 * D * F + F * D)
    assert abs(adaln / 1e9 - float(golden["adaln_params_billion"])) < 0.01 * 13
    assert abs(trunk / 1e9 - float(golden["deploy_params_billion"])) < 0.05 * 20
    assert abs((adaln + trunk) / 1e9 - float(golden["transformer_params_billion"])) < 0.05 * 33


def test_adaln_producer_matches_library_composition():
    """SiLU then linear, read as [n][3][6][D], against torch's silu and
    linear; and each (modality, slot) block of W's rows drives exactly that
    slice of the modulation."""
    rng = np.random.default_rng(23)
    D, C, n = 8, 5, 3
    c = rng.standard_normal((n, C)) * 2
    W = rng.standard_normal((18 * D, C))
    got = O.adaln_modulation(c, W, D)
    ref = TF.linear(TF.silu(torch.from_numpy(c)), torch.from_numpy(W)).reshape(n, 3, 6, D)
    _pin_close(got, ref.numpy(), 1e-12)
    for m in range(3):
        for j in range(6):
            W1 = np.zeros_like(W)
            W1[(m * 6 + j) * D:(m * 6 + j + 1) * D] = W[(m * 6 + j) * D:(m * 6 + j + 1) * D]
            g1 = O.adaln_modulation(c, W1, D)
            mask = np.zeros((3, 6), bool)
            mask[m, j] = True
            assert np.all(g1[:, ~mask] == 0) and np.all(g1[:, mask] != 0)


def test_modulation_uses_each_of_18D_slices_once():
    """Perturbing any one of the 3x6 slices of mod changes exactly the output
    that slice should drive, and only for that modality's rows."""
    rng = np.random.default_rng(0)
    D = 8
    ranges = O.pack_ranges(3, 4, 5)
    x = rng.standard_normal((ranges["L"], D))
    mod = rng.standard_normal((3, 6, D)) * 0.1
    o = rng.standard_normal((ranges["L"], D))
    Wo = np.eye(D)
    base_msa = O.adaln_modulate(x, mod, ranges, O.MSA)
    base_mlp = O.adaln_modulate(x, mod, ranges, O.MLP)
    base_res = O.gated_residual(x, o, Wo, mod, ranges)
    mids = O.modality_of_rows(ranges)
    for m in range(3):
        for j in range(6):
            mod2 = mod.copy()
            mod2[m, j] += 1.0
            d_msa = np.abs(O.adaln_modulate(x, mod2, ranges, O.MSA) - base_msa).max(axis=1)
            d_mlp = np.abs(O.adaln_modulate(x, mod2, ranges, O.MLP) - base_mlp).max(axis=1)
            d_res = np.abs(O.gated_residual(x, o, Wo, mod2, ranges) - base_res).max(axis=1)
            touched = {0: d_msa, 1: d_msa, 2: d_res, 3: d_mlp, 4: d_mlp, 5: None}[j]
            for arr in (d_msa, d_mlp, d_res):
                if arr is touched:
                    assert np.all(arr[mids == m] > 0) and np.all(arr[mids != m] == 0)
                else:
                    assert np.all(arr == 0)


def test_token_grid_counts_and_worked_examples(golden):
    # causal VAE: 49, 121, 361 frames -> 13, 31, 91 latent frames
    assert [O.latent_frames(n) for n in (49, 121, 361)] == [13, 31, 91]
    assert O.latent_hw(768, 768) == (48, 48)
    assert O.latent_hw(768, 1344) == (48, 84)
    assert O.latent_hw(768, 1792) == (48, 112)
    counts = []
    for n, hgt, wid in ((49, 768, 768), (121, 768, 1344), (361, 768, 1792)):
        t, i, j = O.token_grid(O.latent_frames(n), *O.latent_hw(hgt, wid))
        counts.append(t * i * j)
    assert counts == [7488, 31248, 122304]
    # effective spatial stride 32 = VAE 16 x patch 2
    assert int(golden["vae_spatial"]) * 2 == int(golden["effective_spatial_stride"])
    assert 768 // int(golden["effective_spatial_stride"]) == O.token_grid(1, *O.latent_hw(768, 768))[1]
    # oceanz worked example: 100 x 1088 x 1920 -> 25 x 68 x 120 x 24
    lhs, rhs = golden["example_oceanz"].split("->")
    f, hh, ww = map(int, lhs.split())
    assert (O.latent_frames(f), *O.latent_hw(hh, ww), O.patch_width() // 4) == tuple(map(int, rhs.split()))
    # gojay §7.3: 240 x 768 x 1360 -> 60 x 48 x 85 -> tokens 60 x 24 x 42
    parts = golden["example_gojay"].split("->")
    f, hh, ww = map(int, parts[0].split())
    lat = tuple(map(int, parts[1].split()))
    tok = tuple(map(int, parts[2].split()))
    assert (O.latent_frames(f), *O.latent_hw(hh, ww), 24) == lat
    assert O.token_grid(*lat[:3]) == tok


def test_patch_width_and_patchify_matches_library_rearrange(golden):
    assert O.patch_width(int(golden["vae_channels"])) == 96
    rng = np.random.default_rng(1)
    lat = rng.standard_normal((3, 6, 10, 24))
    p = O.patchify(lat)
    assert p.shape == (3 * 3 * 5, 96)
    import einops
    ref = einops.rearrange(lat, "t (i ph) (j pw) c -> (t i j) (ph pw c)", ph=2, pw=2)
    assert np.array_equal(p, ref)
    assert np.array_equal(O.unpatchify(p, 3, 6, 10), lat)


def test_audio_token_counts(golden):
    hz = int(golden["audio_latent_hz"])
    assert 5 * hz == int(golden["audio_5s_tokens_per_channel"])
    assert 2 * 5 * hz == int(golden["audio_5s_tokens_stereo"])
    w = S.WORKLOADS["768x1344_5s"]
    assert w.audio_channels * w.n_audio == int(golden["audio_5s_tokens_stereo"])


def test_pack_ranges_tile_the_sequence():
    r = O.pack_ranges(512, 400, 31248)
    assert r["L"] == 32160 and r["L_pad"] == 32256
    assert r["start"] == [0, 512, 912]
    m = O.modality_of_rows(r)
    assert (m == O.TEXT).sum() == 512 and (m == O.AUDIO).sum() == 400 and (m == O.VIDEO).sum() == 31248
    assert list(m[:1]) == [0] and m[511] == 0 and m[512] == 1 and m[911] == 1 and m[912] == 2
    assert O.pack_ranges(1, 0, 0)["L_pad"] == 128 and O.pack_ranges(64, 64, 0)["L_pad"] == 128
    assert O.pack_ranges(64, 64, 1)["L_pad"] == 256


def test_positions_share_time_axis(golden):
    # audio latent k at k/40 s and video latent frame t at t/(24/4) s share one axis
    r = O.pack_ranges(2, 2 * 40, 2 * 2 * 2)
    pos = O.positions(r, 2, 2, 2, 2, 40)
    fps, hz = int(golden["fps"]), int(golden["audio_latent_hz"])
    vlat_hz = fps / int(golden["vae_temporal"])
    for ch in range(2):
        for k in range(40):
            p = pos[r["start"][O.AUDIO] + ch * 40 + k]
            assert p[1] == 0 and p[2] == 0
            assert math.isclose(p[0], (k / hz) * vlat_hz, rel_tol=1e-15, abs_tol=1e-15)
    # audio latent 6 (0.15 s) ... latent 20 sits exactly at video latent frame 3 (0.5 s)
    assert pos[r["start"][O.AUDIO] + 20][0] == 3.0
    v0 = r["start"][O.VIDEO]
    assert [tuple(pos[v0 + n]) for n in range(8)] == [
        (0, 0, 0), (0, 0, 1), (0, 1, 0), (0, 1, 1), (1, 0, 0), (1, 0, 1), (1, 1, 0), (1, 1, 1)]
    assert np.all(pos[:2] == 0)


# ---------------------------------------------------------------- A3 LN-modulate

def test_layernorm_matches_library():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 33)) * 3 + 1.5
    ref = TF.layer_norm(torch.from_numpy(x), (33,), eps=1e-6).numpy()
    _pin_close(O.layernorm(x), ref, 1e-12)
    # a constant row normalises to exactly 0
    assert np.all(O.layernorm(np.full((2, 9), 4.25)) == 0)
    # mean 0, variance 1/(1 + eps/var) with scale = shift = 0
    h = O.layernorm(x)
    var = x.var(axis=1)
    _pin_close(h.mean(axis=1), 0, 1e-13)
    _pin_close(h.var(axis=1), 1 / (1 + 1e-6 / var), 1e-12)


def test_modulate_scale_shift_forms():
    rng = np.random.default_rng(3)
    D = 16
    r = O.pack_ranges(2, 3, 4)
    x = rng.standard_normal((r["L"], D))
    mod = np.zeros((3, 6, D))
    ref = TF.layer_norm(torch.from_numpy(x), (D,), eps=1e-6).numpy()
    _pin_close(O.adaln_modulate(x, mod, r, O.MSA), ref, 1e-12)       # scale 0 -> plain LN
    mod[:, 1] = 0.5                                                  # scale_msa = 0.5 -> 1.5 LN
    mod[:, 0] = -2.0                                                 # shift_msa = -2
    _pin_close(O.adaln_modulate(x, mod, r, O.MSA), 1.5 * ref - 2.0, 1e-12)
    _pin_close(O.adaln_modulate(x, mod, r, O.MLP), ref, 1e-12)       # MLP slots untouched
    # sentinel on one modality: only that range changes
    for m in range(3):
        mod2 = np.zeros((3, 6, D))
        mod2[m, 3] = 7.0
        out = O.adaln_modulate(x, mod2, r, O.MLP)
        rows = O.modality_of_rows(r) == m
        _pin_close(out[rows], ref[rows] + 7.0, 1e-12)
        _pin_close(out[~rows], ref[~rows], 1e-12)


# ---------------------------------------------------------------- A4/A5

def test_linear_convention_matches_library():
    rng = np.random.default_rng(4)
    x, W = rng.standard_normal((5, 7)), rng.standard_normal((3, 7))
    _pin_close(O.linear(x, W), TF.linear(torch.from_numpy(x), torch.from_numpy(W)).numpy(), 1e-12)


def test_rmsnorm_matches_library():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 3, 128))
    w = 1 + 0.1 * rng.standard_normal(128)
    ref = TF.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(w), eps=1e-6).numpy()
    _pin_close(O.rmsnorm(x, w), ref, 1e-12)
    y = O.rmsnorm(x, np.ones(128))
    _pin_close(np.sqrt((y * y).mean(axis=-1)), 1 / np.sqrt(1 + 1e-6 / (x * x).mean(axis=-1)), 1e-12)


def test_rope_sections_match_library_rope():
    """Each t/h/w section equals a standard 1-D RoPE of that width (library
    implementation with half-split pairing, mapped to interleaved pairs)."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    rng = np.random.default_rng(6)
    L = 9
    x = rng.standard_normal((L, 2, 128))
    pos = np.stack([rng.integers(0, 40, L), rng.integers(0, 24, L), rng.integers(0, 56, L)], 1).astype(np.float64)
    pos[0] = (0, 0, 0)
    pos[1] = (4.35, 0, 0)                      # a fractional audio-style time
    out = O.rope(x, pos, (32, 48, 48))
    base = 0
    for axis, d in enumerate((32, 48, 48)):
        cfg = LlamaConfig(hidden_size=d * 2, num_attention_heads=2, head_dim=d, rope_theta=10000.0)
        emb = LlamaRotaryEmbedding(cfg)
        seg = torch.from_numpy(x[:, :, base:base + d])
        half = torch.cat([seg[..., 0::2], seg[..., 1::2]], dim=-1).transpose(0, 1)[None]  # [1,h,L,d]
        cos, sin = emb(half, torch.from_numpy(pos[:, axis])[None])
        rot, _ = apply_rotary_pos_emb(half, half, cos, sin)
        rot = rot[0].transpose(0, 1).numpy()
        ref = np.empty_like(rot)
        ref[..., 0::2], ref[..., 1::2] = rot[..., :d // 2], rot[..., d // 2:]
        _pin_close(out[:, :, base:base + d], ref, 2e-5)      # library angles are float32
        base += d


def test_rope_invariants():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((6, 3, 128))
    k = rng.standard_normal((6, 3, 128))
    p = rng.uniform(0, 50, (6, 3))
    rq = O.rope(q, p)
    _pin_close(np.linalg.norm(rq, axis=-1), np.linalg.norm(q, axis=-1), 1e-12)     # norm preserved
    _pin_close(O.rope(q, np.zeros((6, 3))), q, 0)                                  # p = 0 -> identity
    # complex-rotation form: pair (2i, 2i+1) as one complex number
    z = q[..., 0::2] + 1j * q[..., 1::2]
    ang = O.rope_angles(p)[:, None, :]
    zr = z * np.exp(1j * ang)
    _pin_close(rq[..., 0::2], zr.real, 1e-12)
    _pin_close(rq[..., 1::2], zr.imag, 1e-12)
    # <R(p) q, R(p') k> depends only on p - p'
    shift = np.array([3.0, -2.0, 5.5])
    d1 = (O.rope(q, p) * O.rope(k, p[::-1])).sum(-1)
    d2 = (O.rope(q, p + shift) * O.rope(k, p[::-1] + shift)).sum(-1)
    _pin_close(d1, d2, 1e-10)


# ---------------------------------------------------------------- A6

def test_attention_matches_library_sdpa():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((37, 3, 128)) for _ in range(3))
    ref = TF.scaled_dot_product_attention(
        *(torch.from_numpy(a).transpose(0, 1) for a in (q, k, v)), is_causal=False)
    _pin_close(O.attention(q, k, v), ref.transpose(0, 1).reshape(37, 3 * 128).numpy(), 1e-12)
    rows = np.array([0, 5, 36])
    _pin_close(O.attention_rows(q[rows], k, v), O.attention(q, k, v)[rows], 1e-13)


def test_attention_special_cases():
    rng = np.random.default_rng(9)
    q, k = rng.standard_normal((11, 2, 128)), rng.standard_normal((11, 2, 128))
    _pin_close(O.attention(q, k, np.ones((11, 2, 128))), 1.0, 1e-13)           # v = 1 -> 1
    v1 = rng.standard_normal((1, 2, 128))
    _pin_close(O.attention(q[:1], k[:1], v1), v1.reshape(1, 256), 1e-15)        # one key -> v
    v = rng.standard_normal((11, 2, 128))
    _pin_close(O.attention(np.zeros_like(q), k, v), np.tile(v.mean(0).reshape(1, 256), (11, 1)), 1e-13)


# ---------------------------------------------------------------- A9

def test_silu_and_ffn_match_library():
    rng = np.random.default_rng(10)
    a = rng.standard_normal(50) * 4
    _pin_close(O.silu(a), TF.silu(torch.from_numpy(a)).numpy(), 1e-14)
    D, Fh = 12, 20
    r = O.pack_ranges(2, 2, 3)
    x = rng.standard_normal((r["L"], D))
    xm = rng.standard_normal((r["L"], D))
    Wgu = rng.standard_normal((2 * Fh, D))
    Wd = rng.standard_normal((D, Fh))
    mod = rng.standard_normal((3, 6, D))
    t = torch.from_numpy
    h = TF.silu(TF.linear(t(xm), t(Wgu[:Fh]))) * TF.linear(t(xm), t(Wgu[Fh:]))
    gate = t(mod[O.modality_of_rows(r), 5])
    ref = t(x) + gate * TF.linear(h, t(Wd))
    _pin_close(O.ffn_swiglu(x, xm, Wgu, Wd, mod, r), ref.numpy(), 1e-12)


# ---------------------------------------------------------------- block

def _tiny_block_inputs(seed=11, D=64, H=2, Fh=96, counts=(5, 6, 8)):
    rng = np.random.default_rng(seed)
    r = O.pack_ranges(*counts)
    L = r["L"]
    x = rng.standard_normal((L, D))
    mod = rng.standard_normal((3, 6, D)) * 0.1
    pos = rng.uniform(0, 10, (L, 3))
    I = H * 128
    W = dict(Wqkv=rng.standard_normal((3 * I, D)) * 0.05, qn_w=1 + 0.1 * rng.standard_normal(128),
             kn_w=1 + 0.1 * rng.standard_normal(128), Wo=rng.standard_normal((D, I)) * 0.05,
             Wgu=rng.standard_normal((2 * Fh, D)) * 0.05, Wd=rng.standard_normal((D, Fh)) * 0.05)
    return r, x, mod, pos, W, H


def test_block_matches_loops_twin():
    r, x, mod, pos, W, H = _tiny_block_inputs(D=24, Fh=40, counts=(3, 4, 6))
    a = O.block_forward(x, mod, r, pos, n_heads=H, **W)
    b = np.array(h3_loops.block_forward_loops(x, mod, r, pos, n_heads=H, **W))
    _pin_close(a, b, 1e-12)


def test_block_matches_library_composition():
    """The block composed from library routines (layer_norm, linear, rms_norm,
    SDPA, silu) with the complex-number RoPE."""
    r, x, mod, pos, W, H = _tiny_block_inputs()
    t = torch.from_numpy
    L, D = x.shape
    m = O.modality_of_rows(r)
    md = t(mod[m])                                         # [L, 6, D]

    def rope_c(a):                                         # a [L, H, 128]
        ang = t(O.rope_angles(pos))[:, None, :]
        z = torch.complex(a[..., 0::2], a[..., 1::2]) * torch.polar(torch.ones_like(ang), ang)
        return torch.stack([z.real, z.imag], dim=-1).reshape(a.shape)

    xt = t(x)
    xm = TF.layer_norm(xt, (D,), eps=1e-6) * (1 + md[:, 1]) + md[:, 0]
    qkv = TF.linear(xm, t(W["Wqkv"])).reshape(L, 3, H, 128)
    q = rope_c(TF.rms_norm(qkv[:, 0], (128,), t(W["qn_w"]), eps=1e-6))
    k = rope_c(TF.rms_norm(qkv[:, 1], (128,), t(W["kn_w"]), eps=1e-6))
    o = TF.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), qkv[:, 2].transpose(0, 1))
    x1 = xt + md[:, 2] * TF.linear(o.transpose(0, 1).reshape(L, H * 128), t(W["Wo"]))
    xm2 = TF.layer_norm(x1, (D,), eps=1e-6) * (1 + md[:, 4]) + md[:, 3]
    Fh = W["Wgu"].shape[0] // 2
    hmid = TF.silu(TF.linear(xm2, t(W["Wgu"][:Fh]))) * TF.linear(xm2, t(W["Wgu"][Fh:]))
    ref = x1 + md[:, 5] * TF.linear(hmid, t(W["Wd"]))
    _pin_close(O.block_forward(x, mod, r, pos, n_heads=H, **W), ref.numpy(), 1e-11)


def test_block_identity_with_zero_modulation():
    r, x, mod, pos, W, H = _tiny_block_inputs()
    zero = np.zeros_like(mod)
    out = O.block_forward(x, zero, r, pos, n_heads=H, **W)
    assert np.array_equal(out, x)                          # exactly: gate 0 adds +0.0
    # gate 0 on one modality leaves exactly that range unchanged
    for m in range(3):
        mod2 = mod.copy()
        mod2[m, 2] = 0
        mod2[m, 5] = 0
        out = O.block_forward(x, mod2, r, pos, n_heads=H, **W)
        rows = O.modality_of_rows(r) == m
        assert np.array_equal(out[rows], x[rows])
        assert np.all(np.abs(out[~rows] - x[~rows]).max(axis=1) > 0)


def test_block_permutation_equivariance():
    """Attention and FFN carry no modality-specific structure: permuting
    tokens together with their positions and modulation rows permutes the
    output.  Modality ranges are contiguous, so permute within each range."""
    r, x, mod, pos, W, H = _tiny_block_inputs(seed=12)
    rng = np.random.default_rng(13)
    perm = np.arange(r["L"])
    for mm in range(3):
        s, c = r["start"][mm], r["count"][mm]
        perm[s:s + c] = s + rng.permutation(c)
    a = O.block_forward(x, mod, r, pos, n_heads=H, **W)
    b = O.block_forward(x[perm], mod, r, pos[perm], n_heads=H, **W)
    _pin_close(b, a[perm], 1e-12)
    # a shift of every position by one constant leaves the block unchanged
    c = O.block_forward(x, mod, r, pos + np.array([2.0, -1.0, 3.0]), n_heads=H, **W)
    _pin_close(c, a, 1e-11)


def test_block_rows_matches_full_block():
    r, x, mod, pos, W, H = _tiny_block_inputs(seed=14)
    full = O.block_forward(x, mod, r, pos, n_heads=H, **W)
    rows = np.array([0, 3, 7, r["L"] - 1])
    part, _ = O.block_forward_rows(x, mod, r, pos, rows, n_heads=H, **W)
    _pin_close(part, full[rows], 1e-12)


# ---------------------------------------------------------------- A11

def test_sigma_schedule_closed_forms(golden):
    for s in (float(golden["video_shift"]), float(golden["audio_shift"]), 1.0, 5.0):
        sig = O.sigma_schedule(8, s)
        assert sig[0] == 1.0 and sig[-1] == 0.0
        assert np.all(np.diff(sig) < 0)
    _pin_close(O.sigma_schedule(8, 1.0), 1 - np.arange(9) / 8, 0)
    # shift maps sigma to the time whose signal-to-noise ratio (1-s)/s is divided by the shift
    sig = O.sigma_schedule(8, 12.0)[1:-1]
    base = (1 - np.arange(1, 8) / 8)
    _pin_close((1 - sig) / sig, (1 - base) / base / 12.0, 1e-12)


def test_euler_and_clean_latent_follow_rf_path():
    rng = np.random.default_rng(15)
    x0, eps = rng.standard_normal(20), rng.standard_normal(20)
    v = eps - x0
    for sig, sig2 in ((0.7, 0.0), (0.7, 0.6), (1.0, 0.25)):
        xs = (1 - sig) * x0 + sig * eps
        _pin_close(O.clean_latent(xs, v, sig), x0, 1e-14)
        _pin_close(O.euler_step(xs, v, sig, sig2), (1 - sig2) * x0 + sig2 * eps, 1e-14)
    # constant velocity: 8 shifted steps from sigma 1 land at x1 - v for any shift
    for s in (12.0, 3.0):
        sig = O.sigma_schedule(8, s)
        x = eps.copy()
        for i in range(8):
            x = O.euler_step(x, v, sig[i], sig[i + 1])
        _pin_close(x, eps - v, 1e-13)


def test_embed_matches_library_composition():
    """The residual stream the embed assembles, rebuilt from library routines:
    each modality's features through torch's linear, the audio latents made
    channel-major by an einops rearrange ((channel, latent) -> token, G6), the
    video by the 1x2x2 patchify rearrange, and the three blocks concatenated
    text -> audio -> video (G1).  Odd, unequal sizes everywhere so that a
    swapped range, an interleaved audio reshape or a transposed weight fails."""
    import einops
    rng = np.random.default_rng(21)
    n_text, d_text, ch, n_aud, c_aud, T, Hl, Wl, D = 5, 7, 2, 3, 11, 2, 4, 6, 9
    text = rng.standard_normal((n_text, d_text))
    audio = rng.standard_normal((ch, n_aud, c_aud))
    video = rng.standard_normal((T, Hl, Wl, 24))
    W_text, W_aud, W_vid = (rng.standard_normal((D, k)) for k in (d_text, c_aud, 96))
    r = O.pack_ranges(n_text, ch * n_aud, T * (Hl // 2) * (Wl // 2))
    t = torch.from_numpy
    ref = torch.cat([TF.linear(t(text), t(W_text)),
                     TF.linear(t(einops.rearrange(audio, "c n d -> (c n) d")), t(W_aud)),
                     TF.linear(t(einops.rearrange(video, "t (i ph) (j pw) c -> (t i j) (ph pw c)", ph=2, pw=2)),
                               t(W_vid))])
    _pin_close(O.embed(text, video, audio, W_text, W_vid, W_aud, r), ref.numpy(), 1e-12)
    # modality ids: the same three blocks as a run-length expansion
    ids = torch.repeat_interleave(torch.tensor([O.TEXT, O.AUDIO, O.VIDEO]), torch.tensor(r["count"]))
    assert np.array_equal(O.modality_of_rows(r), ids.numpy())


def test_head_unpack_matches_library_composition():
    """The head rebuilt from library routines: torch's non-affine layer_norm
    (eps 1e-6), the packed rows split by modality counts, torch's linear per
    modality, and the inverse rearranges of the patchify and of the
    channel-major audio packing.  Non-square head weights and unequal sizes, so
    a transposed weight or a wrong reshape fails."""
    import einops
    rng = np.random.default_rng(22)
    ch, n_aud, c_aud, T, Hl, Wl, D = 2, 5, 13, 2, 4, 6, 40
    r = O.pack_ranges(3, ch * n_aud, T * (Hl // 2) * (Wl // 2))
    x = rng.standard_normal((r["L"], D)) * 3 + 1
    Wv, Wa = rng.standard_normal((96, D)), rng.standard_normal((c_aud, D))
    vv, va = O.head_unpack(x, r, Wv, Wa, T, Hl, Wl, ch, n_aud)
    t = torch.from_numpy
    h = TF.layer_norm(t(x), (D,), eps=1e-6)
    _, ha, hv = torch.split(h, r["count"])
    ref_v = einops.rearrange(TF.linear(hv, t(Wv)).numpy(), "(t i j) (ph pw c) -> t (i ph) (j pw) c",
                             t=T, i=Hl // 2, j=Wl // 2, ph=2, pw=2)
    ref_a = einops.rearrange(TF.linear(ha, t(Wa)).numpy(), "(c n) d -> c n d", c=ch)
    _pin_close(vv, ref_v, 1e-11)
    _pin_close(va, ref_a, 1e-11)


def test_head_unpack_shapes_and_roundtrip():
    """Head shapes and the gather round trip (its form is a reading, G11)."""
    rng = np.random.default_rng(16)
    r = O.pack_ranges(3, 2 * 5, 2 * 2 * 3)
    D = 16
    x = rng.standard_normal((r["L"], D))
    Wv = rng.standard_normal((96, D))
    Wa = rng.standard_normal((64, D))
    vv, va = O.head_unpack(x, r, Wv, Wa, 2, 4, 6, 2, 5)
    assert vv.shape == (2, 4, 6, 24) and va.shape == (2, 5, 64)
    h = O.layernorm(x)
    s = r["start"][O.VIDEO]
    _pin_close(O.patchify(vv), O.linear(h[s:s + 12], Wv), 1e-12)


# ---------------------------------------------------------------- A12

def test_round_to_bf16_matches_library_conversion():
    x = (np.random.default_rng(17).standard_normal(200000) * 7).astype(np.float32)
    x[:6] = [0.0, -0.0, 1.0, -3.0e38, 2.5e-38, 1.00390625]      # 1 + 2^-8: a tie, rounds to even (1.0)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.round_to_bf16(x), ref)


def test_sampler_with_zero_head_keeps_latents_and_text():
    """A head with zero weights gives zero velocity: every Euler step leaves
    the latents exactly unchanged, for any schedule."""
    w = S.WORKLOADS["tiny"]
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, 2, 3)
    io = dict(inp)
    io["W_vhead"] = np.zeros_like(inp["W_vhead"])
    io["W_ahead"] = np.zeros_like(inp["W_ahead"])
    t, i, j = O.token_grid(w.T_lat, w.H_lat, w.W_lat)
    r = O.pack_ranges(w.n_text, w.audio_channels * w.n_audio, t * i * j)
    pos = O.positions(r, t, i, j, w.audio_channels, w.n_audio)
    lv, la = O.sample(inp["text"], st["lat_video"], st["lat_audio"], io, st["blocks"], st["mod_all"], r, pos, w.H, 3)
    assert np.array_equal(lv, st["lat_video"].astype(np.float64))
    assert np.array_equal(la, st["lat_audio"].astype(np.float64))


def test_sampler_one_step_is_euler_of_the_block_stack():
    """One step from sigma 1 to 0 moves each latent by minus its velocity
    (sum of sigma differences = -1), with the velocity of the block stack on
    the bf16-rounded latents."""
    w = S.WORKLOADS["tiny"]
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, 2, 1)
    t, i, j = O.token_grid(w.T_lat, w.H_lat, w.W_lat)
    r = O.pack_ranges(w.n_text, w.audio_channels * w.n_audio, t * i * j)
    pos = O.positions(r, t, i, j, w.audio_channels, w.n_audio)
    lv, la = O.sample(inp["text"], st["lat_video"], st["lat_audio"], inp, st["blocks"], st["mod_all"], r, pos, w.H, 1)
    x = O.embed(inp["text"], O.round_to_bf16(st["lat_video"]), O.round_to_bf16(st["lat_audio"]), inp["W_text"],
                inp["W_vid"], inp["W_aud"], r)
    for b in range(2):
        x = O.block_forward(x, st["mod_all"][0][b], r, pos, n_heads=w.H, **st["blocks"][b])
    vv, va = O.head_unpack(x, r, inp["W_vhead"], inp["W_ahead"], w.T_lat, w.H_lat, w.W_lat, w.audio_channels,
                           w.n_audio)
    _pin_close(lv, st["lat_video"] - vv, 1e-12)
    _pin_close(la, st["lat_audio"] - va, 1e-12)
