"""Float64 CPU oracle of the H3-Omni block step.  TEST INFRASTRUCTURE ONLY.

Only tests/, the graft smoke entry and the bench's CPU-baseline leg may import
this module.  It shares no code with the CUDA library: no kernel, header,
helper, table or constant generator.  It is deliberately plain and slow: NumPy
float64 with library matmuls as the only building block, in the order in which
the pages state the block.

Sources (page title, section):
  [gojay]  "MiniMax-H3 paper reading" (gojay.top), §4 VisualVAE/AudioVAE, §5
           Omni-Transformer, §7.3 VisualVAE shapes, §7.4 3-D MM-RoPE
  [shouss] "MiniMax-H3: native joint audio-video generation" (note.shouss.top),
           §2.2 packed sequence, §3 single-stream trunk with modality
           modulation, §3.1 three groups of modulation, §3.2 config table and
           Q/K RMSNorm + SiLU(gate)*up, §4.1 VisualVAE patch width, §4.3
           AudioVAE, §5 attention mask vs update mask, §6 velocity sampling
  [oceanz] "MiniMax H3 overview" cheatsheet (oceanz.site), VisualVAE section
           worked example
  [0539]   "H3's omni-modal ambition" (0539edu.com), scheduler sigma shifts

Readings adopted where the pages are silent or garbled:
  G1 packing order text -> audio -> video; G2 latent frames 1 + (T-1)//4;
  G3 RoPE split t/h/w = 32/48/48; G4 theta 10000, interleaved pairs;
  G5 positions (video (t,i,j); audio (0.15 k, 0, 0); text (0,0,0));
  G7 patch feature f = (ph*2 + pw)*24 + c; G8 LN without affine, eps 1e-6,
  Q/K RMSNorm eps 1e-6 with a [128] weight shared by heads;
  G9 h*(1+scale)+shift, residual += gate*branch, modulation layout
  [modality][shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp, gate_mlp][D];
  G10 no biases; G11 head = non-affine LN + per-modality linear;
  G12 x0 = x - sigma v, Euler x += (sigma' - sigma) v; G13 uniform sigmas with
  shift s*sigma / (1 + (s-1) sigma); G22 AdaLN producer = SiLU then one
  linear per block from a D/2-wide conditioning vector to 18 D.

Parity pins: every function here is pinned by tests/test_oracle_*.py.
`head_unpack` computes what reading G11 states and is pinned to that
statement composed from library routines; the reading itself (a non-affine LN
and one linear per modality, no final modulation) has nothing on the pages to
pin it against.
"""
from __future__ import annotations

import numpy as np

TEXT, AUDIO, VIDEO = 0, 1, 2          # modality ids, in packing order (G1)
MSA, MLP = 0, 1                        # branch selector
SHIFT, SCALE, GATE = 0, 1, 2           # position inside a branch's triple
EPS_LN = 1e-6
EPS_QK = 1e-6
ROPE_THETA = 10000.0
AUDIO_HZ = 40.0                        # AudioVAE latent rate per channel [shouss §4.3]
VIDEO_LATENT_HZ = 24.0 / 4.0           # 24 fps, 4x temporal compression [gojay §4]


# --------------------------------------------------------------------------
# A1  token grid, patchify, packing, positions
# --------------------------------------------------------------------------

def latent_frames(n_frames: int) -> int:
    """Latent frames of the temporally-causal f16t4d24 VAE: the first frame is
    kept, every further 4 frames make one latent frame [gojay §4] (G2)."""
    return 1 + (n_frames - 1) // 4


def latent_hw(height: int, width: int) -> tuple[int, int]:
    """f16: height and width each divided by 16 [gojay §4; oceanz VisualVAE]."""
    return height // 16, width // 16


def token_grid(t_lat: int, h_lat: int, w_lat: int) -> tuple[int, int, int]:
    """1x2x2 patchify over (t, h, w): time untouched, space halved [gojay §4, §7.3]."""
    return t_lat, h_lat // 2, w_lat // 2


def patch_width(c_lat: int = 24) -> int:
    """Width of one patch before its projection: 1*2*2*channels [shouss §4.1]."""
    return 1 * 2 * 2 * c_lat


def patchify(lat: np.ndarray) -> np.ndarray:
    """(T, H, W, C) channels-last latent -> (T*(H/2)*(W/2), 4C) patches.

    Row r = (t*(H/2) + i)*(W/2) + j, the t-major flatten of the token grid
    [gojay §7.3]; feature f = (ph*2 + pw)*C + c (G7)."""
    T, H, W, C = lat.shape
    assert H % 2 == 0 and W % 2 == 0
    out = np.empty((T * (H // 2) * (W // 2), 4 * C), dtype=lat.dtype)
    r = 0
    for t in range(T):
        for i in range(H // 2):
            for j in range(W // 2):
                for ph in range(2):
                    for pw in range(2):
                        f0 = (ph * 2 + pw) * C
                        out[r, f0:f0 + C] = lat[t, 2 * i + ph, 2 * j + pw, :]
                r += 1
    return out


def unpatchify(patches: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    """Inverse of `patchify` (the gather written the other way round)."""
    C = patches.shape[1] // 4
    lat = np.empty((T, H, W, C), dtype=patches.dtype)
    r = 0
    for t in range(T):
        for i in range(H // 2):
            for j in range(W // 2):
                for ph in range(2):
                    for pw in range(2):
                        f0 = (ph * 2 + pw) * C
                        lat[t, 2 * i + ph, 2 * j + pw, :] = patches[r, f0:f0 + C]
                r += 1
    return lat


def pack_ranges(n_text: int, n_audio_tokens: int, n_video_tokens: int, tile: int = 128) -> dict:
    """Packed-sequence index ranges, text -> audio -> target video -> padding
    [shouss §2.2] (G1).  Returns start/count per modality id, L and L_pad."""
    start = [0, n_text, n_text + n_audio_tokens]
    count = [n_text, n_audio_tokens, n_video_tokens]
    L = n_text + n_audio_tokens + n_video_tokens
    L_pad = -(-L // tile) * tile
    return {"start": start, "count": count, "L": L, "L_pad": L_pad}


def modality_of_rows(ranges: dict) -> np.ndarray:
    """Modality id of each valid row (the range that holds it)."""
    m = np.empty(ranges["L"], dtype=np.int64)
    for mod in (TEXT, AUDIO, VIDEO):
        s, c = ranges["start"][mod], ranges["count"][mod]
        m[s:s + c] = mod
    return m


def positions(ranges: dict, t_lat: int, h_tok: int, w_tok: int,
              audio_channels: int, n_audio: int) -> np.ndarray:
    """(t, h, w) position of every valid token, float64 [L, 3].

    Video token (t, i, j) sits at (t, i, j); audio latent k of either channel at
    (k * 6/40, 0, 0): video latents run at 24/4 = 6 Hz and audio latents at 40
    Hz, so both share one time axis in video-latent-frame units, with h = w = 0
    for audio [gojay §7.4, FAQ Q6; shouss §5] (G5).  Text sits at (0, 0, 0)."""
    pos = np.zeros((ranges["L"], 3), dtype=np.float64)
    s = ranges["start"][AUDIO]
    for c in range(audio_channels):
        for k in range(n_audio):
            pos[s + c * n_audio + k] = (k * VIDEO_LATENT_HZ / AUDIO_HZ, 0.0, 0.0)
    s = ranges["start"][VIDEO]
    r = 0
    for t in range(t_lat):
        for i in range(h_tok):
            for j in range(w_tok):
                pos[s + r] = (t, i, j)
                r += 1
    return pos


# --------------------------------------------------------------------------
# A2  per-modality input projections
# --------------------------------------------------------------------------

def linear(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y = x W^T with W stored [out, in]; no bias (G10)."""
    return np.asarray(x, np.float64) @ np.asarray(W, np.float64).T


def embed(text, video_lat, audio_lat, W_text, W_vid, W_aud, ranges) -> np.ndarray:
    """Residual stream x [L, D]: each modality through its own input projection
    into the shared hidden width [gojay §5; shouss §2.2]."""
    D = W_text.shape[0]
    x = np.zeros((ranges["L"], D), dtype=np.float64)
    patches = patchify(video_lat)
    audio_tokens = audio_lat.reshape(-1, audio_lat.shape[-1])     # channel-major (G6)
    for mod, feats, W in ((TEXT, text, W_text), (AUDIO, audio_tokens, W_aud), (VIDEO, patches, W_vid)):
        s, c = ranges["start"][mod], ranges["count"][mod]
        assert feats.shape[0] == c
        x[s:s + c] = linear(feats, W)
    return x


# --------------------------------------------------------------------------
# A3/A8  LayerNorm + range-selected modulation
# --------------------------------------------------------------------------

def layernorm(x: np.ndarray, eps: float = EPS_LN) -> np.ndarray:
    """Non-affine LayerNorm over the last axis, biased variance (G8)."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def adaln_modulate(x: np.ndarray, mod: np.ndarray, ranges: dict, branch: int) -> np.ndarray:
    """h*(1 + scale_m) + shift_m with the modality m of each row's token range
    [shouss §3, §3.1] (G9).  mod is [3][6][D]."""
    mod = np.asarray(mod, np.float64)
    h = layernorm(x)
    m = modality_of_rows(ranges)
    shift = mod[m, 3 * branch + SHIFT]
    scale = mod[m, 3 * branch + SCALE]
    return h * (1.0 + scale) + shift


# --------------------------------------------------------------------------
# A4/A5  QKV, per-head Q/K RMSNorm, 3-D MM-RoPE
# --------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float = EPS_QK) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis [shouss §3.2]."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def rope_angles(pos: np.ndarray, split=(32, 48, 48), theta: float = ROPE_THETA) -> np.ndarray:
    """Rotation angle of every (token, pair) [L, head_dim/2].

    head_dim is split into t | h | w sections [gojay §7.4] (G3); inside a
    section of width d, pair i rotates by p_axis * theta^(-2i/d) (G4)."""
    cols = []
    for axis, d in enumerate(split):
        i = np.arange(d // 2, dtype=np.float64)
        freq = theta ** (-2.0 * i / d)
        cols.append(pos[:, axis:axis + 1] * freq[None, :])
    return np.concatenate(cols, axis=1)


def rope(x: np.ndarray, pos: np.ndarray, split=(32, 48, 48), theta: float = ROPE_THETA) -> np.ndarray:
    """Rotate interleaved pairs (2i, 2i+1) of each head vector; x [L, n_heads, hd]."""
    ang = rope_angles(pos, split, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x, dtype=np.float64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def qkv_qknorm_mrope(xm, Wqkv, qn_w, kn_w, pos, n_heads, head_dim=128, split=(32, 48, 48)):
    """QKV projection to 3 x heads*128, then per-head RMSNorm of Q and K, then
    RoPE [shouss §3.2].  Returns q, k, v as [L, heads, head_dim]."""
    L = xm.shape[0]
    I = n_heads * head_dim
    qkv = linear(xm, Wqkv)
    q = qkv[:, 0 * I:1 * I].reshape(L, n_heads, head_dim)
    k = qkv[:, 1 * I:2 * I].reshape(L, n_heads, head_dim)
    v = qkv[:, 2 * I:3 * I].reshape(L, n_heads, head_dim)
    q = rope(rmsnorm(q, qn_w), pos, split)
    k = rope(rmsnorm(k, kn_w), pos, split)
    return q, k, v


# --------------------------------------------------------------------------
# A6  full non-causal attention
# --------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) v per head over all valid tokens, non-causal
    [shouss §5; gojay §5].  Two passes: row max, then exp/sum.  Out [L, heads*hd]."""
    L, Hh, hd = q.shape
    out = np.empty((L, Hh, hd), dtype=np.float64)
    for h in range(Hh):
        s = (q[:, h, :] @ k[:, h, :].T) / np.sqrt(hd)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out.reshape(L, Hh * hd)


def attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """`attention` for a subset of query rows against all keys (same formula)."""
    n, Hh, hd = q_rows.shape
    out = np.empty((n, Hh, hd), dtype=np.float64)
    for h in range(Hh):
        s = (q_rows[:, h, :] @ k[:, h, :].T) / np.sqrt(hd)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out.reshape(n, Hh * hd)


# --------------------------------------------------------------------------
# A7/A9  gated residual branches
# --------------------------------------------------------------------------

def gate_rows(mod: np.ndarray, ranges: dict, branch: int, rows=None) -> np.ndarray:
    m = modality_of_rows(ranges)
    if rows is not None:
        m = m[rows]
    return np.asarray(mod, np.float64)[m, 3 * branch + GATE]


def gated_residual(x, o, Wo, mod, ranges, rows=None) -> np.ndarray:
    """x + gate_msa[m] * (o Wo^T) [shouss §3]."""
    return np.asarray(x, np.float64) + gate_rows(mod, ranges, MSA, rows) * linear(o, Wo)


def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def ffn_swiglu(x, xm, Wgu, Wd, mod, ranges, rows=None) -> np.ndarray:
    """x + gate_mlp[m] * ((SiLU(xm Wg^T) * (xm Wu^T)) Wd^T), Wgu = [gate; up]
    [shouss §3, §3.2]."""
    F = Wgu.shape[0] // 2
    g = linear(xm, Wgu[:F])
    u = linear(xm, Wgu[F:])
    h = silu(g) * u
    return np.asarray(x, np.float64) + gate_rows(mod, ranges, MLP, rows) * linear(h, Wd)


# --------------------------------------------------------------------------
# The block
# --------------------------------------------------------------------------

def block_forward(x, mod, ranges, pos, Wqkv, qn_w, kn_w, Wo, Wgu, Wd, n_heads,
                  head_dim=128, split=(32, 48, 48), return_parts=False):
    """One H3-Omni block over the packed sequence [shouss §3]:
    norm + modality shift/scale -> shared attention + modality gate + residual
    -> norm + modality shift/scale -> shared gated FFN + modality gate + residual."""
    x = np.asarray(x, np.float64)
    xm1 = adaln_modulate(x, mod, ranges, MSA)
    q, k, v = qkv_qknorm_mrope(xm1, Wqkv, qn_w, kn_w, pos, n_heads, head_dim, split)
    o = attention(q, k, v)
    x1 = gated_residual(x, o, Wo, mod, ranges)
    xm2 = adaln_modulate(x1, mod, ranges, MLP)
    x2 = ffn_swiglu(x1, xm2, Wgu, Wd, mod, ranges)
    if return_parts:
        return x2, {"xm1": xm1, "q": q, "k": k, "v": v, "o": o, "x1": x1, "xm2": xm2}
    return x2


def block_forward_rows(x, mod, ranges, pos, rows, Wqkv, qn_w, kn_w, Wo, Wgu, Wd, n_heads,
                       head_dim=128, split=(32, 48, 48)):
    """`block_forward` evaluated only at the given output rows.  K and V are
    computed for every token (attention reads all of them), one head at a
    time so that memory stays at one head's K/V; everything row-local is
    computed for the sampled rows only.  Same formulas as `block_forward`."""
    x = np.asarray(x, np.float64)
    rows = np.asarray(rows)
    I = n_heads * head_dim
    xm_all = adaln_modulate(x, mod, ranges, MSA)
    o = np.empty((len(rows), n_heads, head_dim), dtype=np.float64)
    for h in range(n_heads):
        cols = slice(h * head_dim, (h + 1) * head_dim)
        wq = Wqkv[0 * I:1 * I][cols]
        wk = Wqkv[1 * I:2 * I][cols]
        wv = Wqkv[2 * I:3 * I][cols]
        k = rope(rmsnorm(linear(xm_all, wk)[:, None, :], kn_w), pos, split)
        v = linear(xm_all, wv)[:, None, :]
        q = rope(rmsnorm(linear(xm_all[rows], wq)[:, None, :], qn_w), pos[rows], split)
        o[:, h, :] = attention_rows(q, k, v)
    o = o.reshape(len(rows), I)
    x1 = gated_residual(x[rows], o, Wo, mod, ranges, rows)
    m = modality_of_rows(ranges)[rows]
    modv = np.asarray(mod, np.float64)
    xm2 = layernorm(x1) * (1.0 + modv[m, 3 * MLP + SCALE]) + modv[m, 3 * MLP + SHIFT]
    x2 = ffn_swiglu(x1, xm2, Wgu, Wd, mod, ranges, rows)
    return x2, {"x1": x1, "o": o}


# --------------------------------------------------------------------------
# A10  output head (reading G11; pinned to the reading's library composition)
# --------------------------------------------------------------------------

def head_unpack(x, ranges, W_vhead, W_ahead, t_lat, h_lat, w_lat, audio_channels, n_audio):
    """Non-affine LN, per-modality linear to the latent width, then the inverse
    of the packing gather.  Returns (v_video [T,H,W,24], v_audio [ch,N,C_a])."""
    h = layernorm(x)
    sv, cv = ranges["start"][VIDEO], ranges["count"][VIDEO]
    sa, ca = ranges["start"][AUDIO], ranges["count"][AUDIO]
    v_video = unpatchify(linear(h[sv:sv + cv], W_vhead), t_lat, h_lat, w_lat)
    v_audio = linear(h[sa:sa + ca], W_ahead).reshape(audio_channels, n_audio, np.asarray(W_ahead).shape[0])
    return v_video, v_audio


# --------------------------------------------------------------------------
# NEXT-3  AdaLN modulation producer (reading G22)
# --------------------------------------------------------------------------

def adaln_modulation(c, W, D: int) -> np.ndarray:
    """The modulation of one block from conditioning vectors c [n, C]
    (timestep + condition embedding; the pages say the AdaLN outputs depend
    on these alone and can be precomputed [gojay §5; shouss §3.1]): SiLU, then
    the block's own linear W [18 D, C] (no bias, G10), read as
    [3 modalities][shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp,
    gate_mlp][D] (G9).  Returns [n, 3, 6, D]."""
    c = np.atleast_2d(np.asarray(c, np.float64))
    return linear(silu(c), W).reshape(c.shape[0], 3, 6, D)


# --------------------------------------------------------------------------
# A12  the sampler loop
# --------------------------------------------------------------------------

def round_to_bf16(a):
    """Nearest bfloat16 value (8 significant bits, ties to even), as float64:
    the transformer reads its latent inputs in bf16, so the sampler loop
    rounds the latent there, as the GPU path does."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                       # a = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def sample(text, lat_video, lat_audio, io, blocks, mod_all, ranges, pos, n_heads, n_steps,
           shift_video=12.0, shift_audio=3.0, head_dim=128, split=(32, 48, 48)):
    """n_steps Euler steps of the flow sampler over a stack of blocks
    [shouss §6; 0539 scheduler shifts]: each step packs and projects the
    bf16-rounded latents, runs every block with its own modulation
    mod_all[step][block], maps the result to per-modality velocities with the
    head and moves each latent along its own shifted schedule; the text is a
    condition and is never updated [shouss §5].  Returns the final latents."""
    sv, sa = sigma_schedule(n_steps, shift_video), sigma_schedule(n_steps, shift_audio)
    lv = np.asarray(lat_video, np.float64).copy()
    la = np.asarray(lat_audio, np.float64).copy()
    T, Hl, Wl, _ = lv.shape
    ch, na, _ = la.shape
    for s in range(n_steps):
        x = embed(text, round_to_bf16(lv), round_to_bf16(la), io["W_text"], io["W_vid"], io["W_aud"], ranges)
        for b, W in enumerate(blocks):
            x = block_forward(x, mod_all[s][b], ranges, pos, W["Wqkv"], W["qn_w"], W["kn_w"], W["Wo"], W["Wgu"],
                              W["Wd"], n_heads, head_dim, split)
        vv, va = head_unpack(x, ranges, io["W_vhead"], io["W_ahead"], T, Hl, Wl, ch, na)
        lv = euler_step(lv, vv, sv[s], sv[s + 1])
        la = euler_step(la, va, sa[s], sa[s + 1])
    return lv, la


# --------------------------------------------------------------------------
# A11  flow sampler
# --------------------------------------------------------------------------

def shift_sigma(sigma, shift: float):
    """Time shift s*sigma / (1 + (s-1)*sigma); video 12.0, audio 3.0
    [shouss §6; 0539 scheduler configuration] (G13)."""
    sigma = np.asarray(sigma, np.float64)
    return shift * sigma / (1.0 + (shift - 1.0) * sigma)


def sigma_schedule(n_steps: int, shift: float) -> np.ndarray:
    """n_steps + 1 sigmas from 1 to 0, uniform then shifted (G13)."""
    return shift_sigma(1.0 - np.arange(n_steps + 1, dtype=np.float64) / n_steps, shift)


def clean_latent(x, v, sigma):
    """RF convention x_sigma = (1 - sigma) x0 + sigma eps, v = eps - x0, so
    x0 = x - sigma v [shouss §6] (G12)."""
    return np.asarray(x, np.float64) - sigma * np.asarray(v, np.float64)


def euler_step(x, v, sigma, sigma_next):
    """x + (sigma_next - sigma) v: one Euler step of dx/dsigma = v on the
    generation targets only; conditions stay fixed [shouss §5, §6] (G12)."""
    return np.asarray(x, np.float64) + (sigma_next - sigma) * np.asarray(v, np.float64)
