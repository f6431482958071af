"""Seeded synthetic inputs shared by the CUDA path, its tests and the bench.

This module draws random numbers and states workload shapes; it holds none of
the block's arithmetic (no packing, no positions, no norms, no projections).
Every floating-point tensor is drawn in float32 and rounded once to bfloat16
(round-to-nearest-even) so that the GPU path and the float64 oracle see the
identical values: the oracle upcasts the rounded values, the GPU path reads
their bf16 bit patterns.

Workloads (the shapes of the pages' 768p, 24 fps, 32 kHz-stereo outputs; the
latent shapes below are the causal VisualVAE's f16t4d24 output for the stated
frame counts and pixel sizes, and 40 latents per second per audio channel):

  tiny      hidden 320, 4 heads, FFN 896; text 16 x 256; video latent
            2 x 8 x 8 x 24; audio 2 channels x 8 latents x 64; sigma 0.7
  768sq_2s  hidden 5376, 56 heads, FFN 14336; 768x768, 49 frames
            (latent 13 x 48 x 48 x 24); audio 2 x 80 x 64; text 256 x 5120
  768x1344_5s  121 frames (latent 31 x 48 x 84 x 24); audio 2 x 200 x 64;
            text 512 x 5120
  768x1792_15s 361 frames (latent 91 x 48 x 112 x 24); audio 2 x 600 x 64;
            text 512 x 5120

Distributions: weights N(0, 0.02); latents N(0, 1); text features N(0, 1);
modulation N(0, 0.1) as float32 [3][6][D] (not rounded: it is an fp32 input);
Q/K-norm weights 1 + 0.1 N(0, 1).  Seed = 1234 + workload index.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    D: int          # residual width
    H: int          # attention heads
    head_dim: int
    F: int          # gated-FFN inner width
    D_text: int     # text feature width
    n_text: int
    T_lat: int      # video latent frames
    H_lat: int      # video latent height
    W_lat: int      # video latent width
    C_lat: int      # video latent channels
    n_audio: int    # latents per audio channel
    audio_channels: int
    C_audio: int    # audio latent width
    rope_split: tuple = (32, 48, 48)
    sigma: float = 0.7

    @property
    def I(self) -> int:
        return self.H * self.head_dim


WORKLOADS = {
    "tiny": Workload("tiny", 0, 320, 4, 128, 896, 256, 16, 2, 8, 8, 24, 8, 2, 64),
    "768sq_2s": Workload("768sq_2s", 1, 5376, 56, 128, 14336, 5120, 256, 13, 48, 48, 24, 80, 2, 64),
    "768x1344_5s": Workload("768x1344_5s", 2, 5376, 56, 128, 14336, 5120, 512, 31, 48, 84, 24, 200, 2, 64),
    "768x1792_15s": Workload("768x1792_15s", 3, 5376, 56, 128, 14336, 5120, 512, 91, 48, 112, 24, 600, 2, 64),
}


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = u + np.uint32(0x7FFF)                 # new array: the input is not modified
    r += (u >> np.uint32(16)) & np.uint32(1)
    r &= np.uint32(0xFFFF0000)
    out = r.view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = a[nan]
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-exact float32 values, as uint16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _normal(rng, shape, std=1.0, mean=0.0):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return a


def make_inputs(w: Workload, seed: int | None = None, weights: bool = True) -> dict:
    """All inputs of one block step, float32 arrays holding bf16-exact values.

    Keys: text [n_text, D_text], video [T, Hl, Wl, 24], audio [ch, n_audio, C_a],
    W_text [D, D_text], W_vid [D, 96], W_aud [D, C_a], Wqkv [3I, D],
    qn_w [head_dim], kn_w [head_dim], Wo [D, I], Wgu [2F, D] (gate rows then
    up rows), Wd [D, F], W_vhead [96, D], W_ahead [C_a, D], mod [3, 6, D]
    (float32, not rounded).
    """
    rng = np.random.default_rng(1234 + w.index if seed is None else seed)
    out = {}
    out["text"] = bf16_round(_normal(rng, (w.n_text, w.D_text)))
    out["video"] = bf16_round(_normal(rng, (w.T_lat, w.H_lat, w.W_lat, w.C_lat)))
    out["audio"] = bf16_round(_normal(rng, (w.audio_channels, w.n_audio, w.C_audio)))
    out["mod"] = _normal(rng, (3, 6, w.D), std=0.1)
    patch = 4 * w.C_lat
    if weights:
        out["W_text"] = bf16_round(_normal(rng, (w.D, w.D_text), 0.02))
        out["W_vid"] = bf16_round(_normal(rng, (w.D, patch), 0.02))
        out["W_aud"] = bf16_round(_normal(rng, (w.D, w.C_audio), 0.02))
        out["Wqkv"] = bf16_round(_normal(rng, (3 * w.I, w.D), 0.02))
        out["qn_w"] = bf16_round(_normal(rng, (w.head_dim,), 0.1, 1.0))
        out["kn_w"] = bf16_round(_normal(rng, (w.head_dim,), 0.1, 1.0))
        out["Wo"] = bf16_round(_normal(rng, (w.D, w.I), 0.02))
        out["Wgu"] = bf16_round(_normal(rng, (2 * w.F, w.D), 0.02))
        out["Wd"] = bf16_round(_normal(rng, (w.D, w.F), 0.02))
        out["W_vhead"] = bf16_round(_normal(rng, (patch, w.D), 0.02))
        out["W_ahead"] = bf16_round(_normal(rng, (w.C_audio, w.D), 0.02))
    return out


def random_rows(n_valid: int, k: int, seed: int) -> np.ndarray:
    """k distinct sorted row indices in [0, n_valid) (parity sampling at full size)."""
    rng = np.random.default_rng(seed)
    k = min(k, n_valid)
    return np.sort(rng.choice(n_valid, size=k, replace=False))


def make_stack_inputs(w: Workload, n_layers: int, n_steps: int, seed: int | None = None) -> dict:
    """Inputs of the layered sampler: per-block weights (list of dicts with
    Wqkv, qn_w, kn_w, Wo, Wgu, Wd as in make_inputs), modulation
    mod_all [n_steps][n_layers][3][6][D] float32 N(0, 0.1), and the initial
    latents at sigma = 1 (float32 N(0, 1), not rounded: the sampler state is
    fp32; the transformer reads its bf16 rounding)."""
    rng = np.random.default_rng((7777 + w.index) if seed is None else seed)
    blocks = []
    for _ in range(n_layers):
        blocks.append({
            "Wqkv": bf16_round(_normal(rng, (3 * w.I, w.D), 0.02)),
            "qn_w": bf16_round(_normal(rng, (w.head_dim,), 0.1, 1.0)),
            "kn_w": bf16_round(_normal(rng, (w.head_dim,), 0.1, 1.0)),
            "Wo": bf16_round(_normal(rng, (w.D, w.I), 0.02)),
            "Wgu": bf16_round(_normal(rng, (2 * w.F, w.D), 0.02)),
            "Wd": bf16_round(_normal(rng, (w.D, w.F), 0.02)),
        })
    return {
        "blocks": blocks,
        "mod_all": _normal(rng, (n_steps, n_layers, 3, 6, w.D), std=0.1),
        "lat_video": _normal(rng, (w.T_lat, w.H_lat, w.W_lat, w.C_lat)),
        "lat_audio": _normal(rng, (w.audio_channels, w.n_audio, w.C_audio)),
    }
