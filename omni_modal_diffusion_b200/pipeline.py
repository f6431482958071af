"""Device buffers and the call sequence of one H3-Omni block step.

Orchestration only: allocation through torch, then the C-ABI calls in the
order of the block ("MiniMax-H3: native joint audio-video generation"
(note.shouss.top) §3): embed/pack -> LN+modulate -> QKV (+Q/K RMSNorm,
3-D RoPE) -> attention -> gated out-projection -> LN+modulate -> gated
SwiGLU FFN -> head -> Euler.  No arithmetic of the block happens here.
"""
from __future__ import annotations

import numpy as np
import torch

from . import h3
from .synthetic import Workload


def to_dev_bf16(a: np.ndarray, device) -> torch.Tensor:
    """bf16-exact float32 array -> bf16 CUDA tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device).to(torch.bfloat16)


class H3BlockStep:
    WEIGHTS = ("W_text", "W_vid", "W_aud", "Wqkv", "qn_w", "kn_w", "Wo", "Wgu", "Wd", "W_vhead", "W_ahead")

    def __init__(self, w: Workload, device="cuda", weights: dict | None = None, n_layers: int = 1):
        self.w = w
        self.device = torch.device(device)
        self.dims = h3.make_dims(w.D, w.H, w.F, head_dim=w.head_dim, rope=w.rope_split)
        self.n_video = w.T_lat * (w.H_lat // 2) * (w.W_lat // 2)
        self.n_audio_tok = w.audio_channels * w.n_audio
        self.ranges = h3.h3_make_ranges(w.n_text, self.n_audio_tok, self.n_video)
        Lp, D, I, F = self.ranges.L_pad, w.D, w.I, w.F
        dev = self.device
        e = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=dev)
        self.x = e(Lp, D)
        self.pos = e(Lp, 3)
        self.mod_ids = e(Lp, dt=torch.uint8)
        self.patches = e(max(self.n_video, 1), 4 * w.C_lat, dt=torch.bfloat16)
        self.xm = e(Lp, D, dt=torch.bfloat16)
        self.q = e(w.H, Lp, 128, dt=torch.bfloat16)
        self.k = e(w.H, Lp, 128, dt=torch.bfloat16)
        self.v = e(w.H, Lp, 128, dt=torch.bfloat16)
        self.o = e(Lp, I, dt=torch.bfloat16)
        self.ws = e(Lp, F, dt=torch.bfloat16)
        self.hn = e(Lp, D, dt=torch.bfloat16)
        self.v_video = e(w.T_lat, w.H_lat, w.W_lat, w.C_lat)
        self.v_audio = e(w.audio_channels, w.n_audio, w.C_audio)
        self.W = {}
        if weights is not None:
            self.load_weights(weights)

    def load_weights(self, weights: dict):
        for k in self.WEIGHTS:
            v = weights[k]
            self.W[k] = v if isinstance(v, torch.Tensor) else to_dev_bf16(v, self.device)

    # ---------------------------------------------------------- steps
    def embed(self, text, video, audio, stream=None):
        W = self.W
        h3.h3_embed_pack(self.dims, self.ranges, text, video, audio, W["W_text"], W["W_vid"], W["W_aud"],
                         self.patches, self.x, self.pos, self.mod_ids, stream=stream)

    def block(self, mod, W=None, stream=None):
        """One block over self.x in place; W defaults to the step's weights."""
        W = W or self.W
        d, r = self.dims, self.ranges
        h3.h3_adaln_norm_modulate(d, r, self.x, mod, h3.H3_MSA, self.xm, stream=stream)
        h3.h3_qkv_qknorm_mrope(d, r, self.xm, W["Wqkv"], W["qn_w"], W["kn_w"], self.pos, self.q, self.k, self.v,
                               stream=stream)
        h3.h3_attention(d, r, self.q, self.k, self.v, self.o, stream=stream)
        h3.h3_gated_residual(d, r, self.x, self.o, W["Wo"], mod, h3.H3_MSA, stream=stream)
        h3.h3_adaln_norm_modulate(d, r, self.x, mod, h3.H3_MLP, self.xm, stream=stream)
        h3.h3_ffn_swiglu(d, r, self.x, self.xm, W["Wgu"], W["Wd"], mod, self.ws, stream=stream)

    def head(self, stream=None):
        w = self.w
        h3.h3_head_unpack(self.dims, self.ranges, self.x, self.W["W_vhead"], self.W["W_ahead"],
                          (w.T_lat, w.H_lat, w.W_lat, w.C_lat), (w.audio_channels, w.n_audio, w.C_audio),
                          self.hn, self.v_video, self.v_audio, stream=stream)

    def euler(self, lat_video, lat_audio, sig_video, sig_audio, stream=None):
        """sig_* = (sigma, sigma_next) of each modality's own schedule."""
        h3.h3_euler_step(lat_video, self.v_video, sig_video[0], sig_video[1], stream=stream)
        h3.h3_euler_step(lat_audio, self.v_audio, sig_audio[0], sig_audio[1], stream=stream)

    def step(self, text, video, audio, mod, lat_video, lat_audio, sig_video, sig_audio, stream=None):
        """The whole hot path once: pack/project, one block, head, Euler x2."""
        self.embed(text, video, audio, stream)
        self.block(mod, stream=stream)
        self.head(stream)
        self.euler(lat_video, lat_audio, sig_video, sig_audio, stream)

    # kernels launched by one step (for the launch count the bench reports)
    def launches_per_step(self) -> int:
        r = self.ranges
        embed = (1 if r.count[2] > 0 else 0) + 1 + (1 if r.L_pad > r.L else 0) + sum(1 for c in r.count if c > 0)
        block = 1 + 1 + 1 + 1 + 1 + 2
        head = 1 + (1 if r.count[2] > 0 else 0) + (1 if r.count[1] > 0 else 0)
        return embed + block + head + 2
