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
        # where the per-head Q/K RMSNorm + RoPE run: the QKV epilogue (the
        # default, once per token) or, with 0, attention's prologue
        self.qk_flags = h3.H3_QK_NORM_ROPE_IN_QKV
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
        """Upload the weights present in `weights` (block weights are optional:
        the layered sampler keeps them per block)."""
        for k in self.WEIGHTS:
            if k not in weights:
                continue
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
                               flags=self.qk_flags, stream=stream)
        h3.h3_attention(d, r, self.q, self.k, self.v, self.o, qn_w=W["qn_w"], kn_w=W["kn_w"], pos=self.pos,
                        flags=self.qk_flags, stream=stream)
        h3.h3_gated_residual(d, r, self.x, self.o, W["Wo"], mod, h3.H3_MSA, stream=stream)
        h3.h3_adaln_norm_modulate(d, r, self.x, mod, h3.H3_MLP, self.xm, stream=stream)
        h3.h3_ffn_swiglu(d, r, self.x, self.xm, W["Wgu"], W["Wd"], mod, self.ws, stream=stream)

    # ---------------------------------------------------------- e4m3 GEMMs
    def quantize_block_weights_e4m3(self, W=None, stream=None) -> dict:
        """e4m3 codes + per-output-channel scales of a block's GEMM weights
        (h3_quantize_rows_e4m3 on the GPU), with qn_w / kn_w passed through."""
        W = W or self.W
        out = {"qn_w": W["qn_w"], "kn_w": W["kn_w"]}
        for n in ("Wqkv", "Wo", "Wgu", "Wd"):
            t = W[n]
            q = torch.empty(t.shape, dtype=torch.uint8, device=self.device)
            sc = torch.empty(t.shape[0], dtype=torch.float32, device=self.device)
            h3.h3_quantize_rows_e4m3(t, q, sc, stream=stream)
            out[n], out[n + "_s"] = q, sc
        return out

    def alloc_e4m3(self):
        """Activation buffers of the e4m3 path (codes and row scales)."""
        Lp, D, I = self.ranges.L_pad, self.w.D, self.w.I
        dev = self.device
        self.xq = torch.empty(Lp, D, dtype=torch.uint8, device=dev)
        self.xs = torch.empty(Lp, dtype=torch.float32, device=dev)
        self.oq = torch.empty(Lp, I, dtype=torch.uint8, device=dev)
        self.os = torch.empty(Lp, dtype=torch.float32, device=dev)
        self.ws8 = torch.empty(h3.h3_ffn_e4m3_workspace_bytes(self.dims, Lp), dtype=torch.uint8, device=dev)
        # q, k as e4m3 codes (H3_QK_E4M3)
        self.q8 = torch.empty(self.w.H, Lp, 128, dtype=torch.uint8, device=dev)
        self.k8 = torch.empty(self.w.H, Lp, 128, dtype=torch.uint8, device=dev)

    def block_e4m3(self, mod, W8: dict, stream=None, qk_e4m3: bool = False):
        """One block over self.x with the four GEMMs in e4m3 (W8 from
        quantize_block_weights_e4m3; alloc_e4m3 called once before);
        qk_e4m3 also passes q, k to attention as e4m3 codes (H3_QK_E4M3)."""
        d, r = self.dims, self.ranges
        flags = h3.H3_QK_NORM_ROPE_IN_QKV | (h3.H3_QK_E4M3 if qk_e4m3 else 0)
        q, k = (self.q8, self.k8) if qk_e4m3 else (self.q, self.k)
        h3.h3_adaln_norm_modulate_e4m3(d, r, self.x, mod, h3.H3_MSA, self.xq, self.xs, stream=stream)
        h3.h3_qkv_qknorm_mrope_e4m3(d, r, self.xq, self.xs, W8["Wqkv"], W8["Wqkv_s"], W8["qn_w"], W8["kn_w"],
                                    self.pos, q, k, self.v, flags=flags, stream=stream)
        h3.h3_attention(d, r, q, k, self.v, self.o, qn_w=W8["qn_w"], kn_w=W8["kn_w"], flags=flags, stream=stream)
        h3.h3_quantize_rows_e4m3(self.o, self.oq, self.os, stream=stream)
        h3.h3_gated_residual_e4m3(d, r, self.x, self.oq, self.os, W8["Wo"], W8["Wo_s"], mod, h3.H3_MSA,
                                  stream=stream)
        h3.h3_adaln_norm_modulate_e4m3(d, r, self.x, mod, h3.H3_MLP, self.xq, self.xs, stream=stream)
        h3.h3_ffn_swiglu_e4m3(d, r, self.x, self.xq, self.xs, W8["Wgu"], W8["Wgu_s"], W8["Wd"], W8["Wd_s"], mod,
                              self.ws8, stream=stream)

    def head(self, stream=None):
        w = self.w
        h3.h3_head_unpack(self.dims, self.ranges, self.x, self.W["W_vhead"], self.W["W_ahead"],
                          (w.T_lat, w.H_lat, w.W_lat, w.C_lat), (w.audio_channels, w.n_audio, w.C_audio),
                          self.hn, self.v_video, self.v_audio, stream=stream)

    def euler(self, lat_video, lat_audio, sig_video, sig_audio, stream=None):
        """sig_* = (sigma, sigma_next) of each modality's own schedule."""
        h3.h3_euler_step(lat_video, self.v_video, sig_video[0], sig_video[1], stream=stream)
        h3.h3_euler_step(lat_audio, self.v_audio, sig_audio[0], sig_audio[1], stream=stream)

    def head_euler(self, lat_video, lat_audio, sig_video, sig_audio, video_bf16=None, audio_bf16=None, stream=None):
        """Head and Euler step in one call (h3_head_euler): the latents move
        by (sigma_next - sigma) * velocity in the head GEMMs' epilogues; the
        bf16 copies, when given, receive the updated latents."""
        w = self.w
        h3.h3_head_euler(self.dims, self.ranges, self.x, self.W["W_vhead"], self.W["W_ahead"],
                         (w.T_lat, w.H_lat, w.W_lat, w.C_lat), (w.audio_channels, w.n_audio, w.C_audio), self.hn,
                         lat_video, lat_audio, sig_video, sig_audio, video_bf16, audio_bf16, stream=stream)

    def step(self, text, video, audio, mod, lat_video, lat_audio, sig_video, sig_audio, stream=None):
        """The whole hot path once: pack/project, one block, head + Euler."""
        self.embed(text, video, audio, stream)
        self.block(mod, stream=stream)
        self.head_euler(lat_video, lat_audio, sig_video, sig_audio, stream=stream)

    # kernels launched by one step (for the launch count the bench reports)
    def launches_per_step(self, e4m3: bool = False, qk_e4m3: bool = False) -> int:
        r = self.ranges
        embed = (1 if r.count[2] > 0 else 0) + 1 + (1 if r.L_pad > r.L else 0) + sum(1 for c in r.count if c > 0)
        # LN, QKV, attention (the split kernel + the general kernel's fixup
        # launch, bf16 or e4m3 q, k), [quantise o,] out-projection, LN, FFN
        # (2 GEMMs [+ quantise h])
        attn = 2
        block = 1 + 1 + attn + 1 + 1 + 2 + (2 if e4m3 else 0)
        # head + Euler: LN, video head GEMM, audio head GEMM (Euler in their epilogues)
        head = 1 + (1 if r.count[2] > 0 else 0) + (1 if r.count[1] > 0 else 0)
        return embed + block + head


class H3Sampler:
    """The 50-block, N-step flow sampler on one GPU ("MiniMax-H3: native joint
    audio-video generation" §6: separately shifted video / audio schedules,
    Euler update of the generation targets only; text is a fixed condition).

    Per denoise step: pack + project the bf16 latents, n_layers blocks
    (h3_block_forward, modulation [step][layer][3][6][D]), then the head with
    each modality's Euler step in its epilogue (h3_head_euler), which also
    writes the bf16 latents for the next step.  Orchestration only: every step runs in the library's kernels.

    e4m3=True runs the blocks with their four GEMMs on e4m3 operands
    (h3_block_forward_e4m3): each block's weights are quantised once on the
    GPU here and only the e4m3 copies are kept (the caller may drop its bf16
    block weights afterwards).  qk_e4m3=True (with e4m3) also takes attention's
    Q K^T on e4m3 codes (H3_QK_E4M3)."""

    def __init__(self, w: Workload, io_weights: dict, block_weights: list, device="cuda",
                 shift_video: float = 12.0, shift_audio: float = 3.0, e4m3: bool = False, qk_e4m3: bool = False):
        if qk_e4m3 and not e4m3:
            raise ValueError("qk_e4m3 needs e4m3")
        self.st = H3BlockStep(w, device=device, weights=io_weights)
        st = self.st
        self.e4m3 = e4m3
        self.flags = h3.H3_QK_NORM_ROPE_IN_QKV | (h3.H3_QK_E4M3 if qk_e4m3 else 0)
        if e4m3:
            st.alloc_e4m3()
            self.block_tensors = [st.quantize_block_weights_e4m3(Wb) for Wb in block_weights]
            torch.cuda.synchronize(st.device)
            self.blocks = [h3.block_weights_e4m3(Wb) for Wb in self.block_tensors]
            self.bufs = h3.block_buffers_e4m3({"xq": st.xq, "xs": st.xs, "q": st.q8 if qk_e4m3 else st.q,
                                               "k": st.k8 if qk_e4m3 else st.k, "v": st.v, "o": st.o, "oq": st.oq,
                                               "os": st.os, "ws": st.ws8})
        else:
            self.block_tensors = block_weights            # keep the tensors alive
            self.blocks = [h3.block_weights(Wb) for Wb in block_weights]
            self.bufs = h3.block_buffers(st.xm, st.q, st.k, st.v, st.o, st.ws)
        self.shifts = (shift_video, shift_audio)

    @property
    def n_layers(self) -> int:
        return len(self.blocks)

    def step(self, s, text, lat_video, lat_audio, video_bf16, audio_bf16, mod_all, sv, sa, stream=None):
        st = self.st
        st.embed(text, video_bf16, audio_bf16, stream)
        forward = h3.h3_block_forward_e4m3 if self.e4m3 else h3.h3_block_forward
        for b in range(self.n_layers):
            forward(st.dims, st.ranges, st.x, mod_all[s, b], st.pos, self.blocks[b], self.bufs, flags=self.flags,
                    stream=stream)
        st.head_euler(lat_video, lat_audio, (sv[s], sv[s + 1]), (sa[s], sa[s + 1]), video_bf16, audio_bf16, stream)

    def run(self, text, lat_video, lat_audio, video_bf16, audio_bf16, mod_all, n_steps: int, stream=None,
            start_step: int = 0, end_step: int | None = None):
        """lat_*: fp32 latents (at sigma = 1 when start_step is 0), updated in
        place; *_bf16: their bf16 copies (the next step's transformer input),
        kept in step.  Runs steps [start_step, end_step) of the n_steps
        schedule (all of them by default), so that a run can stop after a
        checkpoint and resume from it."""
        sv = h3.h3_sigma_schedule(n_steps, self.shifts[0])
        sa = h3.h3_sigma_schedule(n_steps, self.shifts[1])
        for s in range(start_step, n_steps if end_step is None else end_step):
            self.step(s, text, lat_video, lat_audio, video_bf16, audio_bf16, mod_all, sv, sa, stream)

    def modulation_cache(self, c_steps, adaln_weights: list, stream=None):
        """The modulation cache [n_steps][n_layers][3][6][D] fp32 that run()
        reads, from each step's conditioning vector (c_steps [n_steps][c_dim]
        fp32) and each block's AdaLN producer weight ([18 D][c_dim] bf16),
        one h3_adaln_modulation call per block writing its column of the
        cache."""
        st = self.st
        n_steps, c_dim = c_steps.shape
        if len(adaln_weights) != self.n_layers:
            raise ValueError("one AdaLN weight per block")
        mod_all = torch.empty(n_steps, self.n_layers, 3, 6, st.w.D, dtype=torch.float32, device=st.device)
        ws = torch.empty(h3.h3_adaln_workspace_bytes(n_steps, c_dim) // 2, dtype=torch.bfloat16, device=st.device)
        for b, Wb in enumerate(adaln_weights):
            h3.h3_adaln_modulation(st.dims, c_steps, Wb, ws, mod_all[:, b], stream=stream)
        return mod_all

    # ---------------------------------------------------------- checkpoint / resume
    @staticmethod
    def save_state(path: str, next_step: int, lat_video, lat_audio):
        """The sampler's whole state: the fp32 latents and the index of the
        next denoise step (an .npz file).  Weights and modulation are inputs,
        not state."""
        np.savez(path, next_step=np.int64(next_step), lat_video=lat_video.detach().cpu().numpy(),
                 lat_audio=lat_audio.detach().cpu().numpy())

    @staticmethod
    def load_state(path: str, device):
        """(next_step, lat_video, lat_audio, video_bf16, audio_bf16) on
        `device`; the bf16 copies are the latents rounded to nearest, which is
        what the Euler step writes for the next step."""
        z = np.load(path)
        lv = torch.from_numpy(z["lat_video"]).to(device)
        la = torch.from_numpy(z["lat_audio"]).to(device)
        return int(z["next_step"]), lv, la, lv.to(torch.bfloat16), la.to(torch.bfloat16)

    def launches_per_step(self) -> int:
        st = self.st
        per_block = (9 if self.e4m3 else 7) + 1  # attention: split kernel + fixup launch
        return st.launches_per_step() - 8 + per_block * self.n_layers
