"""Thin ctypes binding of libh3.so (include/h3.h), same names as the C ABI.

Argument marshalling only: torch tensors supply device memory and the CUDA
stream; every step of the block runs in the library's kernels.  There is no
fallback: if the library is missing or a tensor is not a CUDA tensor of the
expected dtype, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libh3.so")

H3_OK, H3_ERR_NULL, H3_ERR_SHAPE, H3_ERR_ALIGN, H3_ERR_UNSUPPORTED, H3_ERR_CUDA, H3_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5, -6
H3_ERR_BOUND = -7
H3_TEXT, H3_AUDIO, H3_VIDEO = 0, 1, 2
H3_MSA, H3_MLP = 0, 1
H3_QK_NORM_ROPE_IN_QKV = 1
H3_QK_E4M3 = 2  # q, k as e4m3 codes between the e4m3 QKV call and attention

EXPORTS = (
    "h3_last_error", "h3_version", "h3_make_ranges", "h3_sigma_schedule", "h3_embed_pack",
    "h3_adaln_norm_modulate", "h3_qkv_qknorm_mrope", "h3_attention", "h3_gated_residual",
    "h3_ffn_workspace_bytes", "h3_ffn_swiglu", "h3_head_unpack", "h3_head_euler", "h3_euler_step",
    "h3_adaln_workspace_bytes", "h3_adaln_modulation",
    "h3_device_status",
    "h3_set_wait_limit_ns", "h3_ffn_swiglu_noalloc", "h3_block_forward",
    "h3_euler_step_bf16", "h3_selftest_wait_timeout",
    "h3_quantize_rows_e4m3", "h3_adaln_norm_modulate_e4m3", "h3_qkv_qknorm_mrope_e4m3", "h3_gated_residual_e4m3",
    "h3_ffn_e4m3_workspace_bytes", "h3_ffn_swiglu_e4m3", "h3_block_forward_e4m3",
    "h3_sp_make_layout", "h3_qkv_qknorm_mrope_sp", "h3_qkv_qknorm_mrope_sp_e4m3", "h3_attention_sp",
    "h3_text_refine",
)
H3_SP_MAX_RANKS = 8
H3_FFN_STATIC_WS_BYTES = 32 * 1024 * 1024


class H3Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"h3 status {code}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("H", ctypes.c_int), ("head_dim", ctypes.c_int), ("I", ctypes.c_int),
                ("F", ctypes.c_int), ("rope_t", ctypes.c_int), ("rope_h", ctypes.c_int), ("rope_w", ctypes.c_int),
                ("theta", ctypes.c_float), ("eps_ln", ctypes.c_float), ("eps_qk", ctypes.c_float)]


class Ranges(ctypes.Structure):
    _fields_ = [("start", ctypes.c_int * 3), ("count", ctypes.c_int * 3), ("L", ctypes.c_int), ("L_pad", ctypes.c_int)]

    def as_dict(self) -> dict:
        return {"start": list(self.start), "count": list(self.count), "L": self.L, "L_pad": self.L_pad}


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Wqkv", "qn_w", "kn_w", "Wo", "Wgu", "Wd")]


class BlockBuffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("xm", "q", "k", "v", "o", "ws")]


E4M3_WEIGHT_FIELDS = ("Wqkv", "Wqkv_s", "qn_w", "kn_w", "Wo", "Wo_s", "Wgu", "Wgu_s", "Wd", "Wd_s")
E4M3_BUFFER_FIELDS = ("xq", "xs", "q", "k", "v", "o", "oq", "os", "ws")


class SPLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_ranks", "rank", "L", "L_shard", "L_total", "row0", "heads")]


class SPPeers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p * 8) for n in ("q", "k", "v", "o")]


class BlockWeightsE4m3(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in E4M3_WEIGHT_FIELDS]


class BlockBuffersE4m3(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in E4M3_BUFFER_FIELDS]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libh3.so (raises if it is missing: there is no other code path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with python -m omni_modal_diffusion_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        pd, pr = ctypes.POINTER(Dims), ctypes.POINTER(Ranges)
        sig = {
            "h3_last_error": (ctypes.c_char_p, []),
            "h3_version": (ci, []),
            "h3_make_ranges": (ci, [ci, ci, ci, pr]),
            "h3_sigma_schedule": (ci, [ci, cf, ctypes.POINTER(ctypes.c_float)]),
            "h3_embed_pack": (ci, [pd, pr, vp, ci, vp, ci, ci, ci, ci, vp, ci, ci, ci, vp, vp, vp, vp, vp, vp, vp, vp]),
            "h3_adaln_norm_modulate": (ci, [pd, pr, vp, vp, ci, vp, vp]),
            "h3_qkv_qknorm_mrope": (ci, [pd, pr, vp, vp, vp, vp, vp, ci, vp, vp, vp, vp]),
            "h3_attention": (ci, [pd, pr, vp, vp, vp, vp, vp, vp, ci, vp, vp]),
            "h3_gated_residual": (ci, [pd, pr, vp, vp, vp, vp, ci, vp]),
            "h3_ffn_workspace_bytes": (ctypes.c_size_t, [pd, ci]),
            "h3_ffn_swiglu": (ci, [pd, pr, vp, vp, vp, vp, vp, vp, vp]),
            "h3_ffn_swiglu_noalloc": (ci, [pd, pr, vp, vp, vp, vp, vp, vp]),
            "h3_head_unpack": (ci, [pd, pr, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, vp, vp, vp, vp]),
            "h3_head_euler": (ci, [pd, pr, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, vp, vp, vp, cf, cf, cf, cf, vp, vp,
                                   vp]),
            "h3_adaln_workspace_bytes": (ctypes.c_size_t, [ci, ci]),
            "h3_adaln_modulation": (ci, [pd, vp, ci, ci, vp, vp, vp, ctypes.c_int64, vp]),
            "h3_euler_step": (ci, [vp, vp, ctypes.c_int64, cf, cf, vp]),
            "h3_euler_step_bf16": (ci, [vp, vp, ctypes.c_int64, cf, cf, vp, vp]),
            "h3_block_forward": (ci, [pd, pr, vp, vp, vp, ctypes.POINTER(BlockWeights), ctypes.POINTER(BlockBuffers),
                                      ci, vp]),
            "h3_device_status": (ci, [vp, ctypes.POINTER(ci)]),
            "h3_set_wait_limit_ns": (ci, [ctypes.c_uint64]),
            "h3_selftest_wait_timeout": (ci, [ctypes.c_uint64, vp]),
            "h3_quantize_rows_e4m3": (ci, [vp, ctypes.c_int64, ci, ci, vp, ctypes.c_int64, vp, vp]),
            "h3_adaln_norm_modulate_e4m3": (ci, [pd, pr, vp, vp, ci, vp, vp, vp]),
            "h3_qkv_qknorm_mrope_e4m3": (ci, [pd, pr, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp, vp]),
            "h3_gated_residual_e4m3": (ci, [pd, pr, vp, vp, vp, vp, vp, vp, ci, vp]),
            "h3_ffn_e4m3_workspace_bytes": (ctypes.c_size_t, [pd, ci]),
            "h3_ffn_swiglu_e4m3": (ci, [pd, pr, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
            "h3_block_forward_e4m3": (ci, [pd, pr, vp, vp, vp, ctypes.POINTER(BlockWeightsE4m3),
                                           ctypes.POINTER(BlockBuffersE4m3), ci, vp]),
            "h3_sp_make_layout": (ci, [pd, pr, ci, ci, ctypes.POINTER(SPLayout), pr]),
            "h3_qkv_qknorm_mrope_sp": (ci, [pd, pr, ctypes.POINTER(SPLayout), vp, vp, vp, vp, vp, ci,
                                            ctypes.POINTER(SPPeers), vp]),
            "h3_qkv_qknorm_mrope_sp_e4m3": (ci, [pd, pr, ctypes.POINTER(SPLayout), vp, vp, vp, vp, vp, vp, vp, ci,
                                                 ctypes.POINTER(SPPeers), vp]),
            "h3_attention_sp": (ci, [pd, ctypes.POINTER(SPLayout), ctypes.POINTER(SPPeers), vp, vp, ci, vp]),
            "h3_text_refine": (ci, [pd, pr, vp, ci, ctypes.POINTER(ctypes.c_void_p), vp,
                                    ctypes.POINTER(BlockWeights), ctypes.POINTER(BlockBuffers), ci, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != H3_OK:
        raise H3Error(rc, lib().h3_last_error().decode())


def _ptr(t, dtype=None, name="tensor"):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_dims(D, H, F, head_dim=128, rope=(32, 48, 48), theta=10000.0, eps_ln=1e-6, eps_qk=1e-6) -> Dims:
    return Dims(D, H, head_dim, H * head_dim, F, rope[0], rope[1], rope[2], theta, eps_ln, eps_qk)


def h3_make_ranges(n_text: int, n_audio_tokens: int, n_video_tokens: int) -> Ranges:
    r = Ranges()
    _check(lib().h3_make_ranges(n_text, n_audio_tokens, n_video_tokens, ctypes.byref(r)))
    return r


def h3_sigma_schedule(n_steps: int, shift: float) -> list[float]:
    out = (ctypes.c_float * (n_steps + 1))()
    _check(lib().h3_sigma_schedule(n_steps, shift, out))
    return list(out)


BF16, F32, U8 = torch.bfloat16, torch.float32, torch.uint8


def h3_embed_pack(dims, ranges, text, video, audio, W_text, W_vid, W_aud, patches, x_out, pos_out, mod_out, stream=None):
    T, Hl, Wl, C_lat = video.shape if video is not None else (0, 0, 0, 0)
    ch, n_a, C_a = audio.shape if audio is not None else (0, 0, 0)
    D_text = text.shape[1] if text is not None else 0
    _check(lib().h3_embed_pack(ctypes.byref(dims), ctypes.byref(ranges), _ptr(text, BF16, "text"), D_text,
                               _ptr(video, BF16, "video"), T, Hl, Wl, C_lat, _ptr(audio, BF16, "audio"), ch, n_a, C_a,
                               _ptr(W_text, BF16, "W_text"), _ptr(W_vid, BF16, "W_vid"), _ptr(W_aud, BF16, "W_aud"),
                               _ptr(patches, BF16, "patches"), _ptr(x_out, F32, "x_out"), _ptr(pos_out, F32, "pos_out"),
                               _ptr(mod_out, U8, "mod_out"), _stream(stream)))


def h3_adaln_norm_modulate(dims, ranges, x, mod, branch, xm, stream=None):
    _check(lib().h3_adaln_norm_modulate(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                                        _ptr(mod, F32, "mod"), branch, _ptr(xm, BF16, "xm"), _stream(stream)))


def h3_qkv_qknorm_mrope(dims, ranges, xm, Wqkv, qn_w, kn_w, pos, q, k, v, flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    _check(lib().h3_qkv_qknorm_mrope(ctypes.byref(dims), ctypes.byref(ranges), _ptr(xm, BF16, "xm"),
                                     _ptr(Wqkv, BF16, "Wqkv"), _ptr(qn_w, BF16, "qn_w"), _ptr(kn_w, BF16, "kn_w"),
                                     _ptr(pos, F32, "pos"), flags, _ptr(q, BF16, "q"), _ptr(k, BF16, "k"),
                                     _ptr(v, BF16, "v"), _stream(stream)))


def h3_attention(dims, ranges, q, k, v, o, qn_w=None, kn_w=None, pos=None, flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    qk = U8 if flags & H3_QK_E4M3 else BF16
    _check(lib().h3_attention(ctypes.byref(dims), ctypes.byref(ranges), _ptr(q, qk, "q"), _ptr(k, qk, "k"),
                              _ptr(v, BF16, "v"), _ptr(qn_w, BF16, "qn_w"), _ptr(kn_w, BF16, "kn_w"),
                              _ptr(pos, F32, "pos"), flags, _ptr(o, BF16, "o"), _stream(stream)))


def h3_gated_residual(dims, ranges, x, o, Wo, mod, branch=H3_MSA, stream=None):
    _check(lib().h3_gated_residual(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"), _ptr(o, BF16, "o"),
                                   _ptr(Wo, BF16, "Wo"), _ptr(mod, F32, "mod"), branch, _stream(stream)))


def h3_ffn_workspace_bytes(dims, L_pad: int) -> int:
    return int(lib().h3_ffn_workspace_bytes(ctypes.byref(dims), L_pad))


def h3_ffn_swiglu(dims, ranges, x, xm, Wgu, Wd, mod, ws, stream=None):
    _check(lib().h3_ffn_swiglu(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"), _ptr(xm, BF16, "xm"),
                               _ptr(Wgu, BF16, "Wgu"), _ptr(Wd, BF16, "Wd"), _ptr(mod, F32, "mod"),
                               _ptr(ws, BF16, "ws"), _stream(stream)))


def h3_ffn_swiglu_noalloc(dims, ranges, x, xm, Wgu, Wd, mod, stream=None):
    """h3_ffn_swiglu with the library's fixed device workspace (no ws argument)."""
    _check(lib().h3_ffn_swiglu_noalloc(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                                       _ptr(xm, BF16, "xm"), _ptr(Wgu, BF16, "Wgu"), _ptr(Wd, BF16, "Wd"),
                                       _ptr(mod, F32, "mod"), _stream(stream)))


def h3_head_unpack(dims, ranges, x, W_vhead, W_ahead, video_shape, audio_shape, hn, v_video, v_audio, stream=None):
    T, Hl, Wl, C_lat = video_shape
    ch, n_a, C_a = audio_shape
    _check(lib().h3_head_unpack(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                                _ptr(W_vhead, BF16, "W_vhead"), _ptr(W_ahead, BF16, "W_ahead"), T, Hl, Wl, C_lat, ch,
                                n_a, C_a, _ptr(hn, BF16, "hn"), _ptr(v_video, F32, "v_video"),
                                _ptr(v_audio, F32, "v_audio"), _stream(stream)))


def h3_head_euler(dims, ranges, x, W_vhead, W_ahead, video_shape, audio_shape, hn, lat_video, lat_audio,
                  sig_video, sig_audio, lat_video_bf16=None, lat_audio_bf16=None, stream=None):
    """sig_video, sig_audio: (sigma, sigma_next) of each modality's schedule."""
    T, Hl, Wl, C_lat = video_shape
    ch, n_a, C_a = audio_shape
    _check(lib().h3_head_euler(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                               _ptr(W_vhead, BF16, "W_vhead"), _ptr(W_ahead, BF16, "W_ahead"), T, Hl, Wl, C_lat, ch,
                               n_a, C_a, _ptr(hn, BF16, "hn"), _ptr(lat_video, F32, "lat_video"),
                               _ptr(lat_audio, F32, "lat_audio"), float(sig_video[0]), float(sig_video[1]),
                               float(sig_audio[0]), float(sig_audio[1]), _ptr(lat_video_bf16, BF16, "lat_video_bf16"),
                               _ptr(lat_audio_bf16, BF16, "lat_audio_bf16"), _stream(stream)))


def h3_adaln_workspace_bytes(n: int, c_dim: int) -> int:
    return int(lib().h3_adaln_workspace_bytes(n, c_dim))


def h3_adaln_modulation(dims, c, W, ws, mod, stream=None):
    """mod = W SiLU(c) for c [n][c_dim] fp32, W [18D][c_dim] bf16; ws: bf16
    scratch of n * c_dim elements.  mod: a contiguous [n][3][6][D] fp32
    tensor, or a view whose rows (first index) are apart by its stride, e.g.
    cache[:, b] of a [step][block][3][6][D] cache."""
    n, c_dim = c.shape
    if ws.numel() * ws.element_size() < h3_adaln_workspace_bytes(n, c_dim):
        raise ValueError("workspace too small")
    if not (isinstance(mod, torch.Tensor) and mod.is_cuda and mod.dtype == F32):
        raise TypeError("mod must be a float32 CUDA tensor")
    if mod.shape[0] != n or mod[0].numel() != 18 * dims.D or (n > 1 and not mod[0].is_contiguous()):
        raise ValueError("mod must be [n][3][6][D] with contiguous rows")
    ld = mod.stride(0) if n > 1 else 18 * dims.D
    _check(lib().h3_adaln_modulation(ctypes.byref(dims), _ptr(c, F32, "c"), n, c_dim, _ptr(W, BF16, "W"),
                                     _ptr(ws, BF16, "ws"), ctypes.c_void_p(mod.data_ptr()), ld, _stream(stream)))


def h3_euler_step(lat, vel, sigma: float, sigma_next: float, stream=None):
    if lat.numel() != vel.numel():
        raise ValueError("lat and vel sizes differ")
    _check(lib().h3_euler_step(_ptr(lat, F32, "lat"), _ptr(vel, F32, "vel"), lat.numel(), sigma, sigma_next,
                               _stream(stream)))


def block_weights(W: dict) -> BlockWeights:
    """Pointer struct of one block's weights (dict of bf16 CUDA tensors)."""
    return BlockWeights(*(_ptr(W[n], BF16, n) for n in ("Wqkv", "qn_w", "kn_w", "Wo", "Wgu", "Wd")))


def block_buffers(xm, q, k, v, o, ws) -> BlockBuffers:
    return BlockBuffers(*(_ptr(t, BF16, n) for n, t in zip(("xm", "q", "k", "v", "o", "ws"), (xm, q, k, v, o, ws))))


def h3_block_forward(dims, ranges, x, mod, pos, weights: BlockWeights, buffers: BlockBuffers,
                     flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    _check(lib().h3_block_forward(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"), _ptr(mod, F32, "mod"),
                                  _ptr(pos, F32, "pos"), ctypes.byref(weights), ctypes.byref(buffers), flags,
                                  _stream(stream)))


def h3_euler_step_bf16(lat, vel, sigma: float, sigma_next: float, lat_bf16, stream=None):
    if lat.numel() != vel.numel() or lat.numel() != lat_bf16.numel():
        raise ValueError("lat, vel and lat_bf16 sizes differ")
    _check(lib().h3_euler_step_bf16(_ptr(lat, F32, "lat"), _ptr(vel, F32, "vel"), lat.numel(), sigma, sigma_next,
                                    _ptr(lat_bf16, BF16, "lat_bf16"), _stream(stream)))


def h3_device_status(stream=None) -> int:
    code = ctypes.c_int(0)
    rc = lib().h3_device_status(_stream(stream), ctypes.byref(code))
    if rc not in (H3_OK, H3_ERR_TIMEOUT, H3_ERR_BOUND):
        _check(rc)
    return code.value


def h3_selftest_wait_timeout(limit_ns: int, stream=None):
    _check(lib().h3_selftest_wait_timeout(limit_ns, _stream(stream)))


def h3_set_wait_limit_ns(ns: int):
    _check(lib().h3_set_wait_limit_ns(ns))


# ------------------------------------------------------------ e4m3 (FP8) GEMMs
# Codes are uint8 tensors, scales float32 (one per row / output channel).

def h3_quantize_rows_e4m3(x, q, scale, stream=None):
    """Row-quantise a 2-D bf16 tensor into e4m3 codes q (uint8, same shape) and
    per-row scales (float32 [rows])."""
    if x.dim() != 2 or q.shape != x.shape or scale.numel() != x.shape[0]:
        raise ValueError("x [rows, cols], q [rows, cols] and scale [rows] required")
    _check(lib().h3_quantize_rows_e4m3(_ptr(x, BF16, "x"), x.shape[1], x.shape[0], x.shape[1], _ptr(q, U8, "q"),
                                       q.shape[1], _ptr(scale, F32, "scale"), _stream(stream)))


def h3_adaln_norm_modulate_e4m3(dims, ranges, x, mod, branch, xq, xs, stream=None):
    _check(lib().h3_adaln_norm_modulate_e4m3(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                                             _ptr(mod, F32, "mod"), branch, _ptr(xq, U8, "xq"), _ptr(xs, F32, "xs"),
                                             _stream(stream)))


def h3_qkv_qknorm_mrope_e4m3(dims, ranges, xq, xs, Wq, Ws, qn_w, kn_w, pos, q, k, v, flags=H3_QK_NORM_ROPE_IN_QKV,
                             stream=None):
    _check(lib().h3_qkv_qknorm_mrope_e4m3(ctypes.byref(dims), ctypes.byref(ranges), _ptr(xq, U8, "xq"),
                                          _ptr(xs, F32, "xs"), _ptr(Wq, U8, "Wq"), _ptr(Ws, F32, "Ws"),
                                          _ptr(qn_w, BF16, "qn_w"), _ptr(kn_w, BF16, "kn_w"), _ptr(pos, F32, "pos"),
                                          flags, _ptr(q, U8 if flags & H3_QK_E4M3 else BF16, "q"),
                                          _ptr(k, U8 if flags & H3_QK_E4M3 else BF16, "k"), _ptr(v, BF16, "v"),
                                          _stream(stream)))


def h3_gated_residual_e4m3(dims, ranges, x, oq, os_, Wq, Ws, mod, branch=H3_MSA, stream=None):
    _check(lib().h3_gated_residual_e4m3(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                                        _ptr(oq, U8, "oq"), _ptr(os_, F32, "os"), _ptr(Wq, U8, "Wq"),
                                        _ptr(Ws, F32, "Ws"), _ptr(mod, F32, "mod"), branch, _stream(stream)))


def h3_ffn_e4m3_workspace_bytes(dims, L_pad: int) -> int:
    return int(lib().h3_ffn_e4m3_workspace_bytes(ctypes.byref(dims), L_pad))


def h3_ffn_swiglu_e4m3(dims, ranges, x, xq, xs, Wgu_q, Wgu_s, Wd_q, Wd_s, mod, ws, stream=None):
    _check(lib().h3_ffn_swiglu_e4m3(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"), _ptr(xq, U8, "xq"),
                                    _ptr(xs, F32, "xs"), _ptr(Wgu_q, U8, "Wgu_q"), _ptr(Wgu_s, F32, "Wgu_s"),
                                    _ptr(Wd_q, U8, "Wd_q"), _ptr(Wd_s, F32, "Wd_s"), _ptr(mod, F32, "mod"),
                                    _ptr(ws, U8, "ws"), _stream(stream)))


def block_weights_e4m3(W: dict) -> BlockWeightsE4m3:
    """Pointer struct of one block's e4m3 weights: codes (uint8) and scales
    (float32) under the names of E4M3_WEIGHT_FIELDS; qn_w, kn_w bf16."""
    dt = {"qn_w": BF16, "kn_w": BF16}
    return BlockWeightsE4m3(*(_ptr(W[n], dt.get(n, F32 if n.endswith("_s") else U8), n) for n in E4M3_WEIGHT_FIELDS))


def block_buffers_e4m3(B: dict) -> BlockBuffersE4m3:
    """q and k may be bf16 or, for the H3_QK_E4M3 block, uint8 code buffers."""
    dt = {"xq": U8, "xs": F32, "q": (BF16, U8), "k": (BF16, U8), "v": BF16, "o": BF16, "oq": U8, "os": F32, "ws": U8}
    for n in ("q", "k"):
        if B[n].dtype not in dt[n]:
            raise TypeError(f"{n} must be bfloat16 or uint8, got {B[n].dtype}")
        dt[n] = B[n].dtype
    return BlockBuffersE4m3(*(_ptr(B[n], dt[n], n) for n in E4M3_BUFFER_FIELDS))


def h3_block_forward_e4m3(dims, ranges, x, mod, pos, weights: BlockWeightsE4m3, buffers: BlockBuffersE4m3,
                          flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    _check(lib().h3_block_forward_e4m3(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"),
                                       _ptr(mod, F32, "mod"), _ptr(pos, F32, "pos"), ctypes.byref(weights),
                                       ctypes.byref(buffers), flags, _stream(stream)))


# ------------------------------------------------------------ sequence parallelism (Ulysses)

def h3_sp_make_layout(dims, global_ranges, n_ranks: int, rank: int):
    """(SPLayout, shard Ranges) of rank `rank` of n_ranks (host only)."""
    lay, shard = SPLayout(), Ranges()
    _check(lib().h3_sp_make_layout(ctypes.byref(dims), ctypes.byref(global_ranges), n_ranks, rank,
                                   ctypes.byref(lay), ctypes.byref(shard)))
    return lay, shard


def sp_peers(q=None, k=None, v=None, o=None, qk_e4m3: bool = False) -> SPPeers:
    """Peer table from per-rank lists of CUDA tensors (index = rank); a list
    may be None when the call does not use it.  qk_e4m3: q and k are uint8
    tensors of e4m3 codes."""
    p = SPPeers()
    for name, ts in (("q", q), ("k", k), ("v", v), ("o", o)):
        if ts is None:
            continue
        if len(ts) > H3_SP_MAX_RANKS:
            raise ValueError(f"at most {H3_SP_MAX_RANKS} ranks")
        arr = getattr(p, name)
        dt = U8 if qk_e4m3 and name in ("q", "k") else BF16
        for i, t in enumerate(ts):
            arr[i] = _ptr(t, dt, f"{name}[{i}]").value
    return p


def h3_qkv_qknorm_mrope_sp(dims, shard, layout, xm, Wqkv, qn_w, kn_w, pos, peers: SPPeers,
                           flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    _check(lib().h3_qkv_qknorm_mrope_sp(ctypes.byref(dims), ctypes.byref(shard), ctypes.byref(layout),
                                        _ptr(xm, BF16, "xm"), _ptr(Wqkv, BF16, "Wqkv"), _ptr(qn_w, BF16, "qn_w"),
                                        _ptr(kn_w, BF16, "kn_w"), _ptr(pos, F32, "pos"), flags, ctypes.byref(peers),
                                        _stream(stream)))


def h3_qkv_qknorm_mrope_sp_e4m3(dims, shard, layout, xq, xs, Wq, Ws, qn_w, kn_w, pos, peers: SPPeers,
                                flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    _check(lib().h3_qkv_qknorm_mrope_sp_e4m3(ctypes.byref(dims), ctypes.byref(shard), ctypes.byref(layout),
                                             _ptr(xq, U8, "xq"), _ptr(xs, F32, "xs"), _ptr(Wq, U8, "Wq"),
                                             _ptr(Ws, F32, "Ws"), _ptr(qn_w, BF16, "qn_w"), _ptr(kn_w, BF16, "kn_w"),
                                             _ptr(pos, F32, "pos"), flags, ctypes.byref(peers), _stream(stream)))


def h3_attention_sp(dims, layout, peers: SPPeers, qn_w=None, kn_w=None, flags=H3_QK_NORM_ROPE_IN_QKV,
                    stream=None):
    _check(lib().h3_attention_sp(ctypes.byref(dims), ctypes.byref(layout), ctypes.byref(peers),
                                 _ptr(qn_w, BF16, "qn_w"), _ptr(kn_w, BF16, "kn_w"), flags, _stream(stream)))


def h3_text_refine(dims, ranges, x, mods: list, pos, weights: list, buffers: BlockBuffers,
                   flags=H3_QK_NORM_ROPE_IN_QKV, stream=None):
    """The text refiner blocks over the packed text rows of x, in place
    (mods: per-block [3][6][D] float32 CUDA tensors; weights: per-block
    BlockWeights)."""
    n = len(weights)
    if len(mods) != n:
        raise ValueError("one modulation per refiner block")
    mod_ptrs = (ctypes.c_void_p * max(n, 1))(*[_ptr(m, F32, "mod").value for m in mods])
    w_arr = (BlockWeights * max(n, 1))(*weights)
    _check(lib().h3_text_refine(ctypes.byref(dims), ctypes.byref(ranges), _ptr(x, F32, "x"), n, mod_ptrs,
                                _ptr(pos, F32, "pos"), w_arr, ctypes.byref(buffers), flags, _stream(stream)))
