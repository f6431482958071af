"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/h3.h declares, its host-only helpers agree with the oracle, and
argument validation rejects bad calls before any CUDA call is made."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import build as B
from omni_modal_diffusion_b200 import h3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return h3.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "h3.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(h3_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 15
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(h3.EXPORTS)
    assert lib.h3_version() == 100


def test_make_ranges_matches_oracle_packing(lib):
    for counts in ((16, 16, 32), (256, 160, 7488), (512, 400, 31248), (512, 1200, 122304), (1, 0, 0), (0, 0, 129)):
        r = h3.h3_make_ranges(*counts).as_dict()
        o = O.pack_ranges(*counts)
        assert r == o


def test_sigma_schedule_matches_oracle(lib):
    for shift in (12.0, 3.0, 1.0):
        got = np.array(h3.h3_sigma_schedule(8, shift), dtype=np.float32)
        ref = O.sigma_schedule(8, shift).astype(np.float32)
        assert np.array_equal(got, ref), (got, ref)


def test_workspace_bytes(lib):
    d = h3.make_dims(5376, 56, 14336)
    assert h3.h3_ffn_workspace_bytes(d, 7936) == 7936 * 14336 * 2


def _call_ln(lib, dims, ranges, x=16, mod=16, xm=16, branch=0):
    return lib.h3_adaln_norm_modulate(ctypes.byref(dims), ctypes.byref(ranges), ctypes.c_void_p(x),
                                      ctypes.c_void_p(mod), branch, ctypes.c_void_p(xm), None)


def test_validation_rejects_bad_arguments_without_launch(lib):
    d = h3.make_dims(320, 4, 896)
    r = h3.h3_make_ranges(16, 16, 32)
    assert _call_ln(lib, d, r, x=0) == h3.H3_ERR_NULL
    assert b"x" in lib.h3_last_error()
    assert _call_ln(lib, d, r, xm=8) == h3.H3_ERR_ALIGN
    assert _call_ln(lib, d, r, branch=2) == h3.H3_ERR_SHAPE
    bad = h3.make_dims(320, 4, 896, head_dim=64)
    assert _call_ln(lib, bad, r) == h3.H3_ERR_UNSUPPORTED
    bad = h3.make_dims(330, 4, 896)
    assert _call_ln(lib, bad, r) == h3.H3_ERR_UNSUPPORTED
    bad = h3.make_dims(320, 4, 900)
    assert _call_ln(lib, bad, r) == h3.H3_ERR_UNSUPPORTED
    bad = h3.make_dims(320, 4, 896, rope=(32, 48, 40))
    assert _call_ln(lib, bad, r) == h3.H3_ERR_SHAPE
    rr = h3.h3_make_ranges(16, 16, 32)
    rr.L_pad = 100
    assert _call_ln(lib, d, rr) == h3.H3_ERR_SHAPE
    rr = h3.h3_make_ranges(16, 16, 32)
    rr.start[1] = 10                       # overlaps the text range
    assert _call_ln(lib, d, rr) == h3.H3_ERR_SHAPE
    rr = h3.h3_make_ranges(16, 16, 32)
    rr.count[2] = 31                       # ranges no longer cover L
    assert _call_ln(lib, d, rr) == h3.H3_ERR_SHAPE
    assert lib.h3_euler_step(None, None, -1, 0.0, 0.0, None) == h3.H3_ERR_SHAPE
    assert lib.h3_euler_step(None, None, 0, 0.0, 0.0, None) == h3.H3_OK
    assert lib.h3_euler_step(ctypes.c_void_p(16), None, 4, 0.0, 0.0, None) == h3.H3_ERR_NULL
    # without the norm+RoPE placement flag attention takes them in its
    # prologue and needs the norm weights and the positions; e4m3 q, k need
    # the flag (the QKV epilogue writes the codes after its norm and RoPE)
    z = ctypes.c_void_p(16)
    assert lib.h3_attention(ctypes.byref(d), ctypes.byref(r), z, z, z, None, None, None, 0, z, None) == \
        h3.H3_ERR_NULL
    assert lib.h3_attention(ctypes.byref(d), ctypes.byref(r), z, z, z, z, z, None, 0, z, None) == h3.H3_ERR_NULL
    assert b"pos" in lib.h3_last_error()
    assert lib.h3_attention(ctypes.byref(d), ctypes.byref(r), z, z, z, z, z, z, h3.H3_QK_E4M3, z, None) == \
        h3.H3_ERR_UNSUPPORTED
    # e4m3 q, k: attention needs the norm weights (their scales), unknown
    # flags are refused, and the bf16 QKV call cannot write e4m3 codes
    qk8 = h3.H3_QK_NORM_ROPE_IN_QKV | h3.H3_QK_E4M3
    assert lib.h3_attention(ctypes.byref(d), ctypes.byref(r), z, z, z, None, None, None, qk8, z, None) == \
        h3.H3_ERR_NULL
    assert lib.h3_attention(ctypes.byref(d), ctypes.byref(r), z, z, z, z, z, None, h3.H3_QK_NORM_ROPE_IN_QKV | 8, z,
                            None) == h3.H3_ERR_UNSUPPORTED
    assert lib.h3_qkv_qknorm_mrope(ctypes.byref(d), ctypes.byref(r), z, z, z, z, z, qk8, z, z, z, None) == \
        h3.H3_ERR_UNSUPPORTED
    assert lib.h3_qkv_qknorm_mrope_e4m3(ctypes.byref(d), ctypes.byref(r), z, z, z, z, z, z, z,
                                        h3.H3_QK_NORM_ROPE_IN_QKV | 8, z, z, z, None) == h3.H3_ERR_UNSUPPORTED
    # embed: video count must match the latent grid
    rc = lib.h3_embed_pack(ctypes.byref(d), ctypes.byref(r), z, 256, z, 2, 8, 6, 24, z, 2, 8, 64, z, z, z, z, z, z,
                           z, None)
    assert rc == h3.H3_ERR_SHAPE
    rc = lib.h3_embed_pack(ctypes.byref(d), ctypes.byref(r), z, 256, z, 2, 8, 8, 24, z, 2, 7, 64, z, z, z, z, z, z,
                           z, None)
    assert rc == h3.H3_ERR_SHAPE


def test_binding_refuses_cpu_tensors(lib):
    import torch
    d = h3.make_dims(320, 4, 896)
    r = h3.h3_make_ranges(16, 16, 32)
    x = torch.zeros(128, 320)
    with pytest.raises(TypeError):
        h3.h3_adaln_norm_modulate(d, r, x, torch.zeros(3, 6, 320), 0, torch.zeros(128, 320, dtype=torch.bfloat16))
