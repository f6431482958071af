"""h3_ffn_swiglu_noalloc: the FFN entry point for callers that cannot obtain
device memory for a workspace (an operator interface that passes only
tensors, a process whose device memory an outside allocator owns, a serving
loop that must not allocate).  It keeps its workspace in a fixed device array
inside the library; this test checks, through the C ABI, that it gives the
same result as h3_ffn_swiglu with a caller workspace, bit for bit (both run
the same two GEMM launches; only the workspace address differs), on calls in
a row: a full-width call whose workspace nearly fills the array, then two
smaller ones that see the earlier calls' leftovers in it; and that an
oversized call is refused before any launch.

Collected last (file name) so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import to_dev_bf16

from parity_util import RAGGED, check_close, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _inputs(w, seed, dev):
    rng = np.random.default_rng(seed)
    d = h3.make_dims(w.D, w.H, w.F)
    r = h3.h3_make_ranges(w.n_text, w.audio_channels * w.n_audio, w.T_lat * (w.H_lat // 2) * (w.W_lat // 2))
    Lp, L = r.L_pad, r.L
    x = np.zeros((Lp, w.D), np.float32)
    x[:L] = rng.standard_normal((L, w.D)).astype(np.float32)
    xm = np.zeros((Lp, w.D), np.float32)
    xm[:L] = S.bf16_round(rng.standard_normal((L, w.D)).astype(np.float32))
    Wgu = S.bf16_round((rng.standard_normal((2 * w.F, w.D)) * 0.02).astype(np.float32))
    Wd = S.bf16_round((rng.standard_normal((w.D, w.F)) * 0.02).astype(np.float32))
    mod = (rng.standard_normal((3, 6, w.D)) * 0.1).astype(np.float32)
    t = lambda a: torch.from_numpy(a).to(dev)
    return d, r, t(x), to_dev_bf16(xm, dev), to_dev_bf16(Wgu, dev), to_dev_bf16(Wd, dev), t(mod)


def _full_width_inputs(L, dev):
    """Full-width FFN operands (D 5376, F 14336) drawn on the device: this
    case only compares the two entry points with each other."""
    g = torch.Generator(device=dev)
    g.manual_seed(303)
    D, F = 5376, 14336
    d = h3.make_dims(D, 56, F)
    r = h3.h3_make_ranges(L, 0, 0)
    rnd = lambda *s, std=1.0: torch.randn(*s, generator=g, device=dev) * std
    x = torch.zeros(r.L_pad, D, device=dev)
    x[:L] = rnd(L, D)
    xm = torch.zeros(r.L_pad, D, dtype=torch.bfloat16, device=dev)
    xm[:L] = rnd(L, D).to(torch.bfloat16)
    return (d, r, x, xm, rnd(2 * F, D, std=0.02).to(torch.bfloat16), rnd(D, F, std=0.02).to(torch.bfloat16),
            rnd(3, 6, D, std=0.1))


def _both(d, r, x, xm, Wgu, Wd, mod, dev):
    ws = torch.empty(h3.h3_ffn_workspace_bytes(d, r.L_pad) // 2, dtype=torch.bfloat16, device=dev)
    x_ref = x.clone()
    h3.h3_ffn_swiglu(d, r, x_ref, xm, Wgu, Wd, mod, ws)
    x_new = x.clone()
    h3.h3_ffn_swiglu_noalloc(d, r, x_new, xm, Wgu, Wd, mod)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    return x_ref, x_new


def test_ffn_noalloc_matches_workspace_entry_point_on_calls_in_a_row():
    dev = torch.device("cuda", 0)
    # 1,100 tokens at full width: L_pad * F * 2 = 1152 * 14336 * 2 bytes, 98% of the array
    args = _full_width_inputs(1100, dev)
    assert args[1].L_pad * 14336 * 2 > 0.95 * h3.H3_FFN_STATIC_WS_BYTES
    x_ref, x_new = _both(*args, dev)
    assert torch.equal(x_new, x_ref), "full-width call"
    w = RAGGED                       # L_pad * F * 2 = 384 * 1280 * 2 bytes, well inside the array
    for call, seed in enumerate((101, 202)):
        d, r, x, xm, Wgu, Wd, mod = _inputs(w, seed, dev)
        x_ref, x_new = _both(d, r, x, xm, Wgu, Wd, mod, dev)
        assert torch.equal(x_new, x_ref), f"call {call}: output differs from h3_ffn_swiglu"
        x0 = to_np(x)
        check_close(to_np(x_new) - x0, to_np(x_ref) - x0, f"call {call}: FFN delta")


def test_ffn_noalloc_rejects_sizes_beyond_its_array():
    lib = h3.lib()
    d = h3.make_dims(5376, 56, 14336)
    r = h3.h3_make_ranges(1200, 0, 0)           # L_pad 1280: 1280 * 14336 * 2 bytes > 32 MiB
    assert r.L_pad * d.F * 2 > h3.H3_FFN_STATIC_WS_BYTES
    z = ctypes.c_void_p(256)                     # never dereferenced: the call must fail first
    rc = lib.h3_ffn_swiglu_noalloc(ctypes.byref(d), ctypes.byref(r), z, z, z, z, z, None)
    assert rc == h3.H3_ERR_SHAPE
    assert b"static workspace" in lib.h3_last_error()
