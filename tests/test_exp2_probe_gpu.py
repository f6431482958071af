"""The attention softmax's FMA-pipe exponential (exp2_fma2) against 2^x.

The softmax takes a fixed share of its exponentials on the FMA pipe with a
cubic of its own fit; the attention parity tests cover it only through the
whole kernel, so this test holds the function itself to its stated bound:
relative error <= 1e-4 of the exact 2^(k s + c) (7.5e-5 from the cubic, the
rest from rounding the argument through u = sat(s k/252 + (125 + c)/252)),
over the range the softmax feeds it, and the clamp at 2^-125 / 2^127.  It runs
through a test-only probe library (tests/cuda), not through libh3.so.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def probe():
    from omni_modal_diffusion_b200 import build
    lib = ctypes.CDLL(build.build_probe())
    lib.exp2_fma2_probe.restype = ctypes.c_int
    lib.exp2_fma2_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_float,
                                    ctypes.c_float, ctypes.c_void_p]
    return lib


def _run(lib, s, k, c):
    x = torch.from_numpy(np.ascontiguousarray(s, np.float32)).cuda()
    y = torch.empty_like(x)
    rc = lib.exp2_fma2_probe(x.data_ptr(), y.data_ptr(), x.numel(), k, c,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("k,c", [(1.0, 0.0), (0.12752, -3.5), (0.12752, -40.0), (2.0, 17.0)])
def test_exp2_fma2_error_bound(probe, k, c):
    # arguments x = k s + c covering [-124.5, 126.5], odd length (ragged pair)
    x = np.concatenate([np.linspace(-124.5, 126.5, 1_000_001), np.arange(-124, 126) + 0.5,
                        np.arange(-124, 127, dtype=np.float64)])
    s = ((x - c) / k).astype(np.float32)
    got = _run(probe, s, k, c)
    ref = np.exp2(np.float64(k) * s.astype(np.float64) + np.float64(c))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 1e-4, rel.max()


def test_exp2_fma2_clamps(probe):
    # below the range: 2^-125 (times the cubic at 0); above: 2^127 (finite,
    # so an overflow check on the row sum still sees a huge value)
    got = _run(probe, np.array([-1e30, -200.0, -126.0, 128.0, 1e30], np.float32), 1.0, 0.0)
    assert np.allclose(got[:3], 2.0 ** -125, rtol=1e-4)
    assert np.allclose(got[3:], 2.0 ** 127, rtol=1e-4)
    assert np.all(np.isfinite(got))
