"""Failure detection without a GPU fault: a bounded device-side wait that
nothing satisfies gives up, records its code, and the host reads it as
H3_ERR_TIMEOUT; the context stays usable for the next call."""
import time

import numpy as np
import pytest
import torch

from omni_modal_diffusion_b200 import h3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


def test_bounded_wait_gives_up_and_reports_timeout():
    assert h3.h3_device_status() == 0
    t0 = time.time()
    h3.h3_selftest_wait_timeout(50_000_000)          # 50 ms limit
    code = h3.h3_device_status()                      # synchronises, reads and clears
    assert code == 1
    assert time.time() - t0 < 5.0
    assert h3.h3_device_status() == 0                 # cleared
    # the context is still usable: a small Euler step runs and is right
    lat = torch.ones(1000, device="cuda")
    vel = torch.full((1000,), 2.0, device="cuda")
    h3.h3_euler_step(lat, vel, 0.75, 0.25)
    torch.cuda.synchronize()
    assert torch.allclose(lat, torch.zeros_like(lat))


def test_selftest_rejects_bad_limits():
    with pytest.raises(h3.H3Error):
        h3.h3_selftest_wait_timeout(0)
