"""GPU parity of the layered flow sampler (block stack x Euler steps) against
the float64 oracle's sampler loop, from the same seeded weights, modulation
and initial latents."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import H3Sampler, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("w,n_layers,n_steps", [(S.WORKLOADS["tiny"], 50, 8), (RAGGED, 4, 2)],
                         ids=["tiny_50x8", "ragged_4x2"])
def test_sampler_against_oracle(w, n_layers, n_steps):
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, n_layers, n_steps)
    dev = torch.device("cuda", 0)
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in st["blocks"]]
    smp = H3Sampler(w, inp, blocks, device=dev)
    text = to_dev_bf16(inp["text"], dev)
    lv = torch.from_numpy(st["lat_video"]).to(dev)
    la = torch.from_numpy(st["lat_audio"]).to(dev)
    lv_bf, la_bf = lv.to(torch.bfloat16), la.to(torch.bfloat16)
    mod_all = torch.from_numpy(st["mod_all"]).to(dev)
    smp.run(text, lv, la, lv_bf, la_bf, mod_all, n_steps)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    assert torch.equal(lv_bf, lv.to(torch.bfloat16)) and torch.equal(la_bf, la.to(torch.bfloat16))
    r, pos = oracle_ranges_and_pos(w)
    rv, ra = O.sample(inp["text"], st["lat_video"], st["lat_audio"], inp, st["blocks"], st["mod_all"], r, pos, w.H,
                      n_steps)
    gv, ga = to_np(lv), to_np(la)
    # the latents' total change over the sampler (the part the model decides)
    check_close(gv - st["lat_video"], rv - st["lat_video"], "video latent change")
    check_close(ga - st["lat_audio"], ra - st["lat_audio"], "audio latent change")
    check_close(gv, rv, "video latent")
    check_close(ga, ra, "audio latent")
