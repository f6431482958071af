"""The text refiner (a reading: the trunk block's form over the text range
alone, in place on the packed sequence) against the oracle: two refiner
blocks on the packed text rows; the audio and video rows must not change."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import H3BlockStep, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("w", [S.WORKLOADS["tiny"], RAGGED], ids=lambda w: w.name)
def test_text_refine_against_oracle(w):
    inp = S.make_inputs(w)
    stk = S.make_stack_inputs(w, 2, 1, seed=4242 + w.index)
    st = H3BlockStep(w, weights=inp)
    dev = st.device
    st.embed(*(to_dev_bf16(inp[k], dev) for k in ("text", "video", "audio")))
    x0 = st.x.clone()
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in stk["blocks"]]
    mods = [torch.from_numpy(np.ascontiguousarray(stk["mod_all"][0][b])).to(dev) for b in range(2)]
    bufs = h3.block_buffers(st.xm, st.q, st.k, st.v, st.o, st.ws)
    h3.h3_text_refine(st.dims, st.ranges, st.x, mods, st.pos, [h3.block_weights(b) for b in blocks], bufs)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    nt = w.n_text
    assert torch.equal(st.x[nt:], x0[nt:]), "audio / video rows changed"
    r, pos = oracle_ranges_and_pos(w)
    xo = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    t_ranges = O.pack_ranges(nt, 0, 0)
    xt = xo[:nt]
    for b in range(2):
        Wb = stk["blocks"][b]
        xt = O.block_forward(xt, stk["mod_all"][0][b], t_ranges, pos[:nt], Wb["Wqkv"], Wb["qn_w"], Wb["kn_w"],
                             Wb["Wo"], Wb["Wgu"], Wb["Wd"], w.H)
    g = to_np(st.x)[:nt]
    check_close(g, xt, "refined text")
    # two blocks: twice the single block's delta bound (see the step test)
    check_close(g - xo[:nt], xt - xo[:nt], "refiner delta", max_rel_rms=1e-1)


def test_text_refine_noops_and_errors():
    w = RAGGED
    st = H3BlockStep(w)
    x = torch.zeros_like(st.x)
    bufs = h3.block_buffers(st.xm, st.q, st.k, st.v, st.o, st.ws)
    h3.h3_text_refine(st.dims, st.ranges, x, [], st.pos, [], bufs)          # no blocks: nothing to do
    no_text = h3.h3_make_ranges(0, 58, 240)
    Wd = {k: torch.zeros(1, dtype=torch.bfloat16, device=st.device) for k in ("Wqkv", "qn_w", "kn_w", "Wo", "Wgu", "Wd")}
    mod = torch.zeros(3, 6, w.D, device=st.device)
    h3.h3_text_refine(st.dims, no_text, x, [mod], st.pos, [h3.block_weights(Wd)], bufs)   # no text rows
    assert not x.any()
    with pytest.raises(ValueError):
        h3.h3_text_refine(st.dims, st.ranges, x, [mod, mod], st.pos, [h3.block_weights(Wd)], bufs)
