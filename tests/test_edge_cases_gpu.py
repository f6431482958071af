"""Degenerate packed sequences through the whole step (pack, projections,
block, head, Euler) against the oracle: one token, and workloads where one or
two modalities are empty."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200.pipeline import H3BlockStep, to_dev_bf16

from parity_util import check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu

TINY = S.WORKLOADS["tiny"]
CASES = {
    "video_only_L1": dataclasses.replace(TINY, name="video_only_L1", n_text=0, n_audio=0, T_lat=1, H_lat=2, W_lat=2),
    "text_only": dataclasses.replace(TINY, name="text_only", n_text=5, n_audio=0, T_lat=0),
    "audio_only": dataclasses.replace(TINY, name="audio_only", n_text=0, n_audio=3, T_lat=0),
    "no_audio": dataclasses.replace(TINY, name="no_audio", n_audio=0, T_lat=3, H_lat=4, W_lat=6),
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("name", list(CASES))
def test_degenerate_sequences_end_to_end(name):
    w = CASES[name]
    inp = S.make_inputs(w, seed=4242)
    st = H3BlockStep(w, weights=inp)
    dev = st.device
    text = to_dev_bf16(inp["text"], dev) if w.n_text else None
    video = to_dev_bf16(inp["video"], dev) if w.T_lat else None
    audio = to_dev_bf16(inp["audio"], dev) if w.n_audio else None
    mod = torch.from_numpy(inp["mod"]).to(dev)
    r, pos = oracle_ranges_and_pos(w)
    L = r["L"]
    assert st.ranges.as_dict() == r
    rng = np.random.default_rng(7)
    lat_v = rng.standard_normal(st.v_video.shape).astype(np.float32)
    lat_a = rng.standard_normal(st.v_audio.shape).astype(np.float32)
    gv, ga = torch.from_numpy(lat_v).to(dev), torch.from_numpy(lat_a).to(dev)
    st.embed(text, video, audio)
    st.block(mod)
    x2 = to_np(st.x)
    st.head()
    st.euler(gv, ga, (1.0, 0.5), (1.0, 0.5))
    torch.cuda.synchronize()
    x0 = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r)
    ref = O.block_forward(x0, inp["mod"], r, pos, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"], inp["Wgu"],
                          inp["Wd"], w.H)
    check_close(x2[:L], ref, f"{name} block output")
    assert np.all(x2[L:] == 0)
    vv, va = O.head_unpack(ref, r, inp["W_vhead"], inp["W_ahead"], w.T_lat, w.H_lat, w.W_lat, w.audio_channels,
                           w.n_audio)
    if vv.size:
        check_close(to_np(st.v_video), vv, f"{name} video velocity")
        check_close(to_np(gv), O.euler_step(lat_v, vv, 1.0, 0.5), f"{name} video latent")
    if va.size:
        check_close(to_np(st.v_audio), va, f"{name} audio velocity")
        check_close(to_np(ga), O.euler_step(lat_a, va, 1.0, 0.5), f"{name} audio latent")
