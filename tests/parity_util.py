"""Shared helpers of the GPU parity tests (tolerances, workloads)."""
import dataclasses

import numpy as np
import torch

from omni_modal_diffusion_b200 import synthetic as S

# Block-level tolerance: max |gpu - oracle| <= 3e-2 * RMS(oracle) and
# mean relative error sum|gpu - oracle| / sum|oracle| <= 5e-3.
MAX_REL_RMS = 3e-2
MEAN_REL = 5e-3


def check_close(gpu, ref, name, max_rel_rms=MAX_REL_RMS, mean_rel=MEAN_REL):
    g = np.asarray(gpu, np.float64)
    o = np.asarray(ref, np.float64)
    assert g.shape == o.shape, (name, g.shape, o.shape)
    assert np.all(np.isfinite(g)), name
    err = np.abs(g - o)
    rms = float(np.sqrt(np.mean(o * o)))
    mx = float(err.max()) if err.size else 0.0
    mr = float(err.sum() / max(np.abs(o).sum(), 1e-300))
    assert mx <= max_rel_rms * rms, f"{name}: max|err| {mx:.3e} > {max_rel_rms} * RMS {rms:.3e} (mean rel {mr:.2e})"
    assert mr <= mean_rel, f"{name}: mean rel {mr:.3e} > {mean_rel} (max {mx:.3e}, rms {rms:.3e})"
    return mx / max(rms, 1e-300), mr


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


# A mid-size workload that spans several tiles with ragged tails everywhere:
# D = 576 (two 256-column tiles, the second 64 wide), text width 200 (a
# 64-deep K step with an 8-wide tail), L = 335 (L_pad 384: three 128-row
# tiles, the last one 79 rows), six heads, FFN 1280.
RAGGED = dataclasses.replace(S.WORKLOADS["tiny"], name="ragged", index=10, D=576, H=6, F=1280, D_text=200,
                             n_text=37, T_lat=5, H_lat=12, W_lat=16, n_audio=29)


def oracle_ranges_and_pos(w):
    from oracle import h3_oracle as O
    t, i, j = O.token_grid(w.T_lat, w.H_lat, w.W_lat)
    r = O.pack_ranges(w.n_text, w.audio_channels * w.n_audio, t * i * j)
    pos = O.positions(r, t, i, j, w.audio_channels, w.n_audio)
    return r, pos
