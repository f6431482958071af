"""GPU parity of the AdaLN modulation producer (h3_adaln_modulation, the
NEXT-3 reading G22: SiLU of a conditioning vector, then one linear per block
to the 18 D modulation features) against the float64 oracle, at the tiny
width and at full width (D = 5376, conditioning width D/2 = 2688, one vector
per sampler step), and the sampler's modulation cache built from it."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200.pipeline import H3Sampler, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _case(D, c_dim, n, seed):
    rng = np.random.default_rng(seed)
    c = (rng.standard_normal((n, c_dim)) * 2).astype(np.float32)
    W = S.bf16_round((rng.standard_normal((18 * D, c_dim)) * 0.02).astype(np.float32))
    return c, W


@pytest.mark.parametrize("D,c_dim,n", [(320, 160, 1), (320, 168, 3), (576, 288, 8), (5376, 2688, 8)],
                         ids=["tiny_n1", "tiny_ragged_k", "ragged_n8", "full_n8"])
def test_adaln_modulation_against_oracle(D, c_dim, n):
    c, W = _case(D, c_dim, n, seed=D + c_dim + n)
    d = h3.make_dims(D, 4, 896)
    ws = torch.empty(h3.h3_adaln_workspace_bytes(n, c_dim) // 2, dtype=torch.bfloat16, device=DEV)
    mod = torch.full((n, 3, 6, D), float("nan"), device=DEV)
    h3.h3_adaln_modulation(d, torch.from_numpy(c).to(DEV), to_dev_bf16(W, DEV), ws, mod)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    ref = O.adaln_modulation(c, W, D)
    # SiLU(c) enters the GEMM rounded to bf16 (like every activation operand)
    check_close(to_np(mod), ref, f"AdaLN modulation D={D} n={n}")


def test_adaln_strided_cache_and_errors():
    """Rows written ld_mod apart (a block's column of a [step][block] cache),
    the other blocks' columns untouched; bad arguments refused before launch."""
    D, c_dim, n, blocks = 320, 160, 4, 3
    c, W = _case(D, c_dim, n, seed=7)
    d = h3.make_dims(D, 4, 896)
    ws = torch.empty(h3.h3_adaln_workspace_bytes(n, c_dim) // 2, dtype=torch.bfloat16, device=DEV)
    cache = torch.zeros(n, blocks, 3, 6, D, device=DEV)
    h3.h3_adaln_modulation(d, torch.from_numpy(c).to(DEV), to_dev_bf16(W, DEV), ws, cache[:, 1])
    torch.cuda.synchronize()
    check_close(to_np(cache[:, 1]), O.adaln_modulation(c, W, D), "cache column 1")
    assert torch.all(cache[:, 0] == 0) and torch.all(cache[:, 2] == 0)
    with pytest.raises(h3.H3Error):
        h3.h3_adaln_modulation(d, torch.zeros(n, 12, device=DEV), to_dev_bf16(np.zeros((18 * D, 12), np.float32), DEV),
                               torch.empty(n * 12, dtype=torch.bfloat16, device=DEV), torch.empty(n, 3, 6, D, device=DEV))


def test_sampler_from_conditioning_matches_oracle():
    """The sampler run on a modulation cache built by the producer equals the
    oracle's sampler on the oracle's producer output (tiny widths, 3 blocks, 2
    steps)."""
    w, n_layers, n_steps = RAGGED, 3, 2
    inp = S.make_inputs(w)
    st = S.make_stack_inputs(w, n_layers, n_steps)
    rng = np.random.default_rng(31)
    c_dim = w.D // 2
    c = rng.standard_normal((n_steps, c_dim)).astype(np.float32)
    Wa = [S.bf16_round((rng.standard_normal((18 * w.D, c_dim)) * 0.02).astype(np.float32)) for _ in range(n_layers)]
    dev = torch.device("cuda", 0)
    blocks = [{k: to_dev_bf16(v, dev) for k, v in b.items()} for b in st["blocks"]]
    smp = H3Sampler(w, inp, blocks, device=dev)
    mod_all = smp.modulation_cache(torch.from_numpy(c).to(dev), [to_dev_bf16(x, dev) for x in Wa])
    lv = torch.from_numpy(st["lat_video"]).to(dev)
    la = torch.from_numpy(st["lat_audio"]).to(dev)
    smp.run(to_dev_bf16(inp["text"], dev), lv, la, lv.to(torch.bfloat16), la.to(torch.bfloat16), mod_all, n_steps)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    ref_mod = np.stack([np.stack([O.adaln_modulation(c[s:s + 1], Wa[b], w.D)[0] for b in range(n_layers)])
                        for s in range(n_steps)])
    check_close(to_np(mod_all), ref_mod, "modulation cache")
    r, pos = oracle_ranges_and_pos(w)
    rv, ra = O.sample(inp["text"], st["lat_video"], st["lat_audio"], inp, st["blocks"], ref_mod, r, pos, w.H, n_steps)
    check_close(to_np(lv) - st["lat_video"], rv - st["lat_video"], "video latent change")
    check_close(to_np(la) - st["lat_audio"], ra - st["lat_audio"], "audio latent change")
