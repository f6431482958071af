"""Sequence parallelism across processes: two ranks, each its own process,
both on GPU 0 (CUDA IPC handles work between processes on one device), the
exchange buffers opened through IPC, the phases ordered by the host barrier
of sp_runner.  The ranks' kernels never wait on one another: every wait is
on the host, so the two contexts sharing the GPU only time-slice.

The sharded block, gathered from the two processes, must equal the
single-sequence block bit for bit and the oracle within the block tolerance.
Every exchange buffer starts as NaN, so a row the exchange misses fails."""
import os
import socket

import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S

from parity_util import RAGGED, check_close, oracle_ranges_and_pos

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, n_blocks, e4m3=False):
    import datetime

    import torch.distributed as dist

    from omni_modal_diffusion_b200 import h3
    from omni_modal_diffusion_b200.pipeline import H3BlockStep, to_dev_bf16
    from omni_modal_diffusion_b200.sp_runner import SPProcessRank

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w = RAGGED
    inp = S.make_inputs(w)
    st = H3BlockStep(w, device=dev, weights=inp)
    st.embed(*(to_dev_bf16(inp[k], dev) for k in ("text", "video", "audio")))
    mod = torch.from_numpy(inp["mod"]).to(dev)
    W8 = st.quantize_block_weights_e4m3() if e4m3 else None
    if e4m3:
        st.alloc_e4m3()
    me = SPProcessRank(w, st.dims, st.ranges, dev, e4m3=e4m3, qk_e4m3=e4m3)
    r = me.rank
    r.x.zero_()
    r.pos.zero_()
    lo, hi = r.rows.start, min(r.rows.stop, st.ranges.L_pad)
    r.x[: hi - lo].copy_(st.x[lo:hi])
    r.pos[: hi - lo].copy_(st.pos[lo:hi])
    for t in (r.q, r.k, r.v, r.o):
        t.fill_(float("nan"))
    if e4m3:
        r.q8.fill_(0x7F)              # e4m3 NaN codes: a row the exchange misses shows
        r.k8.fill_(0x7F)
    me.barrier()                      # every rank's buffers initialised before any peer store
    for _ in range(n_blocks):
        if e4m3:
            me.block_forward_e4m3(mod, W8)
        else:
            me.block_forward(mod, st.W)
    torch.cuda.synchronize()
    status = h3.h3_device_status()
    np.save(os.path.join(out_dir, f"x_rank{rank}.npy"), r.x.cpu().numpy())
    if rank == 0:
        for _ in range(n_blocks):
            if e4m3:
                st.block_e4m3(mod, W8, qk_e4m3=True)
            else:
                st.block(mod)
        torch.cuda.synchronize()
        np.save(os.path.join(out_dir, "x_single.npy"), st.x.cpu().numpy())
    me.close()
    dist.destroy_process_group()
    if status != 0:
        raise RuntimeError(f"rank {rank}: device-side wait gave up (code {status})")


@pytest.mark.timeout(600)
@pytest.mark.parametrize("n_blocks", [1, 2])
def test_sp_two_processes_one_gpu(tmp_path, n_blocks):
    import torch.multiprocessing as mp

    from omni_modal_diffusion_b200 import build
    build.build()
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), n_blocks), nprocs=world, join=True)
    w = RAGGED
    r_o, pos_o = oracle_ranges_and_pos(w)
    L = r_o["L"]
    shards = [np.load(tmp_path / f"x_rank{g}.npy") for g in range(world)]
    x_sp = np.concatenate(shards, 0)[:L]
    x_single = np.load(tmp_path / "x_single.npy")[:L]
    assert np.array_equal(x_sp, x_single), "two-process sharded block differs from the single-sequence block"
    inp = S.make_inputs(w)
    x = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r_o)
    for _ in range(n_blocks):
        x = O.block_forward(x, inp["mod"], r_o, pos_o, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"], inp["Wgu"],
                            inp["Wd"], w.H)
    check_close(x_sp, x, f"two-process sequence-parallel block output ({n_blocks} block(s))")


@pytest.mark.timeout(600)
def test_sp_two_processes_one_gpu_e4m3(tmp_path):
    """The same with e4m3 GEMMs and e4m3 q, k codes over the exchange: the
    two processes' shards equal the single-sequence e4m3 block bit for bit."""
    import torch.multiprocessing as mp

    from omni_modal_diffusion_b200 import build
    build.build()
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), 1, True), nprocs=world, join=True)
    L = oracle_ranges_and_pos(RAGGED)[0]["L"]
    shards = [np.load(tmp_path / f"x_rank{g}.npy") for g in range(world)]
    x_sp = np.concatenate(shards, 0)[:L]
    x_single = np.load(tmp_path / "x_single.npy")[:L]
    assert np.array_equal(x_sp, x_single), "two-process sharded e4m3 block differs from the single-sequence one"
