"""Sequence-parallel host logic on the CPU: the shard layout that every rank
computes (C ABI, host only), and the peer-buffer exchange between two gloo
ranks (the same code that shares CUDA buffers between GPUs, here with CPU
tensors in shared memory)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from omni_modal_diffusion_b200 import h3
from omni_modal_diffusion_b200 import synthetic as S


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()


def _modality_of_rows(r):
    m = np.full(r.L_pad, -1)
    for i in range(3):
        m[r.start[i]: r.start[i] + r.count[i]] = i
    return m


@pytest.mark.parametrize("wname", ["768sq_2s", "768x1344_5s", "768x1792_15s"])
@pytest.mark.parametrize("n", [1, 2, 4, 7, 8])
def test_layout_tiles_the_sequence(wname, n):
    w = S.WORKLOADS[wname]
    d = h3.make_dims(w.D, w.H, w.F)
    n_video = w.T_lat * (w.H_lat // 2) * (w.W_lat // 2)
    g = h3.h3_make_ranges(w.n_text, w.audio_channels * w.n_audio, n_video)
    if w.H % n:
        with pytest.raises(h3.H3Error):
            h3.h3_sp_make_layout(d, g, n, 0)
        return
    gm = _modality_of_rows(g)
    seen = np.zeros(g.L, np.int64)
    for r in range(n):
        lay, s = h3.h3_sp_make_layout(d, g, n, r)
        assert lay.n_ranks == n and lay.rank == r and lay.heads == w.H // n and lay.L == g.L
        assert lay.L_shard % 128 == 0 and lay.L_total == n * lay.L_shard and lay.row0 == r * lay.L_shard
        assert lay.L_shard == -(-(-(-g.L // n)) // 128) * 128
        assert s.L_pad == lay.L_shard and 0 < s.L <= s.L_pad
        assert sum(s.count) == s.L
        sm = _modality_of_rows(s)
        rows = np.arange(lay.row0, lay.row0 + s.L)
        assert np.array_equal(sm[: s.L], gm[rows])       # same modality per row
        assert np.all(sm[s.L:] == -1)
        seen[rows] += 1
    assert np.all(seen == 1)                              # shards tile [0, L) exactly once


def test_layout_rejections():
    w = S.WORKLOADS["tiny"]
    d = h3.make_dims(w.D, w.H, w.F)
    g = h3.h3_make_ranges(16, 16, 32)                    # L = 64: one 128-row shard is all
    h3.h3_sp_make_layout(d, g, 1, 0)
    with pytest.raises(h3.H3Error):
        h3.h3_sp_make_layout(d, g, 2, 0)                 # the second shard would be empty
    with pytest.raises(h3.H3Error):
        h3.h3_sp_make_layout(d, g, 3, 0)                 # H = 4 does not split into 3
    with pytest.raises(h3.H3Error):
        h3.h3_sp_make_layout(d, g, 9, 0)                 # more than H3_SP_MAX_RANKS
    with pytest.raises(h3.H3Error):
        h3.h3_sp_make_layout(d, g, 1, 1)                 # rank out of range


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch
    import torch.distributed as dist
    import torch.multiprocessing as tmp
    from omni_modal_diffusion_b200 import h3 as H
    from omni_modal_diffusion_b200 import sp
    from omni_modal_diffusion_b200 import synthetic as SS
    tmp.set_sharing_strategy("file_system")
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = SS.WORKLOADS["768sq_2s"]
        d = H.make_dims(w.D, w.H, w.F)
        n_video = w.T_lat * (w.H_lat // 2) * (w.W_lat // 2)
        g = H.h3_make_ranges(w.n_text, w.audio_channels * w.n_audio, n_video)
        lay, shard = H.h3_sp_make_layout(d, g, world, rank)
        layouts = [None] * world
        dist.all_gather_object(layouts, (lay.L_shard, lay.L_total, lay.row0, shard.L))
        # exchange buffers: q holds one row per global row block of this rank's
        # heads; o one row per head group of this rank's rows
        qb = torch.full((world, 4), -1.0).share_memory_()
        ob = torch.full((world, 4), -1.0).share_memory_()
        peers = sp.exchange_peer_tensors({"q": qb, "o": ob})
        dist.barrier()
        # like the fused epilogues: write my shard's block into every rank's q
        # (at my row block) and my heads' block into every rank's o (at my head
        # group), tagging each write with (writer, target)
        for tgt in range(world):
            peers["q"][tgt][rank] = torch.tensor([rank, tgt, 0, 1.0])
            peers["o"][tgt][rank] = torch.tensor([rank, tgt, 1, 1.0])
        dist.barrier()
        q.put((rank, layouts, peers["q"][rank].tolist(), peers["o"][rank].tolist(), qb.tolist(), ob.tolist()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_peer_exchange_gloo():
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([qq.get(timeout=90) for _ in range(world)])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, layouts, q_self, o_self, q_local, o_local in out:
        # every rank sees the same layout of every rank
        assert layouts == out[0][1]
        assert [l[2] for l in layouts] == [r * layouts[0][0] for r in range(world)]
        # its own buffers, seen through the peer table and directly, hold one
        # write from every rank, each at the writer's slot
        assert q_self == q_local and o_self == o_local
        for writer in range(world):
            assert q_local[writer] == [writer, rank, 0, 1.0]
            assert o_local[writer] == [writer, rank, 1, 1.0]
