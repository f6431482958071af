"""Sequence parallelism across processes: one process per rank, its exchange
buffers opened by every other rank, the block's phases ordered by a barrier.

"MiniMax-H3 paper reading" (gojay.top) §7.2 serves the trunk with Ulysses
degree 4.  `sp.SPRank` holds one rank's shard and exchange buffers and issues
its calls; this module adds what a multi-process run needs:

* the peer table: every rank shares its q/k/v/o receive buffers with the
  others as CUDA IPC handles (`sp.exchange_peer_tensors`), so the fused
  exchange epilogues of `h3_qkv_qknorm_mrope_sp` and `h3_attention_sp` store
  straight into the owning rank's memory (plain stores, NVLink P2P between
  GPUs; no TMA or bulk load ever reads a peer's memory);
* the barrier between phases (`ProcessBarrier`): the calling rank's stream
  is synchronised, which returns only once every kernel of the phase has
  completed, stores into peer memory included, and then the ranks meet on
  the host (`dist.barrier`).  No rank launches a kernel of the next phase
  before every rank's kernels of the previous one have completed, and a
  kernel that has completed has made its global-memory stores visible to
  kernels launched after it on any device that maps that memory.  Two such
  barriers per block (after the QKV phase, after attention) order every
  write into a peer buffer after the peer's last read of the previous block
  (a rank's next QKV stores follow the attention barrier that every rank
  passed only after its attention reads; the next attention stores into o
  follow a barrier that every rank passes only after its out-projection
  read o);
* teardown: a barrier, then the opened peer handles are dropped, then a
  barrier before any rank frees the buffers it shared.

The kernels never wait on another rank; all waiting is on the host.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import sp


class ProcessBarrier:
    """Orders the ranks between two phases (see the module docstring)."""

    def __init__(self, device, group=None):
        self.device = torch.device(device)
        self.group = group
        self.count = 0

    def __call__(self):
        torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)
        self.count += 1


class SPProcessRank:
    """This process's rank of a sequence-parallel group: its `sp.SPRank`
    (shard of the residual stream, exchange buffers) with a peer table over
    every rank's buffers, opened through CUDA IPC."""

    def __init__(self, w, dims, global_ranges, device, group=None, e4m3: bool = False, qk_e4m3: bool = False):
        self.world = dist.get_world_size(group)
        self.index = dist.get_rank(group)
        self.group = group
        self.rank = sp.SPRank(w, dims, global_ranges, self.world, self.index, device)
        r = self.rank
        if e4m3:  # e4m3 block buffers; with qk_e4m3 the q, k exchange buffers hold codes
            r.alloc_e4m3(qk_e4m3)
        self._peers = sp.exchange_peer_tensors({"q": r.exchange_q(), "k": r.exchange_k(), "v": r.v, "o": r.o}, group)
        r.set_peers(self._peers["q"], self._peers["k"], self._peers["v"], self._peers["o"])
        self.barrier = ProcessBarrier(device, group)

    @property
    def layout(self):
        return self.rank.layout

    @property
    def shard(self):
        return self.rank.shard

    def block_forward(self, mod, W, stream=None):
        """One block on this rank's shard; every rank calls it with the same
        block (its own shard of the residual stream in `self.rank.x`)."""
        sp.block_forward([self.rank], mod, W, barrier=self.barrier, stream=stream)

    def block_forward_e4m3(self, mod, W8, stream=None):
        """One block with e4m3 GEMMs (constructed with e4m3=True)."""
        sp.block_forward_e4m3([self.rank], mod, W8, barrier=self.barrier, stream=stream)

    def close(self):
        """Release the peers' buffers before anyone frees its own."""
        self.barrier()
        self.rank.peers = None
        self._peers = None
        torch.cuda.synchronize(self.barrier.device)
        self.barrier()
