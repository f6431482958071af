"""Sequence parallelism (Ulysses) for the block: buffers and call order of one
rank, and the peer-buffer exchange between processes.

"MiniMax-H3 paper reading" (gojay.top) §7.2 deploys the trunk with Ulysses
degree 4: every rank holds a contiguous shard of the packed sequence, and
attention re-shards tokens -> heads before and heads -> tokens after.  The
library fuses both exchanges into the kernels that produce the data
(h3_qkv_qknorm_mrope_sp, h3_attention_sp), writing through the peer table;
this module only allocates, orders the calls and orders the ranks between
the phases.  Every step runs in the library's kernels.
"""
from __future__ import annotations

import torch

from . import h3


class SPRank:
    """One rank's buffers: its shard of the residual stream and the two
    exchange targets other ranks write into (q/k/v for this rank's heads over
    the whole sequence, o for this rank's rows over all heads)."""

    def __init__(self, w, dims, global_ranges, n_ranks: int, rank: int, device):
        self.w, self.dims = w, dims
        self.layout, self.shard = h3.h3_sp_make_layout(dims, global_ranges, n_ranks, rank)
        lay = self.layout
        Ls, D, I, F = lay.L_shard, w.D, w.I, w.F
        dev = torch.device(device)
        e = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=dev)
        self.x = e(Ls, D)
        self.pos = e(Ls, 3)
        self.xm = e(Ls, D, dt=torch.bfloat16)
        self.q = e(lay.heads, lay.L_total, 128, dt=torch.bfloat16)
        self.k = e(lay.heads, lay.L_total, 128, dt=torch.bfloat16)
        self.v = e(lay.heads, lay.L_total, 128, dt=torch.bfloat16)
        self.o = e(Ls, I, dt=torch.bfloat16)
        self.ws = e(Ls, F, dt=torch.bfloat16)
        self.peers = None
        self.qk_e4m3 = False

    @property
    def rows(self) -> slice:
        """This shard's rows of the global padded sequence."""
        return slice(self.layout.row0, self.layout.row0 + self.layout.L_shard)

    def set_peers(self, q, k, v, o):
        """Peer table: per-rank lists (index = rank) of the q/k/v/o exchange
        buffers, this rank's own entries included (q, k: the e4m3 code
        buffers when the rank exchanges codes, see alloc_e4m3)."""
        self.peers = h3.sp_peers(q, k, v, o, qk_e4m3=self.qk_e4m3)

    def alloc_e4m3(self, qk_e4m3: bool = False):
        """Buffers of the e4m3 block on this shard; qk_e4m3: q and k cross to
        the head-group ranks as e4m3 codes ([H/N][L_total][128] bytes, the
        exchange buffers q8, k8), v stays bf16.  Call before linking peers."""
        lay, w, d = self.layout, self.w, self.dims
        Ls, D, I = lay.L_shard, w.D, w.I
        dev = self.x.device
        self.xq = torch.empty(Ls, D, dtype=torch.uint8, device=dev)
        self.xs = torch.empty(Ls, dtype=torch.float32, device=dev)
        self.oq = torch.empty(Ls, I, dtype=torch.uint8, device=dev)
        self.os = torch.empty(Ls, dtype=torch.float32, device=dev)
        self.ws8 = torch.empty(h3.h3_ffn_e4m3_workspace_bytes(d, Ls), dtype=torch.uint8, device=dev)
        self.qk_e4m3 = qk_e4m3
        if qk_e4m3:
            self.q8 = torch.empty(lay.heads, lay.L_total, 128, dtype=torch.uint8, device=dev)
            self.k8 = torch.empty(lay.heads, lay.L_total, 128, dtype=torch.uint8, device=dev)

    def exchange_q(self):
        return self.q8 if self.qk_e4m3 else self.q

    def exchange_k(self):
        return self.k8 if self.qk_e4m3 else self.k

    # ------------------------------------------------------------ phases
    def phase_qkv(self, mod, W, stream=None):
        """LN + modulation, then QKV with Q/K RMSNorm + RoPE, each head group
        stored into its rank's q/k/v."""
        d, s = self.dims, self.shard
        h3.h3_adaln_norm_modulate(d, s, self.x, mod, h3.H3_MSA, self.xm, stream=stream)
        h3.h3_qkv_qknorm_mrope_sp(d, s, self.layout, self.xm, W["Wqkv"], W["qn_w"], W["kn_w"], self.pos,
                                  self.peers, stream=stream)

    def phase_attention(self, W=None, stream=None):
        """Attention for this rank's heads over all tokens, each output row
        stored into its owner's o (W: the block weights, whose Q/K norm
        weights select the split-softmax kernel, as in the single-sequence
        block)."""
        qn, kn = (W["qn_w"], W["kn_w"]) if W is not None else (None, None)
        h3.h3_attention_sp(self.dims, self.layout, self.peers, qn_w=qn, kn_w=kn, stream=stream)

    def phase_qkv_e4m3(self, mod, W8, stream=None):
        """The e4m3 QKV phase: LN + modulation to e4m3 codes, then the e4m3
        QKV GEMM with its norm + RoPE epilogue, each head group stored into
        its rank's q/k/v (q, k as codes with qk_e4m3)."""
        d, s = self.dims, self.shard
        flags = h3.H3_QK_NORM_ROPE_IN_QKV | (h3.H3_QK_E4M3 if self.qk_e4m3 else 0)
        h3.h3_adaln_norm_modulate_e4m3(d, s, self.x, mod, h3.H3_MSA, self.xq, self.xs, stream=stream)
        h3.h3_qkv_qknorm_mrope_sp_e4m3(d, s, self.layout, self.xq, self.xs, W8["Wqkv"], W8["Wqkv_s"], W8["qn_w"],
                                       W8["kn_w"], self.pos, self.peers, flags=flags, stream=stream)

    def phase_attention_e4m3(self, W8, stream=None):
        flags = h3.H3_QK_NORM_ROPE_IN_QKV | (h3.H3_QK_E4M3 if self.qk_e4m3 else 0)
        h3.h3_attention_sp(self.dims, self.layout, self.peers, qn_w=W8["qn_w"], kn_w=W8["kn_w"], flags=flags,
                           stream=stream)

    def phase_out_ffn_e4m3(self, mod, W8, stream=None):
        d, s = self.dims, self.shard
        h3.h3_quantize_rows_e4m3(self.o, self.oq, self.os, stream=stream)
        h3.h3_gated_residual_e4m3(d, s, self.x, self.oq, self.os, W8["Wo"], W8["Wo_s"], mod, h3.H3_MSA,
                                  stream=stream)
        h3.h3_adaln_norm_modulate_e4m3(d, s, self.x, mod, h3.H3_MLP, self.xq, self.xs, stream=stream)
        h3.h3_ffn_swiglu_e4m3(d, s, self.x, self.xq, self.xs, W8["Wgu"], W8["Wgu_s"], W8["Wd"], W8["Wd_s"], mod,
                              self.ws8, stream=stream)

    def phase_out_ffn(self, mod, W, stream=None):
        """The token-local rest of the block on this shard."""
        d, s = self.dims, self.shard
        h3.h3_gated_residual(d, s, self.x, self.o, W["Wo"], mod, h3.H3_MSA, stream=stream)
        h3.h3_adaln_norm_modulate(d, s, self.x, mod, h3.H3_MLP, self.xm, stream=stream)
        h3.h3_ffn_swiglu(d, s, self.x, self.xm, W["Wgu"], W["Wd"], mod, self.ws, stream=stream)


def link_local(ranks: list[SPRank]):
    """Peer tables for ranks that share one process (and GPU): each rank's
    table points at the others' buffers directly."""
    q = [r.exchange_q() for r in ranks]
    k = [r.exchange_k() for r in ranks]
    v = [r.v for r in ranks]
    o = [r.o for r in ranks]
    for r in ranks:
        r.set_peers(q, k, v, o)


def block_forward(ranks: list[SPRank], mod, W, barrier=None, stream=None):
    """One block on the ranks held by this process.  barrier() must make
    every rank's writes of the previous phase complete and visible to all
    ranks before the next phase starts (between processes: e.g. a
    stream-ordered collective); ranks that share one stream are already
    ordered by it."""
    for r in ranks:
        r.phase_qkv(mod, W, stream)
    if barrier:
        barrier()
    for r in ranks:
        r.phase_attention(W, stream)
    if barrier:
        barrier()
    for r in ranks:
        r.phase_out_ffn(mod, W, stream)


def block_forward_e4m3(ranks: list[SPRank], mod, W8, barrier=None, stream=None):
    """block_forward with the four GEMMs on e4m3 operands (W8: the block's
    e4m3 weights and scales as from H3BlockStep.quantize_block_weights_e4m3;
    every rank's alloc_e4m3 called before its peers were linked)."""
    for r in ranks:
        r.phase_qkv_e4m3(mod, W8, stream)
    if barrier:
        barrier()
    for r in ranks:
        r.phase_attention_e4m3(W8, stream)
    if barrier:
        barrier()
    for r in ranks:
        r.phase_out_ffn_e4m3(mod, W8, stream)


def exchange_peer_tensors(local: dict, group=None) -> dict:
    """Between processes on one node: every rank shares its exchange buffers
    (dict name -> tensor) through the process group and opens the others'
    with torch's multiprocessing reductions (CUDA IPC handles for CUDA
    tensors; shared memory for CPU tensors, which must already be in shared
    memory).  Returns name -> list of tensors indexed by rank, the local
    rank's own tensors at its index.  The tensors passed in must stay alive
    while peers use them."""
    import pickle
    from multiprocessing.reduction import ForkingPickler

    import torch.distributed as dist
    import torch.multiprocessing  # noqa: F401  (registers torch's reducers with ForkingPickler)

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    mine = bytes(ForkingPickler.dumps(local))
    gathered = [None] * world
    dist.all_gather_object(gathered, mine, group=group)
    out = {n: [None] * world for n in local}
    for g in range(world):
        peer = local if g == rank else pickle.loads(gathered[g])
        for n in local:
            out[n][g] = peer[n]
    return out
