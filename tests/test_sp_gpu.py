"""Sequence parallelism (Ulysses) on one GPU: N ranks emulated with all their
buffers on the same device, the phases ordered by the stream.  The fused
exchanges (QKV epilogue -> head-group owner, attention epilogue -> row owner)
then write through the same peer-table code path as between GPUs.

The sharded block must reproduce the single-sequence block bit for bit
(every output element is accumulated over the same K in the same order, and
attention sees the same keys in the same tile order), and the oracle block
within the block tolerance."""
import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from omni_modal_diffusion_b200 import synthetic as S
from omni_modal_diffusion_b200 import h3, sp
from omni_modal_diffusion_b200.pipeline import H3BlockStep, to_dev_bf16

from parity_util import RAGGED, check_close, oracle_ranges_and_pos, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from omni_modal_diffusion_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


import dataclasses

# 2,015 tokens (text 37, audio 58, video 5 x 16 x 24) and 8 heads: long enough
# for four shards of 512 rows, the last one holding 479 valid rows
LONG = dataclasses.replace(RAGGED, name="long", index=11, H=8, T_lat=5, H_lat=32, W_lat=48)


@pytest.mark.parametrize("w,n_ranks", [(RAGGED, 2), (RAGGED, 3), (LONG, 4)], ids=["ragged2", "ragged3", "long4"])
def test_sp_block_matches_single_gpu_block_and_oracle(w, n_ranks):
    inp = S.make_inputs(w)
    st = H3BlockStep(w, weights=inp)
    text, video, audio = (to_dev_bf16(inp[k], st.device) for k in ("text", "video", "audio"))
    mod = torch.from_numpy(inp["mod"]).to(st.device)
    st.embed(text, video, audio)
    x0 = st.x.clone()
    pos = st.pos.clone()
    L = st.ranges.L

    ranks = [sp.SPRank(w, st.dims, st.ranges, n_ranks, r, DEV) for r in range(n_ranks)]
    Lt = ranks[0].layout.L_total
    for r in ranks:
        assert r.layout.L_total == Lt
        r.x.zero_()
        r.pos.zero_()
        rows = r.rows
        lo, hi = rows.start, min(rows.stop, st.ranges.L_pad)
        if hi > lo:
            r.x[: hi - lo].copy_(x0[lo:hi])
            r.pos[: hi - lo].copy_(pos[lo:hi])
        # stale values everywhere the exchange must overwrite
        for t in (r.q, r.k, r.v, r.o):
            t.fill_(float("nan"))
    sp.link_local(ranks)
    sp.block_forward(ranks, mod, st.W)
    st.block(mod)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0

    x_sp = torch.cat([r.x for r in ranks], 0)[:L]
    assert torch.equal(x_sp, st.x[:L]), "sharded block differs from the single-sequence block"
    for r in ranks:  # padding rows of every shard untouched (zero)
        assert torch.all(r.x[r.shard.L:] == 0)

    r_o, pos_o = oracle_ranges_and_pos(w)
    xo = O.embed(inp["text"], inp["video"], inp["audio"], inp["W_text"], inp["W_vid"], inp["W_aud"], r_o)
    ref = O.block_forward(xo, inp["mod"], r_o, pos_o, inp["Wqkv"], inp["qn_w"], inp["kn_w"], inp["Wo"], inp["Wgu"],
                          inp["Wd"], w.H)
    check_close(to_np(x_sp), ref, "sequence-parallel block output")


def test_sp_exchange_targets():
    """Every q/k/v row of every rank's receive buffer and every o row is
    written by the exchange (the buffers start as NaN), with the q of head
    group g at rank g in global row order."""
    w = RAGGED
    inp = S.make_inputs(w)
    st = H3BlockStep(w, weights=inp)
    text, video, audio = (to_dev_bf16(inp[k], st.device) for k in ("text", "video", "audio"))
    mod = torch.from_numpy(inp["mod"]).to(st.device)
    st.embed(text, video, audio)
    n = 2
    ranks = [sp.SPRank(w, st.dims, st.ranges, n, r, DEV) for r in range(n)]
    for r in ranks:
        r.x.zero_()
        r.pos.zero_()
        lo, hi = r.rows.start, min(r.rows.stop, st.ranges.L_pad)
        r.x[: hi - lo].copy_(st.x[lo:hi])
        r.pos[: hi - lo].copy_(st.pos[lo:hi])
        for t in (r.q, r.k, r.v, r.o):
            t.fill_(float("nan"))
    sp.link_local(ranks)
    for r in ranks:
        r.phase_qkv(mod, st.W)
    # the single-sequence QKV for comparison
    h3.h3_adaln_norm_modulate(st.dims, st.ranges, st.x, mod, h3.H3_MSA, st.xm)
    h3.h3_qkv_qknorm_mrope(st.dims, st.ranges, st.xm, st.W["Wqkv"], st.W["qn_w"], st.W["kn_w"], st.pos,
                           st.q, st.k, st.v)
    torch.cuda.synchronize()
    Lp, hpr = st.ranges.L_pad, ranks[0].layout.heads
    for g, r in enumerate(ranks):
        for name in ("q", "k", "v"):
            got = getattr(r, name)
            assert not torch.isnan(got).any(), f"{name} of rank {g} not fully written"
            want = getattr(st, name)[g * hpr:(g + 1) * hpr]
            assert torch.equal(got[:, :Lp], want)
            assert torch.all(got[:, Lp:] == 0)
    for r in ranks:
        r.phase_attention()
    torch.cuda.synchronize()
    for r in ranks:
        assert not torch.isnan(r.o).any()


def test_sp_argument_errors():
    w = RAGGED
    d = h3.make_dims(w.D, w.H, w.F)
    g = h3.h3_make_ranges(37, 58, 240)
    lay, shard = h3.h3_sp_make_layout(d, g, 2, 0)
    buf = torch.empty(16, dtype=torch.bfloat16, device=DEV)
    peers = h3.sp_peers(q=[buf, buf], k=[buf, buf], v=[buf, buf], o=[buf, buf])
    bad = h3.SPLayout.from_buffer_copy(lay)
    bad.L_shard = 200
    with pytest.raises(h3.H3Error):
        h3.h3_attention_sp(d, bad, peers)
    empty = h3.SPPeers()
    with pytest.raises(h3.H3Error):
        h3.h3_attention_sp(d, lay, empty)


@pytest.mark.parametrize("qk_e4m3", [False, True], ids=["qk_bf16", "qk_e4m3"])
@pytest.mark.parametrize("w,n_ranks", [(RAGGED, 2), (RAGGED, 3), (LONG, 4)], ids=["ragged2", "ragged3", "long4"])
def test_sp_e4m3_block_matches_single_gpu_e4m3_block(w, n_ranks, qk_e4m3):
    """Sequence parallelism with the block's GEMMs on e4m3 operands, and with
    qk_e4m3 the q, k crossing to the head-group ranks as e4m3 codes: the
    sharded block equals the single-sequence e4m3 block bit for bit (the
    same codes, scales and accumulation order per row)."""
    inp = S.make_inputs(w)
    st = H3BlockStep(w, weights=inp)
    text, video, audio = (to_dev_bf16(inp[k], st.device) for k in ("text", "video", "audio"))
    mod = torch.from_numpy(inp["mod"]).to(st.device)
    st.embed(text, video, audio)
    W8 = st.quantize_block_weights_e4m3()
    st.alloc_e4m3()
    x0 = st.x.clone()
    pos = st.pos.clone()
    L = st.ranges.L

    ranks = [sp.SPRank(w, st.dims, st.ranges, n_ranks, r, DEV) for r in range(n_ranks)]
    for r in ranks:
        r.alloc_e4m3(qk_e4m3)
        r.x.zero_()
        r.pos.zero_()
        lo, hi = r.rows.start, min(r.rows.stop, st.ranges.L_pad)
        if hi > lo:
            r.x[: hi - lo].copy_(x0[lo:hi])
            r.pos[: hi - lo].copy_(pos[lo:hi])
        for t in (r.v, r.o):
            t.fill_(float("nan"))
        if qk_e4m3:
            r.q8.fill_(0x7F)  # e4m3 NaN codes: a row the exchange misses shows
            r.k8.fill_(0x7F)
        else:
            r.q.fill_(float("nan"))
            r.k.fill_(float("nan"))
    sp.link_local(ranks)
    sp.block_forward_e4m3(ranks, mod, W8)
    st.block_e4m3(mod, W8, qk_e4m3=qk_e4m3)
    torch.cuda.synchronize()
    assert h3.h3_device_status() == 0
    x_sp = torch.cat([r.x for r in ranks], 0)[:L]
    assert torch.equal(x_sp, st.x[:L]), "sharded e4m3 block differs from the single-sequence e4m3 block"
    for r in ranks:
        assert torch.all(r.x[r.shard.L:] == 0)
