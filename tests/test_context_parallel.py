"""Context-parallel decode, host side (CPU): the page slices of each rank, the
inputs a rank hands to the decode, and the exchange over torch.distributed
(gloo, world size 2) with the ranks' partial results computed here from the
oracle's logits on each slice and merged by the softmax identity.  The GPU
side (the decode's vis_end and qkn_merge_partials) is in
test_context_parallel_gpu.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from qk_normed_latent_qkn_b200 import context_parallel as cp
from qkn_inputs import WORKLOADS, make_inputs


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_slices_partition_every_sequence(world):
    rng = np.random.default_rng(world)
    lens = rng.integers(2 * world * 64 - 63, 40 * 64, size=17)
    sl = cp.page_slices(lens, world)
    n = (lens + 63) // 64
    assert sl.shape == (world, 17, 2)
    assert (sl[0, :, 0] == 0).all() and (sl[-1, :, 1] == n).all()
    assert (sl[1:, :, 0] == sl[:-1, :, 1]).all()             # contiguous, no overlap
    assert ((sl[:, :, 1] - sl[:, :, 0]) >= 2).all()          # every slice spans two pages or more


def test_too_short_sequences_are_refused():
    with pytest.raises(ValueError):
        cp.page_slices([64 * 7], 4)                          # 7 pages < 2 x 4
    with pytest.raises(ValueError):
        cp.page_slices([64 * 8], 4, s_q=200)                 # slices of 128 tokens < s_q


def test_rank_view():
    lens = np.array([1000, 64 * 20, 64 * 9 + 1])
    bt = np.arange(3 * 40, dtype=np.int32).reshape(3, 40)
    world = 3
    sl = cp.page_slices(lens, world)
    for r in range(world):
        t, l, ve = cp.rank_view(bt, lens, r, world)
        for b in range(3):
            lo, hi = sl[r, b]
            assert (t[b, :hi - lo] == bt[b, lo:hi]).all()
            assert l[b] == min(lens[b], hi * 64) - lo * 64     # the slice's tokens
            assert ve[b] == lens[b] - lo * 64                  # the sequence's end in the slice's numbering
            assert l[b] >= 64                                  # more than any s_q


def _slice_partial(inp, world, rank):
    """(out [B, s_q, H, r], lse [B, s_q, H]) of one rank: softmax over its slice's tokens only, from
    the oracle's logits over the whole sequence (so the causal limit is the whole sequence's)."""
    wl = inp.wl
    sl = cp.page_slices(inp.seq_lens, world)[rank]
    outs = np.zeros((wl.batch, wl.s_q, wl.heads, wl.r_kv))
    lses = np.full((wl.batch, wl.s_q, wl.heads), -np.inf)
    for b in range(wl.batch):
        l = oracle.sequence_logits(inp, b)                   # [s_q, H, L]
        t0, t1 = sl[b, 0] * 64, min(int(inp.seq_lens[b]), sl[b, 1] * 64)
        ls = l[..., t0:t1]
        m = ls.max(axis=-1, keepdims=True)
        e = np.exp(ls - m)
        s = e.sum(axis=-1, keepdims=True)
        outs[b] = (e / s) @ np.asarray(inp.c[inp.sequence(b)], dtype=np.float64)[t0:t1]
        lses[b] = (m + np.log(s))[..., 0]
    return outs, lses


def _np_merge(outs, lses):
    m = lses.max(axis=0)
    w = np.exp(lses - m)
    den = w.sum(axis=0)
    return (w[..., None] * outs).sum(axis=0) / den[..., None], m + np.log(den)


CP_CASE = WORKLOADS["grouped_mtp_bf16"].with_(batch=2, heads=8, groups=2, r_kv=64, d_h=32, d_rope=16,
                                               context=(300, 700), dtype="f32", seed=81)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = make_inputs(CP_CASE)

        class _Session:
            dims = None

        # the exchange and the merge of ContextParallelDecode, with the slice decode and the merge
        # kernel replaced by host stand-ins (the kernels are tested on the GPU)
        def fake_slice(session, block_table, seq_lens, s_q, r, w, **kw):
            o, l = _slice_partial(inp, w, r)
            return torch.from_numpy(o), torch.from_numpy(l)

        def fake_merge(dims, outs, lses):
            o, l = _np_merge(outs.numpy(), lses.numpy())
            return torch.from_numpy(o), torch.from_numpy(l)

        cp.slice_decode, cp.merge = fake_slice, fake_merge
        out, lse = cp.ContextParallelDecode(_Session(), rank, world).decode(inp.block_table, inp.seq_lens,
                                                                           inp.wl.s_q)
        q.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_slices_merge_to_the_whole_sequence_softmax():
    # the page slices' partial softmaxes merge to the oracle's decode (s_q = 2: the causal limit
    # counts from the whole sequence's end)
    inp = make_inputs(CP_CASE)
    o_ref, lse_ref = oracle.decode(inp)
    for world in (2, 3):
        parts = [_slice_partial(inp, world, r) for r in range(world)]
        o, l = _np_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
        assert np.abs(l - lse_ref).max() <= 1e-12


def test_two_rank_exchange_over_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted((q.get(timeout=10) for _ in range(world)), key=lambda x: x[0])
    o_ref, lse_ref = oracle.decode(make_inputs(CP_CASE))
    for rank, o, l in res:
        assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
        assert np.abs(l - lse_ref).max() <= 1e-12
