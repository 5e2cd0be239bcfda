"""Context-parallel decode: one long sequence's pages split across ranks.

Each rank decodes a contiguous slice of every sequence's pages with the
library's split-KV decode (``qkn_decode`` with ``qkn_decode_opts.vis_end``,
so the causal limit stays the whole sequence's), the ranks' partial results
(normalised output and lse per query row) are all-gathered, and
``qkn_merge_partials`` merges them: the softmax over the union of the
slices' tokens (QKN summary, decode-logit equation; the same identity as the
split-KV merge).  The exchange is one all-gather of ``B·s_q·H·(r·elem + 4)``
bytes per rank (256 KB per sequence at 128 heads, r = 512, bf16), over NCCL
on GPUs.  Host logic only: every arithmetic step runs in libqkn.

Slices: sequence b has ``n_b = ceil(L_b / 64)`` pages; rank k of W takes
pages ``[floor(n_b k / W), floor(n_b (k + 1) / W))``.  Every slice must hold
at least ``s_q`` tokens (the decode's length check): ``n_b >= 2 W`` pages per
sequence, so that each slice spans at least two pages, and enough of them for
a longer query chunk.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
import torch

from . import merge_partials

BLOCK = 64


def page_slices(seq_lens, world: int, s_q: int = 1) -> np.ndarray:
    """[world, B, 2] int64: the page range (lo, hi) of each rank for each sequence."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    n = (lens + BLOCK - 1) // BLOCK
    if world < 1:
        raise ValueError("world must be >= 1")
    if np.any(n < 2 * world):
        raise ValueError(f"context parallelism over {world} ranks needs at least {2 * world} pages per "
                         f"sequence (shortest: {int(n.min())})")
    k = np.arange(world + 1, dtype=np.int64)[:, None]
    bounds = (n[None, :] * k) // world                  # [world + 1, B]
    sl = np.stack([bounds[:-1], bounds[1:]], axis=-1)
    tokens = np.minimum(lens[None, :], sl[..., 1] * BLOCK) - sl[..., 0] * BLOCK
    if np.any(tokens < s_q):
        raise ValueError(f"a slice over {world} ranks would hold fewer than s_q = {s_q} tokens")
    return sl


def rank_view(block_table, seq_lens, rank: int, world: int, s_q: int = 1) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The decode inputs of one rank: its block table (each row starts at the slice's first page),
    its token counts and the causal limit's end in the slice's numbering (vis_end)."""
    bt = np.asarray(block_table, dtype=np.int32)
    lens = np.asarray(seq_lens, dtype=np.int64)
    sl = page_slices(lens, world, s_q)[rank]            # [B, 2]
    width = int((sl[:, 1] - sl[:, 0]).max())
    out = np.zeros((bt.shape[0], width), dtype=np.int32)
    for b, (lo, hi) in enumerate(sl):
        out[b, :hi - lo] = bt[b, lo:hi]
    lens_r = np.minimum(lens, sl[:, 1] * BLOCK) - sl[:, 0] * BLOCK
    vis_end = lens - sl[:, 0] * BLOCK
    return out, lens_r.astype(np.int32), vis_end.astype(np.int32)


def slice_decode(session, block_table, seq_lens, s_q: int, rank: int, world: int, **kw):
    """This rank's partial result (out [B, s_q, H, r], lse [B, s_q, H]) for its page slices."""
    bt, lens, vis_end = rank_view(block_table, seq_lens, rank, world, s_q)
    return session.decode(bt, lens, s_q, vis_end=vis_end, **kw)


def merge(dims, outs, lses):
    """Merge stacked partial results ([P, B, s_q, H, r], [P, B, s_q, H]) with qkn_merge_partials."""
    out = torch.empty(outs.shape[1:], dtype=outs.dtype, device=outs.device)
    lse = torch.empty(lses.shape[1:], dtype=torch.float32, device=lses.device)
    merge_partials(dims, outs.contiguous(), lses.contiguous(), out, lse)
    return out, lse


class ContextParallelDecode:
    """One rank of a context-parallel decode over ``torch.distributed`` (NCCL on GPUs).

    Every rank holds the whole cache pool and block table (the pages it reads are its slices'),
    calls ``decode`` with the same arguments, and gets the full result."""

    def __init__(self, session, rank: int, world: int, group: Optional[object] = None):
        self.session, self.rank, self.world, self.group = session, rank, world, group

    def decode(self, block_table, seq_lens, s_q: int, **kw):
        import torch.distributed as dist
        out_r, lse_r = slice_decode(self.session, block_table, seq_lens, s_q, self.rank, self.world, **kw)
        # gathered as a concatenation along the first dimension, then viewed rank-major
        outs = torch.empty((self.world * out_r.shape[0],) + tuple(out_r.shape[1:]), dtype=out_r.dtype,
                           device=out_r.device)
        lses = torch.empty((self.world * lse_r.shape[0],) + tuple(lse_r.shape[1:]), dtype=lse_r.dtype,
                           device=lse_r.device)
        dist.all_gather_into_tensor(outs, out_r.contiguous(), group=self.group)
        dist.all_gather_into_tensor(lses, lse_r.contiguous(), group=self.group)
        return merge(self.session.dims, outs.view((self.world,) + tuple(out_r.shape)),
                     lses.view((self.world,) + tuple(lse_r.shape)))
