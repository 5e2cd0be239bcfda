"""Algorithmic bytes and FLOPs of one QK-Normed MLA decode step.

Per cached token a decode step must read its bf16 latent (2 r bytes), its
bf16 RoPE key (2 d_R bytes) and, for QK-Normed MLA, its fp32 inverse-RMS
scalar for each KV group (4 g bytes) — the whole per-token cache, since
nothing else is stored ("QK-Normed MLA: QK normalization without full key
caching", technical summary, Metodología item 3).  Each query row that sees
the token spends 2(r + d_R) FLOPs on its logit and 2 r FLOPs on the weighted
sum of latents.  Without the scalar cache this is the absorbed-MLA decode
whose arithmetic intensity the GQLA page quotes as about 242 FLOP/byte at
s_q = 1 with 128 heads, r = 512, d_R = 64 ("GQLA", section 2, Ruta
MQA-Absorbida).
"""
from __future__ import annotations

import dataclasses
from typing import Sequence


@dataclasses.dataclass(frozen=True)
class StepCost:
    cache_bytes: int       # cached tokens x per-token cache bytes
    query_bytes: int       # q~, a_q, q^R^ read once per query row
    output_bytes: int      # o (bf16/fp32) and lse written once per query row
    flops: int

    @property
    def bytes(self) -> int:
        return self.cache_bytes + self.query_bytes + self.output_bytes

    @property
    def intensity(self) -> float:
        return self.flops / self.bytes


def cache_bytes_per_token(r: int, d_rope: int, groups: int, elem: int = 2, scalar_cache: bool = True) -> int:
    return elem * (r + d_rope) + (4 * groups if scalar_cache else 0)


def flops_per_token_row(r: int, d_rope: int) -> int:
    return 2 * (r + d_rope) + 2 * r


def decode_step_cost(seq_lens: Sequence[int], s_q: int, heads: int, groups: int, r: int, d_rope: int,
                     elem: int = 2, scalar_cache: bool = True) -> StepCost:
    """Cost of one decode step over sequences of the given context lengths.

    Query j of a sequence of length L sees L - s_q + j + 1 tokens.
    """
    tokens = sum(int(L) for L in seq_lens)
    pairs = sum(int(L) - s_q + j + 1 for L in seq_lens for j in range(s_q))   # (query token, key) pairs
    rows = len(seq_lens) * s_q * heads
    return StepCost(
        cache_bytes=tokens * cache_bytes_per_token(r, d_rope, groups, elem, scalar_cache),
        query_bytes=rows * (elem * (r + d_rope) + 4),
        output_bytes=rows * (elem * r + 4),
        flops=pairs * heads * flops_per_token_row(r, d_rope),
    )


# ----------------------------------------------------------------- the GQA route
def gqa_bytes_per_token(groups: int, d_h: int, d_rope: int, d_v: int, elem: int = 2) -> int:
    """Cache bytes per token of the GQA route: one key and one value head per group plus the shared
    RoPE key ("GQLA", section 2, Ruta GQA: 2 g d_h values plus the RoPE key when d_v = d_h)."""
    return elem * (groups * (d_h + d_v) + d_rope)


def gqa_flops_per_token_row(d_h: int, d_rope: int, d_v: int) -> int:
    """A query row's FLOPs on one visible token: its logit over d_h + d_R, its share of the values."""
    return 2 * (d_h + d_rope) + 2 * d_v


def gqa_step_cost(seq_lens: Sequence[int], s_q: int, heads: int, groups: int, d_h: int, d_rope: int, d_v: int,
                  elem: int = 2) -> StepCost:
    """Cost of one GQA-route decode step: the expanded cache read once, the raw queries read, o_v and lse
    written; FLOPs over the causal (query token, key) pairs of every head."""
    tokens = sum(int(L) for L in seq_lens)
    pairs = sum(int(L) - s_q + j + 1 for L in seq_lens for j in range(s_q))
    rows = len(seq_lens) * s_q * heads
    return StepCost(
        cache_bytes=tokens * gqa_bytes_per_token(groups, d_h, d_rope, d_v, elem),
        query_bytes=rows * elem * (d_h + d_rope),
        output_bytes=rows * (elem * d_v + 4),
        flops=pairs * heads * gqa_flops_per_token_row(d_h, d_rope, d_v),
    )


# ----------------------------------------------------------------- the merge of the split-KV partials
def split_counts(seq_lens: Sequence[int], s_q: int, max_blocks: int, ht_count: int, ncta: int,
                 item_cost: int, block: int = 64) -> list:
    """Splits (partial results) of each sequence's segments under the decode's split schedule.

    Host restatement of the schedule for cost accounting: sequence b is item_cost + n(b) units
    (n(b) pages; none for a rejected length), laid out one after another; the CTAs form
    G = ncta // min(HT, ncta) groups, group g takes units [g Q, (g + 1) Q), Q = ceil(total / G); a
    segment is split wherever a group boundary falls inside its pages.  Every row tile of a
    sequence has the same count.
    """
    n = [0 if (int(L) < s_q or int(L) > max_blocks * block) else -(-int(L) // block) for L in seq_lens]
    units = [x + item_cost if x > 0 else 0 for x in n]
    total = sum(units)
    hc = min(ht_count, ncta)
    groups = max(1, ncta // max(hc, 1))
    q = max(1, -(-total // groups))
    out, u0 = [], 0
    for nb, ub in zip(n, units):
        if nb == 0:
            out.append(0)
        else:
            pg0 = u0 + item_cost
            out.append((pg0 + nb - 1) // q - pg0 // q + 1)
        u0 += ub
    return out


@dataclasses.dataclass(frozen=True)
class MergeCost:
    partial_bytes: int     # fp32 partial rows and their lse, read once
    weight_bytes: int      # W^UV (fused merge only), read once
    output_bytes: int      # merged rows (or o_v) and lse, written once
    flops: int             # the up-projection (fused merge only)

    @property
    def bytes(self) -> int:
        return self.partial_bytes + self.weight_bytes + self.output_bytes


def merge_cost(splits: Sequence[int], s_q: int, heads: int, r: int, elem: int = 2, d_v: int = 0) -> MergeCost:
    """Bytes of the merge of one step: every query row reads its splits' fp32 partial row (4 r bytes)
    and lse (4 bytes).  d_v = 0: the plain merge writes the latent row (elem r bytes) and lse.
    d_v > 0: the merge fused with the value up-projection also reads W^UV once (heads r d_v elements)
    and writes o_v (elem d_v bytes per row) and lse, at 2 r d_v FLOPs per row."""
    rows_per_seq = s_q * heads
    parts = sum(int(x) for x in splits) * rows_per_seq
    rows = len(splits) * rows_per_seq
    width = d_v if d_v else r
    return MergeCost(partial_bytes=parts * (4 * r + 4), weight_bytes=heads * r * d_v * elem,
                     output_bytes=rows * (elem * width + 4), flops=2 * rows * r * d_v)
