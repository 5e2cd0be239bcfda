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
