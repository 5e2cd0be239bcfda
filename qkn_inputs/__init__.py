"""Seeded synthetic workloads for QK-Normed MLA latent decode.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no norms, no rotations, no attention).  Both the fp64
oracle (``oracle/``) and the CUDA path (tests, ``bench.py``) take their inputs
from here, so that the two see the same bits.

Workload shapes follow the decode setting of "QK-Normed MLA: QK normalization
without full key caching" (abstract and "Resultos": decode at contexts up to
256k tokens) and the absorbed-MQA decode shape of "GQLA" (section 2, "Ruta
MQA-Absorbida": r_kv latent plus one shared RoPE key per token).  The pages
give no model dimensions, so the five workloads below fix them.

Value recipe (identical for every workload):
  * per-token scale s_t = exp(0.5 * N(0,1))  (log-normal(0, 0.5));
  * latent c_t = N(0,1) * s_t, raw RoPE key k^R_t = N(0,1) * s_t;
  * queries q, q^R ~ N(0,1);
  * key up-projection W^K_g ~ N(0, 1/r_kv);
  * norm weights gamma ~ 1 + 0.1 * N(0,1);
  * eps = 1e-6, RoPE base 10000.
Draw order from one ``numpy.random.Generator(PCG64(seed))``: sequence lengths,
block permutation, s_t, c, k^R, q, q^R, W^K, gamma_q, gamma_k, gamma_qR,
gamma_kR, W^UV (value up-projection, N(0, 1/r_kv)).

Tied groups (``Workload.tied_groups``): the GQLA parameterisation, where the
up-projections are indexed by KV group rather than by head ("GQLA", section
2, Arquitectura): one key head W^UK_g [r, d_h] with its norm weight
gamma_k,g [d_h] and one value head W^UV_g [r, d_v] per group.  They are drawn
with the group's shape in the same order, then laid out per head (W^K_g as
n_g copies of W^UK_g side by side, gamma_k and W^UV repeated over the
group's heads), so that the per-head arrays describe the same model and the
absorbed route reads them unchanged.  Values are drawn in fp32
and, for bf16 workloads, the stored activations (c, k^R, q, q^R) and W^UV
(which the library reads in the storage type) are rounded once to bf16 (round
to nearest even); the other weights and the gammas stay fp32.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence, Tuple, Union

import numpy as np

BLOCK_SIZE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and storage type of one decode workload."""
    name: str
    batch: int
    s_q: int
    heads: int
    groups: int
    r_kv: int
    d_h: int
    d_rope: int
    context: Union[int, Tuple[int, int]]   # fixed length, or inclusive (lo, hi) uniform range
    paged: bool                            # random block table (else identity table)
    dtype: str                             # "f32" or "bf16": storage type of activations and cache
    eps: float = 1e-6
    rope_theta: float = 10000.0
    seed: int = 0
    block_size: int = BLOCK_SIZE
    d_v: int = 128                         # per-head value width of the output up-projection
    tied_groups: bool = False              # one key head and one value head per KV group (GQLA)

    @property
    def heads_per_group(self) -> int:
        return self.heads // self.groups

    @property
    def softmax_scale(self) -> float:
        return float(1.0 / np.sqrt(self.d_h + self.d_rope))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five decode workloads and a prefill workload.  d_h = 128 where the workload statement leaves it
# open (long-context and grouped cases), as in the large MLA case.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", batch=1, s_q=1, heads=4, groups=1, r_kv=64, d_h=32,
                         d_rope=16, context=256, paged=False, dtype="f32", d_v=32),
    "small_mla_bf16": Workload("small_mla_bf16", batch=16, s_q=1, heads=16, groups=1, r_kv=512,
                               d_h=128, d_rope=64, context=4096, paged=False, dtype="bf16"),
    "large_mla_bf16": Workload("large_mla_bf16", batch=32, s_q=1, heads=128, groups=1, r_kv=512,
                               d_h=128, d_rope=64, context=(1024, 32768), paged=True,
                               dtype="bf16"),
    "long_ctx_bf16": Workload("long_ctx_bf16", batch=2, s_q=1, heads=128, groups=1, r_kv=512,
                              d_h=128, d_rope=64, context=262144, paged=True, dtype="bf16"),
    "grouped_mtp_bf16": Workload("grouped_mtp_bf16", batch=8, s_q=2, heads=64, groups=4,
                                 r_kv=512, d_h=128, d_rope=64, context=(4096, 65536),
                                 paged=True, dtype="bf16"),
    # attention forward over whole sequences (prefill / training-time forward): every token is a
    # query, causal (s_q = context)
    "prefill_mla_bf16": Workload("prefill_mla_bf16", batch=2, s_q=2048, heads=16, groups=1, r_kv=512,
                                 d_h=128, d_rope=64, context=2048, paged=True, dtype="bf16"),
    # GQLA's configuration for its GQA route (h_q = 128, g = 8, so h_q / g = 16, with a two-token
    # MTP step): keys and values expanded per group; the context mix of the large MLA case
    "gqla_gqa_bf16": Workload("gqla_gqa_bf16", batch=32, s_q=2, heads=128, groups=8, r_kv=512, d_h=128,
                              d_rope=64, context=(1024, 32768), paged=True, dtype="bf16", tied_groups=True),
}
WORKLOAD_ORDER = ["tiny_f32", "small_mla_bf16", "large_mla_bf16", "long_ctx_bf16", "prefill_mla_bf16",
                  "grouped_mtp_bf16", "gqla_gqa_bf16"]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # finite inputs only: the largest finite pattern 0xFF7FFFFF plus 0x8000 stays below 2^32
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fp32 values that are already bf16-exact (the bf16 encoding)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass
class Inputs:
    """One seeded decode problem.

    Token-major arrays are concatenated over sequences; sequence b owns rows
    ``tok_off[b] : tok_off[b] + seq_lens[b]``.  All float arrays are fp32 and,
    for bf16 workloads, hold bf16-exact values.
    """
    wl: Workload
    seq_lens: np.ndarray        # [B] int32
    tok_off: np.ndarray         # [B+1] int64
    block_table: np.ndarray     # [B, max_blocks] int32 physical block ids (unused entries 0)
    num_blocks: int             # size of the physical block pool
    c: np.ndarray               # [T, r]     latent c_t
    k_rope: np.ndarray          # [T, d_R]   raw RoPE key (before norm and rotation)
    q: np.ndarray               # [B, s_q, H, d_h] content query
    q_rope: np.ndarray          # [B, s_q, H, d_R] raw RoPE query
    w_k: np.ndarray             # [g, r, n_g*d_h] key up-projection W^K_g
    gamma_q: np.ndarray         # [H, d_h]
    gamma_k: np.ndarray         # [H, d_h]  head h's slice of its group's key norm weight
    gamma_qr: np.ndarray        # [H, d_R]
    gamma_kr: np.ndarray        # [d_R]     shared RoPE key norm weight
    w_uv: np.ndarray            # [H, r, d_v] value up-projection W^UV_h of every head

    @property
    def total_tokens(self) -> int:
        return int(self.tok_off[-1])

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    def token_positions(self) -> np.ndarray:
        """Position of every cached token inside its sequence, [T] int32."""
        return np.concatenate([np.arange(n, dtype=np.int32) for n in self.seq_lens])

    def token_slots(self) -> np.ndarray:
        """Physical cache slot (block * block_size + offset) of every cached token, [T] int32."""
        bs = self.wl.block_size
        out = []
        for b, n in enumerate(self.seq_lens):
            t = np.arange(n, dtype=np.int64)
            out.append(self.block_table[b, t // bs].astype(np.int64) * bs + t % bs)
        return np.concatenate(out).astype(np.int32)

    def query_positions(self) -> np.ndarray:
        """Position of query token j of sequence b: L_b - s_q + j, [B, s_q] int32."""
        s_q = self.wl.s_q
        return (self.seq_lens[:, None] - s_q + np.arange(s_q)[None, :]).astype(np.int32)

    def sequence(self, b: int) -> slice:
        return slice(int(self.tok_off[b]), int(self.tok_off[b + 1]))

    def group_weights(self) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """The per-group weights of a tied-groups workload, in the group layout:
        W^UK [g, r, d_h], gamma_k [g, d_h], W^UV [g, r, d_v] (slices of the per-head arrays)."""
        if not self.wl.tied_groups:
            raise ValueError("group weights exist only for a tied-groups workload")
        ng = self.wl.heads_per_group
        return (np.ascontiguousarray(self.w_k[:, :, :self.wl.d_h]), np.ascontiguousarray(self.gamma_k[::ng]),
                np.ascontiguousarray(self.w_uv[::ng]))


def make_inputs(wl: Union[str, Workload], seed: Optional[int] = None,
                seq_lens: Optional[Sequence[int]] = None) -> Inputs:
    """Draw one decode problem for workload ``wl`` (a name or a Workload).

    ``seq_lens`` overrides the drawn context lengths (its draw is still
    consumed so that later draws keep their order).
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    if seed is not None:
        wl = wl.with_(seed=seed)
    if wl.heads % wl.groups:
        raise ValueError("heads must be a multiple of groups")
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    B, bs = wl.batch, wl.block_size

    if isinstance(wl.context, tuple):
        lo, hi = wl.context
        drawn = rng.integers(lo, hi + 1, size=B)
    else:
        drawn = np.full(B, wl.context)
    lens = np.asarray(seq_lens if seq_lens is not None else drawn, dtype=np.int32)
    if lens.shape != (B,) or (lens < wl.s_q).any():
        raise ValueError("need one length >= s_q per sequence")

    nblk = (lens.astype(np.int64) + bs - 1) // bs
    pool = int(nblk.sum())
    max_blocks = int(nblk.max())
    drawn_perm = rng.permutation(pool).astype(np.int32)      # drawn either way: keeps later draws aligned
    perm = drawn_perm if wl.paged else np.arange(pool, dtype=np.int32)
    table = np.zeros((B, max_blocks), dtype=np.int32)
    boff = np.concatenate([[0], np.cumsum(nblk)])
    for b in range(B):
        table[b, :nblk[b]] = perm[boff[b]:boff[b + 1]]

    tok_off = np.concatenate([[0], np.cumsum(lens.astype(np.int64))])
    T = int(tok_off[-1])
    f32 = np.float32
    s_t = np.exp(0.5 * rng.standard_normal(T, dtype=f32)).astype(f32)
    c = rng.standard_normal((T, wl.r_kv), dtype=f32) * s_t[:, None]
    k_rope = rng.standard_normal((T, wl.d_rope), dtype=f32) * s_t[:, None]
    q = rng.standard_normal((B, wl.s_q, wl.heads, wl.d_h), dtype=f32)
    q_rope = rng.standard_normal((B, wl.s_q, wl.heads, wl.d_rope), dtype=f32)
    ng = wl.heads_per_group
    kh = 1 if wl.tied_groups else ng                    # key heads drawn per group
    vh = wl.groups if wl.tied_groups else wl.heads      # value heads drawn
    w_k = rng.standard_normal((wl.groups, wl.r_kv, kh * wl.d_h), dtype=f32) * f32(1.0 / np.sqrt(wl.r_kv))
    gamma_q = (1.0 + 0.1 * rng.standard_normal((wl.heads, wl.d_h), dtype=f32)).astype(f32)
    gamma_k = (1.0 + 0.1 * rng.standard_normal((wl.groups * kh, wl.d_h), dtype=f32)).astype(f32)
    gamma_qr = (1.0 + 0.1 * rng.standard_normal((wl.heads, wl.d_rope), dtype=f32)).astype(f32)
    gamma_kr = (1.0 + 0.1 * rng.standard_normal(wl.d_rope, dtype=f32)).astype(f32)
    # drawn last, so that every value above is the same with or without it
    w_uv = rng.standard_normal((vh, wl.r_kv, wl.d_v), dtype=f32) * f32(1.0 / np.sqrt(wl.r_kv))
    if wl.tied_groups:
        # lay the group's single key and value head out over its n_g query heads
        w_k = np.ascontiguousarray(np.tile(w_k, (1, 1, ng)))
        gamma_k = np.ascontiguousarray(np.repeat(gamma_k, ng, axis=0))
        w_uv = np.ascontiguousarray(np.repeat(w_uv, ng, axis=0))

    if wl.dtype == "bf16":
        c, k_rope, q, q_rope, w_uv = (round_to_bf16(a) for a in (c, k_rope, q, q_rope, w_uv))
    elif wl.dtype != "f32":
        raise ValueError(f"unknown dtype {wl.dtype}")

    return Inputs(wl=wl, seq_lens=lens, tok_off=tok_off, block_table=table, num_blocks=pool,
                  c=np.ascontiguousarray(c, f32), k_rope=np.ascontiguousarray(k_rope, f32),
                  q=q, q_rope=q_rope, w_k=w_k, gamma_q=gamma_q, gamma_k=gamma_k,
                  gamma_qr=gamma_qr, gamma_kr=gamma_kr, w_uv=w_uv)


def make_selection(inp: Inputs, k: int, seed: int = 0) -> np.ndarray:
    """Token selections for sparse attention over the GQA route: [B, s_q, g, k] int32.

    For query token j of sequence b and KV group g, ``k`` distinct positions drawn uniformly
    without replacement from the tokens that query can see (positions 0 .. L_b - s_q + j), in
    random order; when fewer are visible, all of them, then -1 (no token) in the remaining
    entries.  Drawn from ``numpy.random.Generator(PCG64(seed))``, one draw per (b, j, g) in
    that order.
    """
    wl = inp.wl
    rng = np.random.Generator(np.random.PCG64(seed))
    out = np.full((wl.batch, wl.s_q, wl.groups, k), -1, dtype=np.int32)
    qpos = inp.query_positions()
    for b in range(wl.batch):
        for j in range(wl.s_q):
            n = int(qpos[b, j]) + 1
            for g in range(wl.groups):
                if n <= k:
                    out[b, j, g, :n] = rng.permutation(n)
                else:
                    out[b, j, g] = rng.choice(n, size=k, replace=False)
    return out
