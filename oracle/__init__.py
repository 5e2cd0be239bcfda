"""fp64 CPU oracle for QK-Normed MLA decode attention (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package.
The product path (``qk_normed_latent_qkn_b200``) never imports, calls or
links it, and shares no code with it; the only common dependency is the
seeded input generator ``qkn_inputs``, which holds none of the method's
arithmetic.

What it computes is the *explicit* form that QK-Normed MLA replaces: every
cached token's full key k_{t,g} = c_t W^K_g is materialised, RMS-normalised
after the up-projection, and used in ordinary softmax attention whose values
are the latents c_t ("QK-Normed MLA: QK normalization without full key
caching", technical summary, "Planteamiento del Problema"; arXiv abstract).
The GPU path never forms these keys; the pages state that the absorbed form is
exactly equal to this one in exact arithmetic (technical summary,
"Contribuciones Clave" item 1; arXiv abstract).

Readings of points the pages leave open:
  * key RMS over the whole n_g*d_h output of W^K_g, one statistic per token
    and KV group (summary, Metodología item 2: one inverse-RMS scalar per
    token and KV group);
  * query RMS per (query token, head) over d_h;
  * S(z) = sqrt(mean(z^2) + eps), the same eps for all four norms;
  * content and RoPE blocks normalised separately (Metodología item 4); the
    RoPE block is normalised, then rotated, half-split pairs, base theta;
    key position = token index, query j of a step at position L - s_q + j;
  * softmax scale sigma on the whole logit, sigma = 1/sqrt(d_h + d_R);
  * values are the unnormalised latents c_t; the output lives in latent space;
  * a query sees the keys whose position is <= its own position.

The GQA route of GQLA (section 2, "Ruta GQA") is here too: the latent is
expanded once per token into one key head and one value head per KV group,
and decode is ordinary grouped-query attention over those cached keys and
values.  Readings: the group's key is RMS-normalised over its d_h columns
after the up-projection with the group's gamma_k (the QK-Normed key norm,
with one key head per group); the RoPE block and the queries as above; the
output is the value-space o_v [s_q, H, d_v].  Sparse GQLA (section 2, "GQLA
Disperso") is read as: every (query token, KV group) pair attends only to
a given list of its visible tokens, the n_g heads of the group sharing it.

Pins (tests/test_oracle_pins.py): exact absorbed == explicit equality in
rational arithmetic; invariance of the logits to rescaling c_t; softmax rows
summing to 1; closed forms (one token, zero queries, identical tokens); a
library softmax-attention routine on materialised keys; brute-force loops for
the causal mask; RoPE's relative-position property; permutation invariance.
The GQA route's pins: equality with the absorbed route over group-tied
weights; torch's grouped-query attention on keys and values the check forms;
a one-token closed form; a full selection equal to dense and an empty one
giving zeros; a brute-force loop over a sparse selection.
The absolute outputs on the workloads are parity unpinned beyond those
properties: the pages print no worked example.
"""
from __future__ import annotations

from typing import Iterable, Optional, Tuple

import numpy as np

__all__ = ["inv_rms", "rms_norm", "rope", "key_inv_rms", "rope_keys", "absorbed_query",
           "sequence_logits", "decode", "decode_sequence", "up_project", "group_keys",
           "group_values",
           "gqa_logits", "gqa_decode_sequence", "gqa_decode"]


def inv_rms(x: np.ndarray, eps: float) -> np.ndarray:
    """1 / S(x) with S(x) = sqrt(mean(x^2) + eps) over the last axis.

    RMSNorm splits into a static weight and this dynamic scalar statistic
    (technical summary, Metodología: RMSNorm(z) = z * gamma / S(z)).
    """
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm(x) = x * gamma / S(x) over the last axis (technical summary, Metodología)."""
    x = np.asarray(x, dtype=np.float64)
    return x * np.asarray(gamma, dtype=np.float64) * inv_rms(x, eps)[..., None]


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, half-split pairs (i, i + d/2), angle pos * theta^(-2i/d).

    ``x`` is [..., d]; ``pos`` broadcasts against x's leading axes.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    freq = theta ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    cos, sin = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def key_inv_rms(c: np.ndarray, w_k: np.ndarray, eps: float, chunk: int = 1024) -> np.ndarray:
    """a_k[t, g] = 1 / S(c_t W^K_g): the per-token, per-group dynamic key statistic.

    Computed from the materialised up-projection (technical summary,
    Metodología item 2; arXiv abstract).  ``c`` is [T, r], ``w_k`` [g, r, n_g*d_h].
    Returns [T, g].
    """
    c = np.asarray(c, dtype=np.float64)
    w = np.asarray(w_k, dtype=np.float64)
    out = np.empty((c.shape[0], w.shape[0]))
    for t0 in range(0, c.shape[0], chunk):
        cc = c[t0:t0 + chunk]
        for g in range(w.shape[0]):
            out[t0:t0 + chunk, g] = inv_rms(cc @ w[g], eps)
    return out


def rope_keys(k_rope: np.ndarray, gamma_kr: np.ndarray, pos: np.ndarray, eps: float,
              theta: float) -> np.ndarray:
    """RoPE key block: RMS-normalised on its own, then rotated (Metodología item 4)."""
    return rope(rms_norm(k_rope, gamma_kr, eps), pos, theta)


def absorbed_query(q: np.ndarray, w_k: np.ndarray, gamma_q: np.ndarray, gamma_k: np.ndarray,
                   eps: float, softmax_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Absorbed query and its row scale.

    q~[h] = W^K_{g(h),h} (gamma_q[h] * gamma_k[h] * q[h]) in R^r: both static
    norm weights are folded into the query side before the latent dot product
    (technical summary, Metodología item 1).  a_q[h] = sigma / S(q[h]) is the
    query-side inverse RMS with the softmax scale folded in, the row factor
    of the decode logit (Metodología, decode-logit equation).
    ``q`` is [..., H, d_h]; returns (q~ [..., H, r], a_q [..., H]).
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w_k, dtype=np.float64)
    g, r, width = w.shape
    H, d_h = q.shape[-2], q.shape[-1]
    ng = H // g
    scaled = q * np.asarray(gamma_q, np.float64) * np.asarray(gamma_k, np.float64)
    qt = np.empty(q.shape[:-1] + (r,))
    for h in range(H):
        grp, m = divmod(h, ng)
        w_h = w[grp][:, m * d_h:(m + 1) * d_h]            # [r, d_h]
        qt[..., h, :] = scaled[..., h, :] @ w_h.T
    a_q = softmax_scale * inv_rms(q, eps)
    return qt, a_q


def sequence_logits(inp, b: int, chunk: int = 1024,
                    key_pos: Optional[np.ndarray] = None) -> np.ndarray:
    """Explicit QK-RMSNorm attention logits of sequence b, [s_q, H, L] (fp64).

    l[j, h, t] = sigma * (RMSNorm(q_jh) . RMSNorm(c_t W^K_g)[h]
                          + RoPE(RMSNorm(q^R_jh)) . RoPE(RMSNorm(k^R_t))),
    -inf where key t sits after query j.  Keys are materialised chunk by chunk
    (technical summary, "Planteamiento del Problema": the naive form needs the
    fully projected key of every cached token).
    """
    wl = inp.wl
    sl = inp.sequence(b)
    c = np.asarray(inp.c[sl], dtype=np.float64)
    L = c.shape[0]
    kpos = np.arange(L) if key_pos is None else np.asarray(key_pos)
    qpos = inp.query_positions()[b]                                   # [s_q]
    H, ng, d_h = wl.heads, wl.heads_per_group, wl.d_h
    sigma = wl.softmax_scale

    qh = rms_norm(inp.q[b], inp.gamma_q, wl.eps)                      # [s_q, H, d_h]
    qrh = rope(rms_norm(inp.q_rope[b], inp.gamma_qr, wl.eps), qpos[:, None], wl.rope_theta)
    krh = rope_keys(inp.k_rope[sl], inp.gamma_kr, kpos, wl.eps, wl.rope_theta)   # [L, d_R]

    logits = np.empty((wl.s_q, H, L))
    w = np.asarray(inp.w_k, dtype=np.float64)
    for t0 in range(0, L, chunk):
        cc = c[t0:t0 + chunk]
        for g in range(wl.groups):
            heads = slice(g * ng, (g + 1) * ng)
            gk = np.asarray(inp.gamma_k[heads], np.float64).reshape(-1)   # [n_g*d_h]
            k = rms_norm(cc @ w[g], gk, wl.eps).reshape(cc.shape[0], ng, d_h)
            logits[:, heads, t0:t0 + chunk] = np.einsum("jmd,tmd->jmt", qh[:, heads], k)
    logits += np.einsum("jhd,td->jht", qrh, krh)
    logits *= sigma
    visible = kpos[None, :] <= qpos[:, None]                          # [s_q, L]
    logits[~np.broadcast_to(visible[:, None, :], logits.shape)] = -np.inf
    return logits


def decode_sequence(inp, b: int, chunk: int = 1024,
                    key_pos: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax over the cached context, then the weighted sum of latents c_t.

    Returns (o [s_q, H, r], lse [s_q, H]) for sequence b.
    """
    l = sequence_logits(inp, b, chunk, key_pos)
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    s = e.sum(axis=-1, keepdims=True)
    p = e / s
    lse = (m + np.log(s))[..., 0]
    c = np.asarray(inp.c[inp.sequence(b)], dtype=np.float64)
    return p @ c, lse


def decode(inp, seqs: Optional[Iterable[int]] = None,
           chunk: int = 1024) -> Tuple[np.ndarray, np.ndarray]:
    """Decode outputs for the listed sequences (all by default).

    Returns (o [B, s_q, H, r], lse [B, s_q, H]); rows of sequences not listed
    are NaN.
    """
    wl = inp.wl
    B = wl.batch
    o = np.full((B, wl.s_q, wl.heads, wl.r_kv), np.nan)
    lse = np.full((B, wl.s_q, wl.heads), np.nan)
    for b in (range(B) if seqs is None else seqs):
        o[b], lse[b] = decode_sequence(inp, b, chunk)
    return o, lse


def up_project(o_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """Per-head value up-projection of the latent attention output.

    The values of the absorbed path are the latents c_t themselves, so the
    attention output lives in latent space; the value up-projection W^UV_h of
    each head is applied once to that output instead of to every cached
    token (GQLA summary, section 2, absorbed MQA route: the up-projections
    move into the query and output projections).
    ``o_lat`` is [..., H, r] and ``w_uv`` [H, r, d_v]; returns [..., H, d_v].
    """
    o = np.asarray(o_lat, dtype=np.float64)
    w = np.asarray(w_uv, dtype=np.float64)
    out = np.empty(o.shape[:-1] + (w.shape[2],))
    for h in range(w.shape[0]):
        out[..., h, :] = o[..., h, :] @ w[h]
    return out


def group_keys(c: np.ndarray, w_uk: np.ndarray, gamma_k: np.ndarray, eps: float) -> np.ndarray:
    """Keys of the GQA route: k_{t,g} = RMSNorm(c_t W^UK_g) gamma_k[g] over the group's d_h columns.

    The latent expanded into one key head per KV group, which that route
    caches (GQLA summary, section 2, "Ruta GQA"), normalised after its
    up-projection as the QK-Normed key is (technical summary, "Planteamiento
    del Problema").  ``c`` [T, r], ``w_uk`` [g, r, d_h], ``gamma_k`` [g, d_h];
    returns [T, g, d_h].
    """
    c = np.asarray(c, dtype=np.float64)
    wk = np.asarray(w_uk, dtype=np.float64)
    return np.stack([rms_norm(c @ wk[g], np.asarray(gamma_k[g], np.float64), eps) for g in range(wk.shape[0])],
                    axis=1)


def group_values(c: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """Values of the GQA route: v_{t,g} = c_t W^UV_g (GQLA summary, section 2, "Ruta GQA").

    ``c`` [T, r], ``w_uv`` [g, r, d_v]; returns [T, g, d_v].
    """
    c = np.asarray(c, dtype=np.float64)
    wv = np.asarray(w_uv, dtype=np.float64)
    return np.stack([c @ wv[g] for g in range(wv.shape[0])], axis=1)


def gqa_logits(inp, b: int, w_uk: np.ndarray, gamma_k: np.ndarray,
               selection: Optional[np.ndarray] = None) -> np.ndarray:
    """Logits of grouped-query attention over the expanded keys of sequence b, [s_q, H, L].

    l[j, h, t] = sigma * (RMSNorm(q_jh) . k_{t,g(h)} + RoPE(RMSNorm(q^R_jh)) . RoPE(RMSNorm(k^R_t))),
    g(h) = h // n_g; -inf where key t sits after query j, and, with ``selection``
    ([s_q, g, K] token positions, -1 = none), where t is not listed for (j, g(h))
    (GQLA summary, section 2, "Ruta GQA" and "GQLA Disperso").
    """
    wl = inp.wl
    sl = inp.sequence(b)
    c = np.asarray(inp.c[sl], dtype=np.float64)
    L = c.shape[0]
    qpos = inp.query_positions()[b]
    H, ng = wl.heads, wl.heads_per_group
    k = group_keys(c, w_uk, gamma_k, wl.eps)                                       # [L, g, d_h]
    qh = rms_norm(inp.q[b], inp.gamma_q, wl.eps)                                   # [s_q, H, d_h]
    qrh = rope(rms_norm(inp.q_rope[b], inp.gamma_qr, wl.eps), pos=qpos[:, None], theta=wl.rope_theta)
    krh = rope_keys(inp.k_rope[sl], inp.gamma_kr, np.arange(L), wl.eps, wl.rope_theta)
    grp = np.arange(H) // ng
    logits = np.empty((wl.s_q, H, L))
    for g in range(wl.groups):                       # the group's n_g heads share its key head
        logits[:, g * ng:(g + 1) * ng] = np.einsum("jmd,td->jmt", qh[:, g * ng:(g + 1) * ng], k[:, g, :])
    logits = logits + np.einsum("jhd,td->jht", qrh, krh)
    logits *= wl.softmax_scale
    visible = np.arange(L)[None, :] <= qpos[:, None]                               # [s_q, L]
    mask = np.broadcast_to(visible[:, None, :], logits.shape).copy()
    if selection is not None:
        listed = np.zeros((wl.s_q, wl.groups, L), dtype=bool)
        for j in range(wl.s_q):
            for g in range(wl.groups):
                idx = np.asarray(selection[j, g])
                idx = idx[(idx >= 0) & (idx < L)]
                listed[j, g, idx] = True
        mask &= listed[:, grp, :]
    logits[~mask] = -np.inf
    return logits


def gqa_decode_sequence(inp, b: int, w_uk: np.ndarray, gamma_k: np.ndarray, w_uv: np.ndarray,
                        selection: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax over the listed / visible tokens, then the weighted sum of the group's values.

    Returns (o_v [s_q, H, d_v], lse [s_q, H]) for sequence b; a row with no
    token gives zeros and lse = -inf.
    """
    wl = inp.wl
    c = np.asarray(inp.c[inp.sequence(b)], dtype=np.float64)
    v = group_values(c, w_uv)                                                      # [L, g, d_v]
    l = gqa_logits(inp, b, w_uk, gamma_k, selection)
    m = l.max(axis=-1, keepdims=True)
    has = np.isfinite(m)
    e = np.exp(l - np.where(has, m, 0.0))
    s = e.sum(axis=-1, keepdims=True)
    p = np.where(has, e / np.where(has, s, 1.0), 0.0)
    lse = np.where(has, m + np.log(np.where(has, s, 1.0)), -np.inf)[..., 0]
    ng = wl.heads_per_group
    o = np.empty((wl.s_q, wl.heads, v.shape[2]))
    for g in range(wl.groups):                       # ... and its value head
        o[:, g * ng:(g + 1) * ng] = np.einsum("jmt,td->jmd", p[:, g * ng:(g + 1) * ng], v[:, g, :])
    return o, lse


def gqa_decode(inp, w_uk: np.ndarray, gamma_k: np.ndarray, w_uv: np.ndarray,
               seqs: Optional[Iterable[int]] = None,
               selection: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """GQA-route decode outputs for the listed sequences (all by default).

    ``selection`` [B, s_q, g, K] selects sparse attention.  Returns
    (o_v [B, s_q, H, d_v], lse [B, s_q, H]); rows of sequences not listed are NaN.
    """
    wl = inp.wl
    B = wl.batch
    o = np.full((B, wl.s_q, wl.heads, w_uv.shape[2]), np.nan)
    lse = np.full((B, wl.s_q, wl.heads), np.nan)
    for b in (range(B) if seqs is None else seqs):
        o[b], lse[b] = gqa_decode_sequence(inp, b, w_uk, gamma_k, w_uv,
                                           None if selection is None else selection[b])
    return o, lse
