"""Checks that pin the fp64 oracle to facts other than itself.

Each check is a plain function that raises AssertionError on failure, so
that ``test_oracle_pins.py`` runs them as tests and
``test_oracle_mutations.py`` can plant mistakes in the oracle and confirm
that at least one check catches each.  Nothing here reuses the oracle's own
helpers to build an expected value: every expected value is re-derived here
along a different route (exact rationals, the Gram identity, complex
rotation, a library attention routine, plain Python loops, closed forms).
"""
from __future__ import annotations

import cmath
import math
from fractions import Fraction

import numpy as np
import torch

import oracle
from qkn_inputs import Workload, make_inputs, make_selection

TINY = Workload("pin_tiny", batch=2, s_q=1, heads=4, groups=2, r_kv=8, d_h=4, d_rope=4,
                context=(5, 19), paged=True, dtype="f32", seed=3)
TINY_MTP = TINY.with_(name="pin_mtp", s_q=2, seed=4)


# --------------------------------------------------------------------------
# 1. Absorbed == explicit (technical summary, "Contribuciones Clave" item 1;
#    arXiv abstract: exact equivalence in exact arithmetic).
# --------------------------------------------------------------------------
def check_absorbed_query_exact():
    """q~ . c equals the explicit bilinear form, exactly, on small integers."""
    rng = np.random.default_rng(11)
    r, d_h, H, g = 5, 3, 4, 2
    ng = H // g
    c = rng.integers(-4, 5, size=(6, r)).astype(np.float64)
    w = rng.integers(-3, 4, size=(g, r, ng * d_h)).astype(np.float64)
    q = rng.integers(-3, 4, size=(H, d_h)).astype(np.float64)
    gq = rng.integers(1, 4, size=(H, d_h)).astype(np.float64)
    gk = rng.integers(1, 4, size=(H, d_h)).astype(np.float64)
    qt, _ = oracle.absorbed_query(q, w, gq, gk, eps=1e-6, softmax_scale=1.0)
    for h in range(H):
        grp, m = h // ng, h % ng
        for t in range(c.shape[0]):
            # explicit: key slice of head h from the group's up-projection, weighted by gamma_k,
            # dotted with the gamma_q-weighted query (norm scalars factored out)
            z = [sum(Fraction(int(c[t, i])) * Fraction(int(w[grp, i, m * d_h + d])) for i in range(r))
                 for d in range(d_h)]
            expl = sum(Fraction(int(q[h, d])) * Fraction(int(gq[h, d])) * Fraction(int(gk[h, d])) * z[d]
                       for d in range(d_h))
            absb = float(np.dot(qt[h], c[t]))
            assert Fraction(absb) == expl, (h, t, absb, expl)


def _rotate_complex(x, pos, theta):
    """RoPE restated as complex multiplication of pairs (x_i, x_{i+d/2})."""
    d = len(x)
    half = d // 2
    out = np.empty(d)
    for i in range(half):
        z = complex(x[i], x[i + half]) * cmath.exp(1j * pos * theta ** (-2.0 * i / d))
        out[i], out[i + half] = z.real, z.imag
    return out


def _absorbed_logits(inp, b):
    """Logits along the absorbed route, with a_k from the Gram identity ||c W||^2 = c (W W^T) c^T."""
    wl = inp.wl
    sl = inp.sequence(b)
    c = inp.c[sl].astype(np.float64)
    L = c.shape[0]
    ng, d_h = wl.heads // wl.groups, wl.d_h
    width = ng * d_h
    sigma = 1.0 / math.sqrt(wl.d_h + wl.d_rope)
    w = inp.w_k.astype(np.float64)
    a_k = np.empty((L, wl.groups))
    for g in range(wl.groups):
        gram = w[g] @ w[g].T
        a_k[:, g] = 1.0 / np.sqrt(np.einsum("ti,ij,tj->t", c, gram, c) / width + wl.eps)
    kr = np.empty((L, wl.d_rope))
    for t in range(L):
        x = inp.k_rope[sl][t].astype(np.float64)
        xn = x * inp.gamma_kr / math.sqrt(float(np.mean(x * x)) + wl.eps)
        kr[t] = _rotate_complex(xn, t, wl.rope_theta)
    out = np.empty((wl.s_q, wl.heads, L))
    for j in range(wl.s_q):
        qpos = int(inp.seq_lens[b]) - wl.s_q + j
        for h in range(wl.heads):
            grp, m = h // ng, h % ng
            qv = inp.q[b, j, h].astype(np.float64)
            qtil = w[grp][:, m * d_h:(m + 1) * d_h] @ (qv * inp.gamma_q[h] * inp.gamma_k[h])
            a_q = sigma / math.sqrt(float(np.mean(qv * qv)) + wl.eps)
            xr = inp.q_rope[b, j, h].astype(np.float64)
            qr = _rotate_complex(xr * inp.gamma_qr[h] / math.sqrt(float(np.mean(xr * xr)) + wl.eps),
                                 qpos, wl.rope_theta)
            # decode logit: (q~ . c_t) * a_q * a_k[t, g(h)] plus the RoPE block
            out[j, h] = (c @ qtil) * a_q * a_k[:, grp] + sigma * (kr @ qr)
            out[j, h, np.arange(L) > qpos] = -np.inf
    return out


def check_absorbed_query_row_scale():
    """The absorbed route's content logit a_q * a_k * (q~ . c_t), with q~ and a_q taken from
    oracle.absorbed_query, equals sigma * RMSNorm(q) gamma_q . RMSNorm(c_t W^K_g)_h gamma_k with
    the key materialised here (technical summary, Metodología, decode-logit equation: the row
    scalar carries the query's inverse RMS over d_h and the softmax scale).  a_k comes from the
    Gram identity, so no oracle helper enters the expected value."""
    for wl in (TINY, TINY_MTP):
        inp = make_inputs(wl)
        ng, d_h = wl.heads // wl.groups, wl.d_h
        sigma = 1.0 / math.sqrt(wl.d_h + wl.d_rope)
        w = inp.w_k.astype(np.float64)
        for b in range(wl.batch):
            c = inp.c[inp.sequence(b)].astype(np.float64)
            qt, a_q = oracle.absorbed_query(inp.q[b], inp.w_k, inp.gamma_q, inp.gamma_k, wl.eps, sigma)
            assert a_q.shape == (wl.s_q, wl.heads)
            for g in range(wl.groups):
                gram = w[g] @ w[g].T
                a_k = 1.0 / np.sqrt(np.einsum("ti,ij,tj->t", c, gram, c) / (ng * d_h) + wl.eps)
                z = c @ w[g]                                           # materialised keys [L, n_g*d_h]
                zn = z / np.sqrt((z * z).mean(-1, keepdims=True) + wl.eps)
                for m in range(ng):
                    h = g * ng + m
                    key = zn[:, m * d_h:(m + 1) * d_h] * inp.gamma_k[h].astype(np.float64)
                    for j in range(wl.s_q):
                        qv = inp.q[b, j, h].astype(np.float64)
                        qn = qv / math.sqrt(float(np.mean(qv * qv)) + wl.eps) * inp.gamma_q[h].astype(np.float64)
                        expl = sigma * (key @ qn)
                        absb = a_q[j, h] * a_k * (c @ qt[j, h])
                        np.testing.assert_allclose(absb, expl, rtol=1e-10, atol=1e-12)


def check_absorbed_logits_match():
    for wl in (TINY, TINY_MTP):
        inp = make_inputs(wl)
        for b in range(wl.batch):
            ref = _absorbed_logits(inp, b)
            got = oracle.sequence_logits(inp, b)
            fin = np.isfinite(ref)
            assert np.array_equal(fin, np.isfinite(got))
            np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-10, atol=1e-12)


def check_key_inv_rms_gram():
    inp = make_inputs(TINY)
    w = inp.w_k.astype(np.float64)
    c = inp.c.astype(np.float64)
    got = oracle.key_inv_rms(c, w, TINY.eps, chunk=7)
    width = w.shape[2]
    for g in range(w.shape[0]):
        ref = 1.0 / np.sqrt(np.einsum("ti,ij,tj->t", c, w[g] @ w[g].T, c) / width + TINY.eps)
        np.testing.assert_allclose(got[:, g], ref, rtol=1e-12)


# --------------------------------------------------------------------------
# 2. RMSNorm makes the content logit invariant to rescaling c_t
#    (technical summary, Metodología: RMSNorm(z) = z * gamma / S(z)).
# --------------------------------------------------------------------------
def check_latent_scale_invariance():
    wl = TINY.with_(eps=0.0)
    inp = make_inputs(wl)
    base = [oracle.sequence_logits(inp, b) for b in range(wl.batch)]
    o0, _ = oracle.decode(inp)
    s = np.exp(np.random.default_rng(5).standard_normal(inp.total_tokens))
    inp.c = (inp.c.astype(np.float64) * s[:, None])
    for b in range(wl.batch):
        got = oracle.sequence_logits(inp, b)
        fin = np.isfinite(base[b])
        np.testing.assert_allclose(got[fin], base[b][fin], rtol=1e-11, atol=1e-12)
    # a uniform scale of every latent scales the output (values are c_t) and nothing else
    inp.c = inp.c / s[:, None] * 3.0
    o1, _ = oracle.decode(inp)
    np.testing.assert_allclose(o1, 3.0 * o0, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# 3. Softmax over the cached context: rows sum to one.
# --------------------------------------------------------------------------
def check_softmax_rows_sum_to_one():
    inp = make_inputs(TINY_MTP)
    for b in range(TINY_MTP.batch):
        l = oracle.sequence_logits(inp, b)
        _, lse = oracle.decode_sequence(inp, b)
        p = np.exp(l - lse[..., None])
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# 4. Closed forms.
# --------------------------------------------------------------------------
def check_single_token_returns_latent():
    wl = TINY.with_(context=1)
    inp = make_inputs(wl, seq_lens=[1, 1])
    o, lse = oracle.decode(inp)
    for b in range(wl.batch):
        np.testing.assert_allclose(o[b, 0], np.broadcast_to(inp.c[inp.sequence(b)][0], o[b, 0].shape),
                                   rtol=0, atol=1e-14)
        l = oracle.sequence_logits(inp, b)
        np.testing.assert_allclose(lse[b], l[..., 0], rtol=0, atol=1e-14)


def check_zero_query_is_uniform_mean():
    inp = make_inputs(TINY_MTP)
    inp.q[:] = 0.0
    inp.q_rope[:] = 0.0
    o, lse = oracle.decode(inp)
    for b in range(TINY_MTP.batch):
        c = inp.c[inp.sequence(b)].astype(np.float64)
        L = c.shape[0]
        for j in range(TINY_MTP.s_q):
            n = L - TINY_MTP.s_q + j + 1          # visible tokens
            np.testing.assert_allclose(o[b, j], np.broadcast_to(c[:n].mean(0), o[b, j].shape),
                                       rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse[b, j], math.log(n), rtol=1e-12)


def check_identical_tokens_return_that_token():
    inp = make_inputs(TINY)
    for b in range(TINY.batch):
        sl = inp.sequence(b)
        inp.c[sl] = inp.c[sl][0]
        inp.k_rope[sl] = 0.0
    o, _ = oracle.decode(inp)
    for b in range(TINY.batch):
        np.testing.assert_allclose(o[b, 0], np.broadcast_to(inp.c[inp.sequence(b)][0], o[b, 0].shape),
                                   rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# 5. Library routine: torch fp64 scaled_dot_product_attention on keys that
#    this check materialises itself (content block and RoPE block side by side).
# --------------------------------------------------------------------------
def check_against_library_attention():
    for wl in (TINY, TINY_MTP):
        inp = make_inputs(wl)
        o_ref, _ = oracle.decode(inp)
        ng, d_h = wl.heads // wl.groups, wl.d_h
        sigma = 1.0 / math.sqrt(wl.d_h + wl.d_rope)
        for b in range(wl.batch):
            sl = inp.sequence(b)
            c = torch.tensor(inp.c[sl], dtype=torch.float64)
            L = c.shape[0]
            w = torch.tensor(inp.w_k, dtype=torch.float64)
            keys = []
            for g in range(wl.groups):
                z = c @ w[g]
                z = z / torch.sqrt((z * z).mean(-1, keepdim=True) + wl.eps)
                gk = torch.tensor(inp.gamma_k[g * ng:(g + 1) * ng], dtype=torch.float64)
                keys.append(z.view(L, ng, d_h) * gk)
            k = torch.cat(keys, dim=1).permute(1, 0, 2)                         # [H, L, d_h]
            krs = inp.k_rope[sl].astype(np.float64)
            kr = torch.tensor(np.stack([_rotate_complex(
                krs[t] * inp.gamma_kr.astype(np.float64) / math.sqrt(float(np.mean(krs[t] ** 2)) + wl.eps),
                t, wl.rope_theta) for t in range(L)]))
            qv = torch.tensor(inp.q[b], dtype=torch.float64)                     # [s_q, H, d_h]
            qn = qv / torch.sqrt((qv * qv).mean(-1, keepdim=True) + wl.eps) * torch.tensor(
                inp.gamma_q, dtype=torch.float64)
            qr = np.empty((wl.s_q, wl.heads, wl.d_rope))
            for j in range(wl.s_q):
                for h in range(wl.heads):
                    x = inp.q_rope[b, j, h].astype(np.float64)
                    qr[j, h] = _rotate_complex(x * inp.gamma_qr[h].astype(np.float64) / math.sqrt(float(np.mean(x * x)) + wl.eps),
                                               L - wl.s_q + j, wl.rope_theta)
            qcat = torch.cat([qn, torch.tensor(qr)], -1).permute(1, 0, 2)        # [H, s_q, d]
            kcat = torch.cat([k, kr.unsqueeze(0).expand(wl.heads, L, wl.d_rope)], -1)
            v = c.unsqueeze(0).expand(wl.heads, L, c.shape[1])
            mask = (torch.arange(L)[None, :] <= (L - wl.s_q + torch.arange(wl.s_q))[:, None])
            out = torch.nn.functional.scaled_dot_product_attention(
                qcat, kcat, v, attn_mask=mask, scale=sigma)                        # [H, s_q, r]
            np.testing.assert_allclose(o_ref[b], out.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# 6. Brute force in plain Python on a tiny case, causal within the step.
# --------------------------------------------------------------------------
def check_brute_force_causal():
    wl = Workload("pin_brute", batch=1, s_q=2, heads=2, groups=1, r_kv=3, d_h=2, d_rope=2,
                  context=4, paged=False, dtype="f32", eps=0.25, seed=9)
    inp = make_inputs(wl)
    o, lse = oracle.decode(inp)
    L, r = 4, 3
    c = [[float(inp.c[t, i]) for i in range(r)] for t in range(L)]
    sigma = 1.0 / math.sqrt(wl.d_h + wl.d_rope)

    def rmsinv(v):
        return 1.0 / math.sqrt(sum(x * x for x in v) / len(v) + wl.eps)

    def rot(v, pos):   # d = 2: one pair, frequency 1
        a = pos * 1.0
        return [v[0] * math.cos(a) - v[1] * math.sin(a), v[1] * math.cos(a) + v[0] * math.sin(a)]

    for j in range(2):
        qpos = L - 2 + j
        for h in range(2):
            logits = []
            for t in range(L):
                if t > qpos:
                    continue
                z = [sum(c[t][i] * float(inp.w_k[0, i, col]) for i in range(r)) for col in range(4)]
                zs = rmsinv(z)
                key = [z[h * 2 + d] * zs * float(inp.gamma_k[h, d]) for d in range(2)]
                qv = [float(x) for x in inp.q[0, j, h]]
                qs = rmsinv(qv)
                qn = [qv[d] * qs * float(inp.gamma_q[h, d]) for d in range(2)]
                kr = [float(x) for x in inp.k_rope[t]]
                krn = rot([kr[d] * rmsinv(kr) * float(inp.gamma_kr[d]) for d in range(2)], t)
                qr = [float(x) for x in inp.q_rope[0, j, h]]
                qrn = rot([qr[d] * rmsinv(qr) * float(inp.gamma_qr[h, d]) for d in range(2)], qpos)
                logits.append(sigma * (sum(a * b for a, b in zip(qn, key)) +
                                       sum(a * b for a, b in zip(qrn, krn))))
            mx = max(logits)
            ex = [math.exp(x - mx) for x in logits]
            s = sum(ex)
            ov = [sum(ex[t] / s * c[t][i] for t in range(len(ex))) for i in range(r)]
            np.testing.assert_allclose(o[0, j, h], ov, rtol=1e-12, atol=1e-14)
            assert abs(lse[0, j, h] - (mx + math.log(s))) < 1e-12


def check_prefill_rows_are_prefix_decodes():
    # a whole sequence as queries (s_q = L): query j sits at position j and sees tokens 0 .. j, so
    # its output is the one-query decode of the length-(j + 1) prefix, and query 0 returns c_0
    import dataclasses
    L = 7
    wl = TINY.with_(name="pin_prefill", batch=1, s_q=L, context=L, seed=11)
    inp = make_inputs(wl)
    o, lse = oracle.decode(inp)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(inp.c[0], o[0, 0].shape), rtol=0, atol=1e-14)
    for j in range(L):
        pre = dataclasses.replace(
            inp, wl=wl.with_(s_q=1, context=j + 1), seq_lens=np.array([j + 1], dtype=np.int32),
            tok_off=np.array([0, j + 1]), c=inp.c[:j + 1], k_rope=inp.k_rope[:j + 1],
            q=inp.q[:, j:j + 1], q_rope=inp.q_rope[:, j:j + 1])
        oj, lj = oracle.decode(pre)
        np.testing.assert_allclose(o[0, j], oj[0, 0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[0, j], lj[0, 0], rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# 7. RoPE: a rotation whose inner products depend on relative position only.
# --------------------------------------------------------------------------
def check_rope_properties():
    rng = np.random.default_rng(2)
    d = 16
    x, y = rng.standard_normal(d), rng.standard_normal(d)
    for m, n, delta in ((0, 0, 5), (3, 11, 7), (1000, 17, -900)):
        a = np.dot(oracle.rope(x, m, 1e4), oracle.rope(y, n, 1e4))
        b = np.dot(oracle.rope(x, m + delta, 1e4), oracle.rope(y, n + delta, 1e4))
        assert abs(a - b) < 1e-10
    np.testing.assert_allclose(oracle.rope(x, 0, 1e4), x, rtol=0, atol=0)
    for pos in (1, 7, 4095, 262143):
        np.testing.assert_allclose(oracle.rope(x, pos, 1e4), _rotate_complex(x, pos, 1e4),
                                   rtol=1e-9, atol=1e-9)


# --------------------------------------------------------------------------
# 8. Permuting cached tokens (each keeping its position) changes nothing.
# --------------------------------------------------------------------------
def check_permutation_invariance():
    inp = make_inputs(TINY_MTP)
    b = 1
    o0, lse0 = oracle.decode_sequence(inp, b)
    sl = inp.sequence(b)
    L = sl.stop - sl.start
    perm = np.random.default_rng(8).permutation(L)
    inp.c[sl] = inp.c[sl][perm]
    inp.k_rope[sl] = inp.k_rope[sl][perm]
    o1, lse1 = oracle.decode_sequence(inp, b, key_pos=np.arange(L)[perm])
    np.testing.assert_allclose(o1, o0, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse1, lse0, rtol=1e-12)


# --------------------------------------------------------------------------
# 9. Output up-projection: applying W^UV_h once to the latent output equals
#    attending over the per-token values c_t W^UV_h (GQLA summary, section 2,
#    absorbed route: the up-projection moves to the output side).
# --------------------------------------------------------------------------
def check_up_projection_equals_explicit_values():
    for wl in (TINY, TINY_MTP):
        inp = make_inputs(wl.with_(d_v=3))
        o_lat, _ = oracle.decode(inp)
        got = oracle.up_project(o_lat, inp.w_uv)
        for b in range(wl.batch):
            c = inp.c[inp.sequence(b)].astype(np.float64)
            l = oracle.sequence_logits(inp, b)                       # [s_q, H, L]
            p = np.exp(l - l.max(-1, keepdims=True))
            p /= p.sum(-1, keepdims=True)
            for h in range(wl.heads):
                v = c @ inp.w_uv[h].astype(np.float64)                 # values materialised per token
                np.testing.assert_allclose(got[b, :, h], p[:, h] @ v, rtol=1e-11, atol=1e-13)


def check_up_projection_selectors():
    """W^UV_h picking latent columns (a column selection of the identity) returns exactly those columns."""
    rng = np.random.default_rng(12)
    H, r, d_v = 3, 7, 4
    o = rng.standard_normal((2, 5, H, r))
    w = np.zeros((H, r, d_v))
    cols = [rng.permutation(r)[:d_v] for _ in range(H)]
    for h in range(H):
        w[h, cols[h], np.arange(d_v)] = 1.0
    got = oracle.up_project(o, w)
    for h in range(H):
        assert np.array_equal(got[:, :, h], o[:, :, h][..., cols[h]])


# --------------------------------------------------------------------------
# 10. The GQA route (GQLA summary, section 2, "Ruta GQA"): keys and values
#     expanded per group, grouped-query attention over them.  Sparse GQLA
#     ("GQLA Disperso"): each (query token, group) attends to a token list.
# --------------------------------------------------------------------------
TINY_GQLA = Workload("pin_gqla", batch=2, s_q=2, heads=6, groups=2, r_kv=8, d_h=4, d_rope=4,
                     context=(5, 19), paged=True, dtype="f32", seed=13, d_v=3, tied_groups=True)


def check_gqa_route_equals_absorbed_route():
    """With one key and one value head per group, the two routes over the same weights agree
    (GQLA summary, section 2: two algebraically equivalent decode routes over the same parameters)."""
    for wl in (TINY_GQLA, TINY_GQLA.with_(s_q=1, seed=14)):
        inp = make_inputs(wl)
        o_gqa, lse_gqa = oracle.gqa_decode(inp, *inp.group_weights())
        o_lat, lse = oracle.decode(inp)
        np.testing.assert_allclose(o_gqa, oracle.up_project(o_lat, inp.w_uv), rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(lse_gqa, lse, rtol=1e-12, atol=1e-12)


def _gqa_group_weights(wl, seed):
    rng = np.random.default_rng(seed)
    w_uk = rng.standard_normal((wl.groups, wl.r_kv, wl.d_h)) / math.sqrt(wl.r_kv)
    gamma_k = 1.0 + 0.1 * rng.standard_normal((wl.groups, wl.d_h))
    w_uv = rng.standard_normal((wl.groups, wl.r_kv, wl.d_v)) / math.sqrt(wl.r_kv)
    return w_uk, gamma_k, w_uv


def check_gqa_against_library_attention():
    """torch fp64 grouped-query scaled_dot_product_attention on keys and values this check forms."""
    wl = TINY_GQLA.with_(tied_groups=False, seed=15)
    inp = make_inputs(wl)
    w_uk, gamma_k, w_uv = _gqa_group_weights(wl, 16)
    o_ref, lse_ref = oracle.gqa_decode(inp, w_uk, gamma_k, w_uv)
    sigma = 1.0 / math.sqrt(wl.d_h + wl.d_rope)
    for b in range(wl.batch):
        sl = inp.sequence(b)
        c = torch.tensor(inp.c[sl], dtype=torch.float64)
        L = c.shape[0]
        z = torch.einsum("tr,grd->gtd", c, torch.tensor(w_uk))
        k = z / torch.sqrt((z * z).mean(-1, keepdim=True) + wl.eps) * torch.tensor(gamma_k)[:, None, :]
        v = torch.einsum("tr,grd->gtd", c, torch.tensor(w_uv))
        krs = inp.k_rope[sl].astype(np.float64)
        kr = torch.tensor(np.stack([_rotate_complex(
            krs[t] * inp.gamma_kr.astype(np.float64) / math.sqrt(float(np.mean(krs[t] ** 2)) + wl.eps),
            t, wl.rope_theta) for t in range(L)]))
        qv = torch.tensor(inp.q[b], dtype=torch.float64)
        qn = qv / torch.sqrt((qv * qv).mean(-1, keepdim=True) + wl.eps) * torch.tensor(inp.gamma_q, dtype=torch.float64)
        qr = np.empty((wl.s_q, wl.heads, wl.d_rope))
        for j in range(wl.s_q):
            for h in range(wl.heads):
                x = inp.q_rope[b, j, h].astype(np.float64)
                qr[j, h] = _rotate_complex(x * inp.gamma_qr[h].astype(np.float64) / math.sqrt(float(np.mean(x * x)) + wl.eps),
                                           L - wl.s_q + j, wl.rope_theta)
        qcat = torch.cat([qn, torch.tensor(qr)], -1).permute(1, 0, 2)                # [H, s_q, d]
        kcat = torch.cat([k, kr.unsqueeze(0).expand(wl.groups, L, wl.d_rope)], -1)  # [g, L, d]
        mask = (torch.arange(L)[None, :] <= (L - wl.s_q + torch.arange(wl.s_q))[:, None])
        out = torch.nn.functional.scaled_dot_product_attention(qcat, kcat, v, attn_mask=mask, scale=sigma,
                                                               enable_gqa=True)     # [H, s_q, d_v]
        np.testing.assert_allclose(o_ref[b], out.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def check_gqa_single_token_returns_value():
    wl = TINY_GQLA.with_(s_q=1, context=1, seed=17)
    inp = make_inputs(wl, seq_lens=[1, 1])
    w_uk, gamma_k, w_uv = _gqa_group_weights(wl, 18)
    o, _ = oracle.gqa_decode(inp, w_uk, gamma_k, w_uv)
    ng = wl.heads // wl.groups
    for b in range(wl.batch):
        c0 = inp.c[inp.sequence(b)][0].astype(np.float64)
        for h in range(wl.heads):
            want = [sum(c0[i] * w_uv[h // ng, i, d] for i in range(wl.r_kv)) for d in range(wl.d_v)]
            np.testing.assert_allclose(o[b, 0, h], want, rtol=1e-12, atol=1e-14)


def check_gqa_sparse_full_selection_equals_dense():
    """Listing every visible token, in any order, is dense attention."""
    inp = make_inputs(TINY_GQLA)
    wts = inp.group_weights()
    sel = make_selection(inp, 32, seed=19)
    o_s, lse_s = oracle.gqa_decode(inp, *wts, selection=sel)
    o_d, lse_d = oracle.gqa_decode(inp, *wts)
    np.testing.assert_allclose(o_s, o_d, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse_s, lse_d, rtol=1e-12, atol=1e-14)
    none = np.full_like(sel, -1)
    o_n, lse_n = oracle.gqa_decode(inp, *wts, selection=none)
    assert (o_n == 0).all() and np.isneginf(lse_n).all()


def check_gqa_sparse_brute_force():
    """Plain Python loops over a three-token selection per (query token, group)."""
    wl = Workload("pin_sparse", batch=1, s_q=2, heads=4, groups=2, r_kv=3, d_h=2, d_rope=2,
                  context=9, paged=False, dtype="f32", eps=0.25, seed=21, d_v=2, tied_groups=True)
    inp = make_inputs(wl)
    w_uk, gamma_k, w_uv = inp.group_weights()
    sel = make_selection(inp, 3, seed=22)
    o, lse = oracle.gqa_decode(inp, w_uk, gamma_k, w_uv, selection=sel)
    L, r, ng = 9, 3, 2
    c = [[float(inp.c[t, i]) for i in range(r)] for t in range(L)]
    sigma = 1.0 / math.sqrt(wl.d_h + wl.d_rope)

    def rmsinv(v):
        return 1.0 / math.sqrt(sum(x * x for x in v) / len(v) + wl.eps)

    def rot(v, pos):   # d = 2: one pair, frequency 1
        return [v[0] * math.cos(pos) - v[1] * math.sin(pos), v[1] * math.cos(pos) + v[0] * math.sin(pos)]

    for j in range(2):
        qpos = L - 2 + j
        for h in range(4):
            g = h // ng
            toks = [int(t) for t in sel[0, j, g] if t >= 0]
            logits, vals = [], []
            for t in toks:
                z = [sum(c[t][i] * float(w_uk[g, i, d]) for i in range(r)) for d in range(2)]
                key = [z[d] * rmsinv(z) * float(gamma_k[g, d]) for d in range(2)]
                qv = [float(x) for x in inp.q[0, j, h]]
                qn = [qv[d] * rmsinv(qv) * float(inp.gamma_q[h, d]) for d in range(2)]
                kr = [float(x) for x in inp.k_rope[t]]
                krn = rot([kr[d] * rmsinv(kr) * float(inp.gamma_kr[d]) for d in range(2)], t)
                qr = [float(x) for x in inp.q_rope[0, j, h]]
                qrn = rot([qr[d] * rmsinv(qr) * float(inp.gamma_qr[h, d]) for d in range(2)], qpos)
                logits.append(sigma * (sum(a * b for a, b in zip(qn, key)) + sum(a * b for a, b in zip(qrn, krn))))
                vals.append([sum(c[t][i] * float(w_uv[g, i, d]) for i in range(r)) for d in range(2)])
            mx = max(logits)
            ex = [math.exp(x - mx) for x in logits]
            s = sum(ex)
            want = [sum(ex[n] / s * vals[n][d] for n in range(len(toks))) for d in range(2)]
            np.testing.assert_allclose(o[0, j, h], want, rtol=1e-12, atol=1e-14)
            assert abs(lse[0, j, h] - (mx + math.log(s))) < 1e-12


ALL_CHECKS = [
    check_absorbed_query_exact,
    check_absorbed_query_row_scale,
    check_absorbed_logits_match,
    check_key_inv_rms_gram,
    check_latent_scale_invariance,
    check_softmax_rows_sum_to_one,
    check_single_token_returns_latent,
    check_zero_query_is_uniform_mean,
    check_identical_tokens_return_that_token,
    check_against_library_attention,
    check_brute_force_causal,
    check_prefill_rows_are_prefix_decodes,
    check_rope_properties,
    check_permutation_invariance,
    check_up_projection_equals_explicit_values,
    check_up_projection_selectors,
    check_gqa_route_equals_absorbed_route,
    check_gqa_against_library_attention,
    check_gqa_single_token_returns_value,
    check_gqa_sparse_full_selection_equals_dense,
    check_gqa_sparse_brute_force,
]
