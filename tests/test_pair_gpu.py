"""The CTA-pair decode (tiles of 128 query rows, latent split across the two
CTAs of a cluster) against the fp64 oracle, through the C ABI (GPU).

The kernel is taken when a caller asks for 128-row tiles (head_tile = 128);
these cases pin its edges: page and tile boundaries with two query tokens and
four KV groups, row counts that leave padding rows in a tile (96 rows, and
160 rows = one full and one partial tile), plain-MLA mode (whose unnormalised
logits make the output rescale on many pages), and agreement with the
single-CTA kernel on 64-row tiles.
"""
import numpy as np
import pytest

import oracle
import qk_normed_latent_qkn_b200 as qkn
from gpu_common import assert_close_to_oracle, run_decode
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

PAIR = 128


@pytest.mark.parametrize("name", ["large_mla_bf16", "long_ctx_bf16", "grouped_mtp_bf16"])
def test_pair_and_single_cta_tiles_match_oracle(name):
    base = WORKLOADS[name]
    wl = {"large_mla_bf16": base.with_(batch=3, context=(200, 900), seed=41),
          "long_ctx_bf16": base.with_(context=2113, seed=42),
          "grouped_mtp_bf16": base.with_(batch=3, context=(130, 700), seed=43)}[name]
    inp = make_inputs(wl)
    s, o_pair, l_pair = run_decode(inp, kernel=qkn.KERNEL_TCGEN05, head_tile=PAIR)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o_pair, l_pair, what=f"{name}/pair")
    _, o_one, l_one = run_decode(inp, kernel=qkn.KERNEL_TCGEN05, head_tile=64, session=s)
    assert_close_to_oracle(inp, o_one, l_one, what=f"{name}/64-row tiles")
    assert np.abs(o_pair - o_one).max() <= 1e-2 * np.abs(o_one).max()


def test_pair_page_boundaries_two_tokens_four_groups():
    # 64 heads x 2 query tokens = one 128-row tile; lengths at and around page edges, and L = s_q
    wl = WORKLOADS["grouped_mtp_bf16"].with_(batch=8, seed=44)
    inp = make_inputs(wl, seq_lens=[2, 63, 64, 65, 127, 128, 129, 257])
    s, o, lse = run_decode(inp, kernel=qkn.KERNEL_TCGEN05, head_tile=PAIR)
    assert qkn.decode_kernel_for(s.dims, wl.s_q, head_tile=PAIR) == qkn.KERNEL_TCGEN05
    assert_close_to_oracle(inp, o, lse, what="pair boundaries")


@pytest.mark.parametrize("heads,s_q", [(96, 1), (80, 2)])
def test_pair_tiles_with_padding_rows(heads, s_q):
    # 96 rows: one tile with 32 padding rows; 160 rows: a full tile and one with 32 valid rows
    wl = WORKLOADS["large_mla_bf16"].with_(batch=3, heads=heads, s_q=s_q, context=(150, 700), seed=45 + heads)
    inp = make_inputs(wl)
    s, o, lse = run_decode(inp, kernel=qkn.KERNEL_TCGEN05, head_tile=PAIR)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o, lse, what=f"{heads} heads x {s_q}")


@pytest.mark.parametrize("context", [(300, 500), (1500, 4000)])
def test_pair_plain_mla_mode(context):
    # a_k treated as 1: against a direct fp64 evaluation of the absorbed logits without the key scale.
    # Without the key normalisation the logits are large and their row maxima keep rising along the
    # context, so the output accumulator is rescaled row by row on many pages: this covers the
    # rescale path with rows of one warp changing and others not.
    wl = WORKLOADS["large_mla_bf16"].with_(batch=2, context=context, seed=47)
    inp = make_inputs(wl)
    s, o, _ = run_decode(inp, kernel=qkn.KERNEL_TCGEN05, head_tile=PAIR, ak_mode=qkn.AK_ONE)
    q = inp.q.reshape(wl.batch * wl.s_q, wl.heads, wl.d_h)
    qt, aq = oracle.absorbed_query(q, inp.w_k, inp.gamma_q, inp.gamma_k, wl.eps, wl.softmax_scale)
    for b in range(wl.batch):
        sl = inp.sequence(b)
        c = inp.c[sl].astype(np.float64)
        L = c.shape[0]
        kr = oracle.rope_keys(inp.k_rope[sl], inp.gamma_kr, np.arange(L), wl.eps, wl.rope_theta)
        qr = wl.softmax_scale * oracle.rope(oracle.rms_norm(inp.q_rope[b], inp.gamma_qr, wl.eps),
                                            inp.query_positions()[b][:, None], wl.rope_theta)
        for j in range(wl.s_q):
            i = b * wl.s_q + j
            l = aq[i][:, None] * (qt[i] @ c.T) + qr[j] @ kr.T
            l -= l.max(-1, keepdims=True)
            p = np.exp(l)
            p /= p.sum(-1, keepdims=True)
            ref = p @ c
            assert np.abs(o[b, j] - ref).max() <= 1e-2 * np.abs(ref).max()
