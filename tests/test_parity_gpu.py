"""CUDA path vs the fp64 oracle, element by element, through the C ABI (GPU)."""
import numpy as np
import pytest
import torch

import oracle
import qk_normed_latent_qkn_b200 as qkn
from gpu_common import assert_close_to_oracle, run_decode
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# Reduced-context versions of the workloads: same heads, groups, widths and
# value recipe, contexts short enough for the oracle yet spanning several
# 64-token pages and 128-token tiles with ragged tails.
SMALL = {
    "tiny_f32": WORKLOADS["tiny_f32"],
    "tiny_f32_ragged": WORKLOADS["tiny_f32"].with_(batch=3, context=(1, 300), paged=True, seed=5),
    "small_mla_bf16": WORKLOADS["small_mla_bf16"].with_(batch=4, context=700, seed=1),
    "large_mla_bf16": WORKLOADS["large_mla_bf16"].with_(batch=3, context=(200, 900), seed=2),
    "long_ctx_bf16": WORKLOADS["long_ctx_bf16"].with_(context=1537, seed=3),
    "grouped_mtp_bf16": WORKLOADS["grouped_mtp_bf16"].with_(batch=3, context=(130, 700), seed=4),
}

KERNELS = {"simt": qkn.KERNEL_SIMT, "auto": qkn.KERNEL_AUTO, "tcgen05": qkn.KERNEL_TCGEN05}


def _skip_if_fp32_tc(wl, kernel):
    if kernel == "tcgen05" and wl.dtype != "bf16":
        pytest.skip("the tensor-core kernel takes bf16 storage only")


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_decode_matches_oracle(name, kernel):
    _skip_if_fp32_tc(SMALL[name], kernel)
    inp = make_inputs(SMALL[name])
    _, o, lse = run_decode(inp, kernel=KERNELS[kernel])
    assert_close_to_oracle(inp, o, lse, what=f"{name}/{kernel}")


def test_append_unit_parity():
    for name in ("tiny_f32_ragged", "grouped_mtp_bf16"):
        inp = make_inputs(SMALL[name])
        s = session_from_inputs(inp)
        torch.cuda.synchronize()
        slots = inp.token_slots()
        bs = inp.wl.block_size
        a_k = s.cache.a_k.cpu().numpy().reshape(-1, inp.wl.groups)[slots]
        ref = oracle.key_inv_rms(inp.c, inp.w_k, inp.wl.eps)
        np.testing.assert_allclose(a_k, ref, rtol=2e-5)
        lat = s.cache.latent.float().cpu().numpy().reshape(-1, inp.wl.r_kv)[slots]
        assert np.array_equal(lat, inp.c)                   # copied bit for bit
        kr = s.cache.k_rope.float().cpu().numpy().reshape(-1, inp.wl.d_rope)[slots]
        kref = oracle.rope_keys(inp.k_rope, inp.gamma_kr, inp.token_positions(), inp.wl.eps, inp.wl.rope_theta)
        tol = 1e-5 if inp.wl.dtype == "f32" else 2 ** -8
        assert np.abs(kr - kref).max() <= tol * max(1.0, np.abs(kref).max())
        del bs


def test_absorb_unit_parity():
    for name in ("tiny_f32", "grouped_mtp_bf16"):
        inp = make_inputs(SMALL[name])
        wl = inp.wl
        s = session_from_inputs(inp)
        torch.cuda.synchronize()
        B, s_q, H = wl.batch, wl.s_q, wl.heads
        q = inp.q.reshape(B * s_q, H, wl.d_h)
        qt_ref, aq_ref = oracle.absorbed_query(q, inp.w_k, inp.gamma_q, inp.gamma_k, wl.eps, wl.softmax_scale)
        qt = s.q_tilde.float().cpu().numpy()
        aq = s.a_q.cpu().numpy()
        rel = 1e-5 if wl.dtype == "f32" else 2 ** -8
        assert np.abs(qt - qt_ref).max() <= rel * np.abs(qt_ref).max() * 2
        np.testing.assert_allclose(aq, aq_ref, rtol=1e-5)
        pos = inp.query_positions().reshape(-1)
        qr_ref = wl.softmax_scale * oracle.rope(
            oracle.rms_norm(inp.q_rope.reshape(B * s_q, H, wl.d_rope), inp.gamma_qr, wl.eps), pos[:, None],
            wl.rope_theta)
        qr = s.q_rope_hat.float().cpu().numpy()
        assert np.abs(qr - qr_ref).max() <= rel * np.abs(qr_ref).max() * 2


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_page_boundaries(kernel):
    # lengths at, just below and just above page and tile edges, and L = s_q
    wl = WORKLOADS["grouped_mtp_bf16"].with_(batch=8, heads=16, groups=4, seed=7)
    inp = make_inputs(wl, seq_lens=[2, 63, 64, 65, 127, 128, 129, 257])
    _, o, lse = run_decode(inp, kernel=KERNELS[kernel])
    assert_close_to_oracle(inp, o, lse, what=f"boundaries/{kernel}")


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_split_count_and_determinism(kernel):
    inp = make_inputs(SMALL["large_mla_bf16"])
    s, o_many, _ = run_decode(inp, kernel=KERNELS[kernel])
    _, o_many2, _ = run_decode(inp, kernel=KERNELS[kernel], session=s)
    assert np.array_equal(o_many, o_many2)                  # same split plan -> same bits
    _, o_one, lse_one = run_decode(inp, kernel=KERNELS[kernel], max_ctas=1, session=s)
    assert_close_to_oracle(inp, o_one, lse_one, what="one split")
    scale = np.abs(o_one).max()
    assert np.abs(o_many - o_one).max() <= 1e-2 * scale


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_identity_table_equals_random_table(kernel):
    wl = SMALL["large_mla_bf16"]
    paged = make_inputs(wl)
    flat = make_inputs(wl.with_(paged=False))
    _, o1, l1 = run_decode(paged, kernel=KERNELS[kernel])
    _, o2, l2 = run_decode(flat, kernel=KERNELS[kernel])
    # qkn_append accumulates sum(z^2) with fp32 atomics, so the two caches may differ in the
    # last bit of a_k, which can move a bf16 output by one unit in the last place (2^-8 relative)
    assert np.abs(o1 - o2).max() <= 2 ** -7 * np.abs(o1).max()
    assert np.abs(l1 - l2).max() <= 1e-3


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_plain_mla_mode_matches_oracle_with_unit_key_scale(kernel):
    # a_k == 1 everywhere: compare against the oracle with the a_k cache forced to 1, which is the
    # explicit form with keys c W^K_g * gamma_k (no key RMS): emulate by rescaling W so that every
    # token's key RMS is ~1 is not exact, so instead check a_k = 1 against a direct fp64 evaluation.
    inp = make_inputs(SMALL["small_mla_bf16"].with_(batch=2, context=300))
    s, o, lse = run_decode(inp, kernel=KERNELS[kernel], ak_mode=qkn.AK_ONE)
    wl = inp.wl
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
            l = aq[i][:, None] * (qt[i] @ c.T) + qr[j] @ kr.T        # [H, L]
            l -= l.max(-1, keepdims=True)
            p = np.exp(l)
            p /= p.sum(-1, keepdims=True)
            ref = p @ c
            assert np.abs(o[b, j] - ref).max() <= 1e-2 * np.abs(ref).max()


def test_bad_sequence_length_is_reported_not_faulted():
    inp = make_inputs(SMALL["small_mla_bf16"].with_(batch=2, context=200))
    s = session_from_inputs(inp)
    lens = inp.seq_lens.copy()
    lens[1] = inp.max_blocks * 64 + 5           # beyond the block table
    out, lse = s.decode(inp.block_table, lens, 1)
    assert s.device_status() == qkn.ERR_BOUNDS
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    s.clear_status()
    assert s.device_status() == qkn.OK


@pytest.mark.parametrize("kernel,max_ctas", [("tcgen05", 1), ("tcgen05", 3), ("tcgen05", 7), ("simt", 5), ("simt", 1)])
def test_cta_group_edges(kernel, max_ctas):
    # 128 heads: two 64-row tiles per sequence on the tensor cores (groups of two CTAs; an odd CTA
    # count leaves one idle, one CTA takes both tiles of every sequence), sixteen 8-row tiles on the
    # CUDA cores (five CTAs form one group, each taking every fifth tile of the same pages)
    inp = make_inputs(SMALL["large_mla_bf16"])
    s, o, lse = run_decode(inp, kernel=KERNELS[kernel], max_ctas=max_ctas)
    assert_close_to_oracle(inp, o, lse, what=f"{kernel}, {max_ctas} CTAs")
    _, o_all, _ = run_decode(inp, kernel=KERNELS[kernel], session=s)
    assert np.abs(o - o_all).max() <= 1e-2 * np.abs(o_all).max()
