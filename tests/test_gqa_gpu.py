"""The GQA route of GQLA on the GPU: the expanded cache and the dense and sparse decode (GPU).

qkn_gqa_append expands every token into per-group normalised keys, values and the shared RoPE
key; qkn_gqa_decode runs grouped-query attention over them ("GQLA", section 2, "Ruta GQA"), or,
with a selection, over each (query token, group) pair's listed tokens ("GQLA Disperso").  Both
are compared with the oracle (oracle.group_keys / group_values / rope_keys, oracle.gqa_decode)
element by element under the decode's bf16 tolerances (relative to max |o_v|), on cases that
span 16- and 32-row tiles with padding rows, several row tiles per group, one and two query
tokens, both head widths the kernels take, ragged last pages, many splits of one long sequence,
list lengths that leave a ragged last chunk, and the degenerate cases (length s_q, an empty
list, a rejected length, a block id outside the pool).  The route also matches the library's
absorbed route over the same group-tied weights.
"""
import numpy as np
import pytest
import torch

import oracle
import qk_normed_latent_qkn_b200 as qkn
from gpu_common import LSE_TOL, REL_TOL
from qk_normed_latent_qkn_b200.session import gqa_session_from_inputs, session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs, make_selection

pytestmark = pytest.mark.gpu

GQLA = WORKLOADS["gqla_gqa_bf16"]

CASES = {
    # h_q = 128, g = 8, two query tokens: 32-row tiles, one per group
    "gqla_mtp": GQLA.with_(batch=3, context=(100, 700), seed=101),
    # one query token: 16-row tiles
    "gqla_sq1": GQLA.with_(batch=4, s_q=1, context=(65, 900), seed=102),
    # four heads per group, two tokens: 8 rows in a 16-row tile (8 padding rows)
    "ng4": GQLA.with_(batch=3, heads=16, groups=4, context=(64, 300), seed=103),
    # 24 heads per group, two tokens: 48 rows in two 32-row tiles (16 padding rows in the second)
    "ng24": GQLA.with_(batch=2, heads=48, groups=2, context=(129, 513), seed=104),
    # the narrow head widths
    "narrow": GQLA.with_(batch=3, heads=32, groups=2, d_h=64, d_rope=32, d_v=64, context=(70, 400), seed=105),
    # one long sequence: every CTA of the schedule works on it (many splits per row tile)
    "long": GQLA.with_(batch=1, context=30000, seed=106),
}


def _np(x):
    return x.float().cpu().numpy().astype(np.float64)


def _assert_close(o, lse, o_ref, lse_ref, dtype="bf16", what=""):
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    scale = np.abs(o_ref).max()
    err = np.abs(o - o_ref).max()
    tol = REL_TOL[dtype] * scale
    assert err <= tol, f"{what}: max|o_v - o_v_ref| = {err:.3e} > {tol:.3e} (max|o_v_ref| = {scale:.3e})"
    fin = np.isfinite(lse_ref)
    assert (np.isneginf(lse) == ~fin).all(), f"{what}: rows without a token differ"
    if fin.any():
        lerr = np.abs(lse[fin] - lse_ref[fin]).max()
        assert lerr <= LSE_TOL[dtype], f"{what}: max|lse - lse_ref| = {lerr:.3e}"


def _run(inp, selection=None, max_ctas=0, session=None):
    s = session if session is not None else gqa_session_from_inputs(inp)
    o_v, lse = s.decode(inp.block_table, inp.seq_lens, inp.wl.s_q, selection=selection, max_ctas=max_ctas)
    torch.cuda.synchronize()
    return s, _np(o_v), lse.cpu().numpy().astype(np.float64)


def _oracle(inp, seqs=None, selection=None):
    o, lse = oracle.gqa_decode(inp, *inp.group_weights(), seqs=seqs, selection=selection)
    sel = list(range(inp.wl.batch)) if seqs is None else list(seqs)
    return o[sel], lse[sel], sel


@pytest.mark.parametrize("name", sorted(CASES))
def test_dense_matches_oracle(name):
    inp = make_inputs(CASES[name])
    s, o, lse = _run(inp)
    assert s.device_status() == qkn.OK
    o_ref, lse_ref, sel = _oracle(inp)
    _assert_close(o[sel], lse[sel], o_ref, lse_ref, what=name)


def test_append_matches_oracle():
    # the expanded cache itself: keys, values and RoPE keys of every token at its slot
    inp = make_inputs(CASES["gqla_mtp"])
    s = gqa_session_from_inputs(inp)
    torch.cuda.synchronize()
    w_uk, gamma_k, w_uv = inp.group_weights()
    slots = inp.token_slots()
    blk, off = slots // 64, slots % 64
    k = _np(s.cache.k)[blk, :, off]                       # [T, g, d_h]
    v = _np(s.cache.v)[blk, :, off]
    kr = _np(s.cache.k_rope)[blk, off]
    wl = inp.wl
    k_ref = oracle.group_keys(inp.c, w_uk, gamma_k, wl.eps)
    v_ref = oracle.group_values(inp.c, w_uv)
    kr_ref = oracle.rope_keys(inp.k_rope, inp.gamma_kr, inp.token_positions(), wl.eps, wl.rope_theta)
    for got, ref, what in ((k, k_ref, "keys"), (v, v_ref, "values"), (kr, kr_ref, "RoPE keys")):
        # one bf16 rounding of the stored value: 2^-8 relative, plus fp32 products
        np.testing.assert_allclose(got, ref, rtol=8e-3, atol=8e-3 * np.abs(ref).max(), err_msg=what)


@pytest.mark.parametrize("max_ctas", [1, 7, 37])
def test_cta_counts(max_ctas):
    # fewer CTAs than row tiles, an odd count, and several groups of CTAs: the schedule's splits
    inp = make_inputs(CASES["gqla_mtp"])
    s, o, lse = _run(inp, max_ctas=max_ctas)
    assert s.device_status() == qkn.OK
    o_ref, lse_ref, _ = _oracle(inp)
    _assert_close(o, lse, o_ref, lse_ref, what=f"max_ctas={max_ctas}")


def test_boundary_lengths():
    # lengths around page edges, the shortest (s_q) and a sequence of one page
    lens = [2, 3, 63, 64, 65, 127, 128, 129]
    inp = make_inputs(GQLA.with_(batch=len(lens), context=(2, 200), seed=107), seq_lens=lens)
    s, o, lse = _run(inp)
    assert s.device_status() == qkn.OK
    o_ref, lse_ref, _ = _oracle(inp)
    _assert_close(o, lse, o_ref, lse_ref, what="boundary lengths")


def test_route_matches_absorbed_route():
    # over the same group-tied weights the two routes are algebraically equal (GQLA section 2): the
    # GQA decode against the library's absorbed decode with the fused value up-projection
    inp = make_inputs(CASES["gqla_mtp"])
    _, o, lse = _run(inp)
    a = session_from_inputs(inp)
    o_abs, lse_abs = a.decode_up(inp.block_table, inp.seq_lens, inp.wl.s_q)
    torch.cuda.synchronize()
    o_abs = _np(o_abs)
    assert np.abs(o - o_abs).max() <= 2e-2 * np.abs(o_abs).max()
    assert np.abs(lse - lse_abs.cpu().numpy()).max() <= 4e-2


@pytest.mark.parametrize("k", [1, 64, 100, 300])
def test_sparse_matches_oracle(k):
    # list lengths of one token, one whole chunk, a ragged second chunk and five chunks; short
    # sequences give lists padded with -1
    inp = make_inputs(GQLA.with_(batch=3, context=(120, 700), seed=108))
    sel = make_selection(inp, k, seed=109)
    s, o, lse = _run(inp, selection=sel)
    assert s.device_status() == qkn.OK
    o_ref, lse_ref, _ = _oracle(inp, selection=sel)
    _assert_close(o, lse, o_ref, lse_ref, what=f"sparse k={k}")


def test_sparse_one_token_rows_and_narrow_heads():
    inp = make_inputs(CASES["narrow"].with_(s_q=1))
    sel = make_selection(inp, 80, seed=110)
    s, o, lse = _run(inp, selection=sel)
    assert s.device_status() == qkn.OK
    o_ref, lse_ref, _ = _oracle(inp, selection=sel)
    _assert_close(o, lse, o_ref, lse_ref, what="sparse narrow")


def test_sparse_full_lists_equal_dense():
    # listing every visible token is dense attention (up to the order of the sums)
    inp = make_inputs(GQLA.with_(batch=2, context=(150, 400), seed=111))
    sel = make_selection(inp, 512, seed=112)
    s, o_s, lse_s = _run(inp, selection=sel)
    _, o_d, lse_d = _run(inp, session=s)
    assert np.abs(o_s - o_d).max() <= 1e-2 * np.abs(o_d).max()
    assert np.abs(lse_s - lse_d).max() <= 1e-3


def test_sparse_empty_and_invisible_entries():
    # an empty list gives zeros and lse = -inf; entries after the query's position are not attended
    inp = make_inputs(GQLA.with_(batch=2, context=(200, 300), seed=113))
    sel = make_selection(inp, 16, seed=114)
    sel[0, :, 3] = -1                                     # group 3 of sequence 0: nothing listed
    L1 = int(inp.seq_lens[1])
    sel[1, 0, 5, :4] = [L1 - 1, L1 + 7, 10 ** 6, L1 - 1]  # query 0 sits at L - 2: all four invisible
    s, o, lse = _run(inp, selection=sel)
    assert s.device_status() == qkn.OK
    o_ref, lse_ref, _ = _oracle(inp, selection=sel)
    ng = inp.wl.heads_per_group
    assert (o[0][:, 3 * ng:4 * ng] == 0).all() and np.isneginf(lse[0][:, 3 * ng:4 * ng]).all()
    _assert_close(o, lse, o_ref, lse_ref, what="sparse with empty and invisible entries")


def test_rejected_length_and_bad_block_are_recorded():
    inp = make_inputs(CASES["gqla_mtp"])
    s = gqa_session_from_inputs(inp)
    sl = inp.seq_lens.copy()
    sl[1] = inp.block_table.shape[1] * 64 + 1            # past the block table
    o_v, lse = s.decode(inp.block_table, sl, inp.wl.s_q)
    torch.cuda.synchronize()
    assert s.device_status() == qkn.ERR_BOUNDS
    o, lse = _np(o_v), lse.cpu().numpy().astype(np.float64)
    assert (o[1] == 0).all() and np.isneginf(lse[1]).all()
    o_ref, lse_ref, sel = _oracle(inp, seqs=[0, 2])
    _assert_close(o[sel], lse[sel], o_ref, lse_ref, what="other sequences")
    # sparse, the same rejected length
    s.clear_status()
    sel_tok = make_selection(inp, 32, seed=115)
    o_v, lse = s.decode(inp.block_table, sl, inp.wl.s_q, selection=sel_tok)
    torch.cuda.synchronize()
    assert s.device_status() == qkn.ERR_BOUNDS
    assert (_np(o_v)[1] == 0).all() and np.isneginf(lse.cpu().numpy()[1]).all()
    # a block id outside the pool is read as block 0 and recorded, without a fault
    s.clear_status()
    bt = inp.block_table.copy()
    bt[0, 0] = inp.num_blocks + 5
    o_v, lse = s.decode(bt, inp.seq_lens, inp.wl.s_q)
    torch.cuda.synchronize()
    assert s.device_status() == qkn.ERR_BOUNDS
    assert np.isfinite(_np(o_v)).all()


def test_append_skips_slots_outside_the_pool():
    # tokens whose slot ids lie outside the pool write nothing: every byte of the three caches is
    # unchanged (compared as bit patterns, since slots no append has written may hold NaN patterns)
    inp = make_inputs(CASES["ng4"])
    s = gqa_session_from_inputs(inp)
    caches = (s.cache.k, s.cache.v, s.cache.k_rope)
    before = [x.view(torch.int16).clone() for x in caches]
    n = 5
    slots = np.array([-1, inp.num_blocks * 64, inp.num_blocks * 64 + 100, -64, 2 ** 31 - 1], dtype=np.int32)
    s.append(inp.c[:n], inp.k_rope[:n], slots, np.arange(n, dtype=np.int32))
    torch.cuda.synchronize()
    for b, a in zip(before, caches):
        assert torch.equal(b, a.view(torch.int16))


def test_full_size_workload_sampled():
    # the GQLA configuration at full size (32 sequences up to 32k tokens, 8 groups of 16 heads,
    # two query tokens), in the launch configuration of the benchmark, against the oracle on the
    # shortest, a middle and the longest sequence
    inp = make_inputs("gqla_gqa_bf16")
    s, o, lse = _run(inp)
    assert s.device_status() == qkn.OK
    order = np.argsort(inp.seq_lens)
    sample = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    o_ref, lse_ref, sel = _oracle(inp, seqs=sample)
    _assert_close(o[sel], lse[sel], o_ref, lse_ref, what="gqla_gqa_bf16 full size")
