"""The decode step with each head's value up-projection fused into the merge (GPU).

qkn_decode_up returns o_v[i, h] = o_lat[i, h] W^UV_h (GQLA summary, section
2, absorbed MQA route) and qkn_decode's lse.  It is compared with the oracle's
up_project(decode(...)) element by element, under the decode's tolerances
(relative to max |o_v|), on cases that span several 32- and 64-row CTAs with a
ragged last one, many splits per row, both split sources (the tcgen05 decode's
segment descriptors and the CUDA-core decode's recomputed schedule), fp32 and
bf16 storage, several value widths, and a sequence with a rejected length.
"""
import numpy as np
import pytest
import torch

import oracle
import qk_normed_latent_qkn_b200 as qkn
from gpu_common import LSE_TOL, REL_TOL
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _run_up(s, inp, **kw):
    o_v, lse = s.decode_up(inp.block_table, inp.seq_lens, inp.wl.s_q, **kw)
    torch.cuda.synchronize()
    return o_v.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _assert_up_close(inp, o_v, lse, seqs=None, what=""):
    o_ref, lse_ref = oracle.decode(inp, seqs=seqs)
    sel = list(range(inp.wl.batch)) if seqs is None else list(seqs)
    ov_ref = oracle.up_project(o_ref[sel], inp.w_uv)
    o_v, lse, lse_ref = o_v[sel], lse[sel], lse_ref[sel]
    assert np.isfinite(o_v).all(), f"{what}: non-finite output"
    scale = np.abs(ov_ref).max()
    err = np.abs(o_v - ov_ref).max()
    tol = REL_TOL[inp.wl.dtype] * scale
    assert err <= tol, f"{what}: max|o_v - o_v_ref| = {err:.3e} > {tol:.3e} (max|o_v_ref| = {scale:.3e})"
    lerr = np.abs(lse - lse_ref).max()
    assert lerr <= LSE_TOL[inp.wl.dtype], f"{what}: max|lse - lse_ref| = {lerr:.3e}"


CASES = {
    # fp32 storage: the CUDA-core decode (schedule-recomputed splits) and the FMA product, d_v = 32
    "tiny_f32": WORKLOADS["tiny_f32"].with_(batch=3, context=(100, 300), seed=71),
    # 4 query rows of 16 heads: one 32-row CTA per head, 28 padding rows
    "small_mla_bf16": WORKLOADS["small_mla_bf16"].with_(batch=4, context=700, seed=72),
    # 40 query rows: 64-row CTAs, 24 padding rows in the second m-tile group
    "large_mla_bf16": WORKLOADS["large_mla_bf16"].with_(batch=40, context=(64, 600), seed=73),
    # s_q = 2 and four groups: query rows i = 2 b + j
    "grouped_mtp_bf16": WORKLOADS["grouped_mtp_bf16"].with_(batch=5, context=(130, 900), seed=74),
    # one long sequence: about one split per CTA for every row (148-way merge)
    "long_ctx_bf16": WORKLOADS["long_ctx_bf16"].with_(batch=1, context=40000, seed=75),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_up_matches_oracle(name):
    inp = make_inputs(CASES[name])
    s = session_from_inputs(inp)
    o_v, lse = _run_up(s, inp)
    assert s.device_status() == qkn.OK
    assert o_v.shape == (inp.wl.batch, inp.wl.s_q, inp.wl.heads, inp.wl.d_v)
    _assert_up_close(inp, o_v, lse, what=name)


@pytest.mark.parametrize("d_v", [16, 48, 176])
def test_value_widths(d_v):
    # an odd number of 16-column pairs per warp pass, and the widest d_v at r = 512
    inp = make_inputs(WORKLOADS["large_mla_bf16"].with_(batch=36, context=(64, 400), d_v=d_v, seed=76))
    s = session_from_inputs(inp)
    o_v, lse = _run_up(s, inp)
    assert s.device_status() == qkn.OK
    _assert_up_close(inp, o_v, lse, what=f"d_v={d_v}")


def test_simt_decode_splits_from_the_schedule():
    # bf16 storage through the CUDA-core decode: the merge recomputes every row's splits
    inp = make_inputs(CASES["small_mla_bf16"])
    s = session_from_inputs(inp)
    o_v, lse = _run_up(s, inp, kernel=qkn.KERNEL_SIMT)
    assert s.device_status() == qkn.OK
    _assert_up_close(inp, o_v, lse, what="simt")


@pytest.mark.parametrize("head_tile", [16, 32, 128])
def test_row_tiles(head_tile):
    # the merge finds a row's partials at the tile and row the decode used
    inp = make_inputs(CASES["grouped_mtp_bf16"])
    s = session_from_inputs(inp)
    o_v, lse = _run_up(s, inp, head_tile=head_tile)
    assert s.device_status() == qkn.OK
    _assert_up_close(inp, o_v, lse, what=f"head_tile={head_tile}")


def test_fused_equals_latent_output_times_w_uv():
    # the fused product against the library's own latent output multiplied by W^UV_h in fp64: both
    # round the merged row to bf16, so they differ only by the merge's summation order and the
    # final rounding
    inp = make_inputs(CASES["large_mla_bf16"])
    s = session_from_inputs(inp)
    o_v, lse_up = _run_up(s, inp)
    out, lse = s.decode(inp.block_table, inp.seq_lens, inp.wl.s_q)
    torch.cuda.synchronize()
    o_lat = out.float().cpu().numpy().astype(np.float64)
    ref = oracle.up_project(o_lat, inp.w_uv)
    assert np.abs(o_v - ref).max() <= 4e-3 * np.abs(ref).max()
    assert np.abs(lse_up - lse.cpu().numpy()).max() <= 1e-5


def test_rejected_length_gives_zero_rows():
    inp = make_inputs(CASES["large_mla_bf16"])
    s = session_from_inputs(inp)
    sl = inp.seq_lens.copy()
    sl[3] = inp.block_table.shape[1] * 64 + 1         # past the block table
    o_v, lse = s.decode_up(inp.block_table, sl, inp.wl.s_q)
    torch.cuda.synchronize()
    assert s.device_status() == qkn.ERR_BOUNDS
    o_v = o_v.float().cpu().numpy()
    lse = lse.cpu().numpy()
    assert (o_v[3] == 0).all() and np.isneginf(lse[3]).all()
    others = [b for b in range(inp.wl.batch) if b != 3]
    _assert_up_close(inp, o_v.astype(np.float64), lse.astype(np.float64), seqs=others, what="other sequences")


def test_full_size_headline_workload_sampled():
    # the 128-head workload at full size, in the launch configuration of the benchmark, against the
    # oracle on a sample of sequences (the shortest, the longest and one between)
    inp = make_inputs("large_mla_bf16")
    s = session_from_inputs(inp)
    o_v, lse = _run_up(s, inp)
    assert s.device_status() == qkn.OK
    order = np.argsort(inp.seq_lens)
    sample = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    _assert_up_close(inp, o_v, lse, seqs=sample, what="large_mla_bf16 full size")


def test_decode_up_after_a_prefill_chunk():
    # long query chunk: the decode's row tiles skip their invisible pages (items that may be empty
    # write zero partials with lse = -inf) and the fused merge applies W^UV to the merged rows
    inp = make_inputs(WORKLOADS["prefill_mla_bf16"].with_(batch=2, s_q=150, context=(300, 700), seed=77))
    s = session_from_inputs(inp)
    o_v, lse = _run_up(s, inp)
    assert s.device_status() == qkn.OK
    _assert_up_close(inp, o_v, lse, what="prefill chunk")
