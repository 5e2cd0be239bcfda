"""Context-parallel decode on the GPU, ranks emulated in one process (GPU).

Each rank's page slices are decoded by the library with the causal limit's
end passed as qkn_decode_opts.vis_end, the ranks' partial results are
stacked (the all-gather on one GPU) and merged by qkn_merge_partials; the
result is compared with the oracle's decode of the whole sequences under the
decode's tolerances.  Covers s_q = 1 and s_q = 2 with four groups (where
vis_end decides which of a slice's tokens the queries see), the tcgen05,
CTA-pair and CUDA-core decodes, 2 to 4 ranks, and the merge kernel alone on
random partials against its definition."""
import numpy as np
import pytest
import torch

import qk_normed_latent_qkn_b200 as qkn
from gpu_common import assert_close_to_oracle
from qk_normed_latent_qkn_b200 import context_parallel as cp
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "large_mla_bf16": WORKLOADS["large_mla_bf16"].with_(batch=5, context=(600, 2500), seed=91),
    "grouped_mtp_bf16": WORKLOADS["grouped_mtp_bf16"].with_(batch=3, context=(600, 1800), seed=92),
    "long_ctx_bf16": WORKLOADS["long_ctx_bf16"].with_(batch=1, context=30000, seed=93),
    "small_mla_bf16": WORKLOADS["small_mla_bf16"].with_(batch=4, context=1100, seed=94),
}


def _cp_decode(s, inp, world, **kw):
    outs, lses = [], []
    for r in range(world):
        o, l = cp.slice_decode(s, inp.block_table, inp.seq_lens, inp.wl.s_q, r, world, **kw)
        outs.append(o.clone())
        lses.append(l.clone())
    torch.cuda.synchronize()
    assert s.device_status() == qkn.OK
    out, lse = cp.merge(s.dims, torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("world", [2, 4])
def test_context_parallel_matches_oracle(name, world):
    inp = make_inputs(CASES[name])
    s = session_from_inputs(inp)
    o, lse = _cp_decode(s, inp, world)
    assert_close_to_oracle(inp, o, lse, what=f"{name} over {world} ranks")


@pytest.mark.parametrize("kw", [dict(head_tile=128), dict(kernel=qkn.KERNEL_SIMT)], ids=["pair", "simt"])
def test_context_parallel_other_kernels(kw):
    inp = make_inputs(CASES["grouped_mtp_bf16"])
    s = session_from_inputs(inp)
    o, lse = _cp_decode(s, inp, 3, **kw)
    assert_close_to_oracle(inp, o, lse, what=f"grouped over 3 ranks, {kw}")


def test_vis_end_is_what_keeps_the_limit():
    # a slice that does not hold the sequence's end: without vis_end the decode would take its last
    # tokens for this step's and hide them from the first query; with it they are visible
    inp = make_inputs(CASES["grouped_mtp_bf16"])
    s = session_from_inputs(inp)
    bt, lens, vis_end = cp.rank_view(inp.block_table, inp.seq_lens, 0, 2)
    o1, l1 = s.decode(bt, lens, 2, vis_end=vis_end)
    o0, l0 = s.decode(bt, lens, 2)
    torch.cuda.synchronize()
    # query 0 sees every token of a leading slice with vis_end, one fewer without it
    assert not torch.equal(l1[:, 0], l0[:, 0])
    assert torch.equal(l1[:, 1], l0[:, 1]) or torch.allclose(l1[:, 1], l0[:, 1], atol=1e-6)


def test_merge_kernel_against_its_definition():
    rng = np.random.default_rng(5)
    dims = qkn.Dims(num_heads=8, num_groups=1, r_kv=512, d_h=128, d_rope=64)
    P, rows = 5, 37
    parts = rng.standard_normal((P, rows, 512)).astype(np.float32)
    lses = rng.normal(3.0, 4.0, size=(P, rows)).astype(np.float32)
    lses[1, :5] = -np.inf                                  # parts that saw nothing of some rows
    lses[:, 7] = -np.inf                                   # a row no part saw
    pt = torch.from_numpy(parts).to("cuda", torch.bfloat16)
    lt = torch.from_numpy(lses).to("cuda")
    out = torch.empty((rows, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
    qkn.merge_partials(dims, pt, lt, out, lse)
    torch.cuda.synchronize()
    p64 = pt.float().cpu().numpy().astype(np.float64)
    l64 = lses.astype(np.float64)
    m = l64.max(axis=0)
    ok = np.isfinite(m)
    w = np.where(ok[None], np.exp(l64 - np.where(ok, m, 0)[None]), 0.0)
    den = w.sum(axis=0)
    ref = np.where(ok[:, None], (w[..., None] * p64).sum(axis=0) / np.where(ok, den, 1)[:, None], 0.0)
    lref = np.where(ok, m + np.log(np.where(ok, den, 1)), -np.inf)
    o = out.float().cpu().numpy()
    assert np.abs(o - ref).max() <= 1e-2 * np.abs(ref).max()
    assert (o[7] == 0).all() and np.isneginf(lse.cpu().numpy()[7])
    lg = lse.cpu().numpy()
    assert np.abs(lg[ok] - lref[ok]).max() <= 1e-4


def test_context_parallel_over_a_prefill_chunk():
    # 200 new tokens per sequence after a history, over 2 ranks: the decode skips each row tile's
    # invisible pages counting from vis_end, and whole segments go straight to each rank's output
    inp = make_inputs(WORKLOADS["prefill_mla_bf16"].with_(batch=2, s_q=200, context=(900, 1500), seed=95))
    s = session_from_inputs(inp)
    o, lse = _cp_decode(s, inp, 2)
    assert_close_to_oracle(inp, o, lse, what="prefill chunk over 2 ranks")
