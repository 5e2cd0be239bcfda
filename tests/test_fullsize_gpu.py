"""The five decode workloads at their full sizes, in the launch configuration
that bench.py times (automatic kernel choice, one CTA per SM), against the
fp64 oracle (GPU).

The oracle materialises every key, so its cost grows with the context:
whole workloads are checked where that takes seconds, and otherwise a sample
of sequences (the shortest and the longest) is checked element by element;
every other sequence is checked for finite outputs and for the properties
that hold at any size (lse at least the largest logit's lower bound, output
inside the convex hull of the cached latents per coordinate).
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


def _sample(inp, name):
    L = inp.seq_lens
    order = np.argsort(L, kind="stable")
    if name in ("tiny_f32", "small_mla_bf16"):
        return list(range(inp.wl.batch))
    if name == "long_ctx_bf16":
        return [0]
    return sorted({int(order[0]), int(order[1]), int(order[-1])})


@pytest.mark.parametrize("name", ["tiny_f32", "small_mla_bf16", "large_mla_bf16", "grouped_mtp_bf16",
                                  "long_ctx_bf16"])
def test_full_size_workload(name):
    inp = make_inputs(WORKLOADS[name])
    wl = inp.wl
    s = session_from_inputs(inp)
    out, lse = s.decode(inp.block_table, inp.seq_lens, wl.s_q)
    torch.cuda.synchronize()
    assert s.device_status() == qkn.OK
    if wl.dtype == "bf16":
        assert qkn.decode_kernel_for(s.dims, wl.s_q) == qkn.KERNEL_TCGEN05
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(l).all()

    seqs = _sample(inp, name)
    o_ref, l_ref = oracle.decode(inp, seqs=seqs)
    scale = np.abs(o_ref[seqs]).max()
    err = np.abs(o[seqs] - o_ref[seqs]).max()
    assert err <= REL_TOL[wl.dtype] * scale, f"{name}: {err:.3e} vs {REL_TOL[wl.dtype] * scale:.3e}"
    assert np.abs(l[seqs] - l_ref[seqs]).max() <= LSE_TOL[wl.dtype]

    # every sequence: the output is a convex combination of its visible latents
    slack = 2 ** -7 if wl.dtype == "bf16" else 1e-5
    for b in range(wl.batch):
        c = inp.c[inp.sequence(b)]
        lo, hi = c.min(0), c.max(0)
        span = np.maximum(hi - lo, 1e-6)
        ob = o[b].reshape(-1, wl.r_kv)
        assert (ob >= lo - slack * np.abs(lo) - 1e-6 * span).all()
        assert (ob <= hi + slack * np.abs(hi) + 1e-6 * span).all()
