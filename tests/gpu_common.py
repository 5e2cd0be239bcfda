"""Helpers for the GPU parity tests: run the library on a seeded problem and
compare with the fp64 oracle under the tolerances of the decode workloads.

Tolerances: max |o_gpu - o_oracle| <= 1e-4 * max|o_oracle| for fp32 storage
and <= 1e-2 * max|o_oracle| for bf16 storage.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import qk_normed_latent_qkn_b200 as qkn
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import make_inputs

REL_TOL = {"f32": 1e-4, "bf16": 1e-2}
LSE_TOL = {"f32": 1e-4, "bf16": 2e-2}


def run_decode(inp, kernel=qkn.KERNEL_AUTO, ak_mode=qkn.AK_CACHE, max_ctas=0, head_tile=0, session=None):
    s = session if session is not None else session_from_inputs(inp)
    out, lse = s.decode(inp.block_table, inp.seq_lens, inp.wl.s_q, ak_mode=ak_mode, kernel=kernel,
                        max_ctas=max_ctas, head_tile=head_tile)
    torch.cuda.synchronize()
    return s, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def assert_close_to_oracle(inp, o, lse, seqs=None, what=""):
    o_ref, lse_ref = oracle.decode(inp, seqs=seqs)
    sel = list(range(inp.wl.batch)) if seqs is None else list(seqs)
    o_ref, lse_ref, o, lse = o_ref[sel], lse_ref[sel], o[sel], lse[sel]
    scale = np.abs(o_ref).max()
    err = np.abs(o - o_ref).max()
    tol = REL_TOL[inp.wl.dtype] * scale
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err <= tol, f"{what}: max|o - o_ref| = {err:.3e} > {tol:.3e} (max|o_ref| = {scale:.3e})"
    lerr = np.abs(lse - lse_ref).max()
    assert lerr <= LSE_TOL[inp.wl.dtype], f"{what}: max|lse - lse_ref| = {lerr:.3e}"
    return err / scale
