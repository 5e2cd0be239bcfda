"""qkn_decode_noalloc against qkn_decode (GPU).

qkn_decode_noalloc serves callers that cannot allocate device memory — an
operator inside another engine that is handed only its input and output
pointers, or a serving loop whose memory pool already owns the GPU — by
keeping the decode's scratch in a fixed array inside libqkn.  Its output must
match the ordinary entry point's, call after call, since every call reuses
the same scratch.  This file is collected last so that a run stopping at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import qk_normed_latent_qkn_b200 as qkn
from gpu_common import LSE_TOL, REL_TOL
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "small_mla_bf16": WORKLOADS["small_mla_bf16"].with_(batch=4, context=700, seed=11),
    "large_mla_bf16": WORKLOADS["large_mla_bf16"].with_(batch=3, context=(200, 900), seed=12),
    "grouped_mtp_bf16": WORKLOADS["grouped_mtp_bf16"].with_(batch=3, context=(130, 700), seed=13),
}


def _noalloc_raw(s, inp, out, lse, status):
    """Call qkn_decode_noalloc through the C ABI with raw pointers."""
    lib = qkn.raw_library()
    bt = torch.from_numpy(inp.block_table).cuda()
    sl = torch.from_numpy(inp.seq_lens).cuda()
    rc = lib.qkn_decode_noalloc(ctypes.byref(s.dims.c()), ctypes.byref(s.cache.c()), qkn.AK_CACHE,
                                s.q_tilde.data_ptr(), s.a_q.data_ptr(), s.q_rope_hat.data_ptr(), bt.data_ptr(),
                                bt.shape[1], sl.data_ptr(), bt.shape[0], inp.wl.s_q, out.data_ptr(),
                                lse.data_ptr(), status.data_ptr(), None,
                                torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return rc


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_decode_on_two_calls_in_a_row(name):
    inp = make_inputs(CASES[name])
    wl = inp.wl
    s = session_from_inputs(inp)
    ref_o, ref_l = s.decode(inp.block_table, inp.seq_lens, wl.s_q)
    torch.cuda.synchronize()
    ref_o = ref_o.float().cpu().numpy()
    ref_l = ref_l.cpu().numpy()
    scale = np.abs(ref_o).max()
    for call in range(2):
        out = torch.full((wl.batch, wl.s_q, wl.heads, wl.r_kv), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((wl.batch, wl.s_q, wl.heads), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        assert _noalloc_raw(s, inp, out, lse, status) == qkn.OK
        assert int(status.item()) == qkn.OK, f"call {call}: device status {int(status.item())}"
        o = out.float().cpu().numpy()
        l = lse.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(l).all(), f"call {call}"
        assert np.abs(o - ref_o).max() <= REL_TOL[wl.dtype] * scale, f"call {call}"
        assert np.abs(l - ref_l).max() <= LSE_TOL[wl.dtype], f"call {call}"


def test_noalloc_rejects_a_problem_larger_than_its_scratch():
    inp = make_inputs(CASES["small_mla_bf16"])
    s = session_from_inputs(inp)
    big_batch = 4096     # needs far more than the fixed scratch for its split partials
    need = qkn.decode_workspace_size(s.dims, big_batch, 1)
    assert need > qkn.NOALLOC_SCRATCH_BYTES
    lib = qkn.raw_library()
    rc = lib.qkn_decode_noalloc(ctypes.byref(s.dims.c()), ctypes.byref(s.cache.c()), qkn.AK_CACHE,
                                s.q_tilde.data_ptr(), s.a_q.data_ptr(), s.q_rope_hat.data_ptr(), 0x100, 1, 0x100,
                                big_batch, 1, 0x100, 0x100, None, None, torch.cuda.current_stream().cuda_stream)
    assert rc == qkn.ERR_UNSUPPORTED


def test_noalloc_with_nothing_to_decode_reports_ok():
    """batch == 0 decodes nothing, returns QKN_OK and writes QKN_OK to the caller's status word."""
    inp = make_inputs(CASES["small_mla_bf16"])
    s = session_from_inputs(inp)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    lib = qkn.raw_library()
    rc = lib.qkn_decode_noalloc(ctypes.byref(s.dims.c()), ctypes.byref(s.cache.c()), qkn.AK_CACHE,
                                s.q_tilde.data_ptr(), s.a_q.data_ptr(), s.q_rope_hat.data_ptr(), 0x100, 1, 0x100,
                                0, 1, 0x100, 0x100, status.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == qkn.OK
    assert int(status.item()) == qkn.OK
