"""Failure paths of the decode, in forms that neither fault nor hang the GPU (GPU).

- A bounded wait that runs out: the test-only option ``test_withhold_ak``
  makes the tcgen05 decode's producer skip one a_k copy, so the softmax's wait
  for that barrier phase (which nothing else completes) runs out after
  ``wait_limit`` cycles.  The decode must record QKN_ERR_TIMEOUT, wind down
  with every copy and MMA it issued waited for, and leave the context usable:
  after the status is cleared, the next decode on the same workspace matches
  the oracle.
- A block id outside the pool: the kernels clamp it to block 0 and record
  QKN_ERR_BOUNDS; the other sequences' results are unaffected.
- A slot id outside the pool in an append: the token is skipped in every
  append path (one launch, three launches, the GEMM form for many tokens).
"""
import numpy as np
import pytest
import torch

import qk_normed_latent_qkn_b200 as qkn
from gpu_common import assert_close_to_oracle
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

# about half a millisecond at the B200's clocks: every wait that nothing completes ends quickly
SHORT_WAIT = 1_000_000

CASES = {
    "small_mla_bf16": WORKLOADS["small_mla_bf16"].with_(batch=4, context=700, seed=31),
    "large_mla_bf16": WORKLOADS["large_mla_bf16"].with_(batch=3, context=(200, 900), seed=32),
    "grouped_mtp_bf16": WORKLOADS["grouped_mtp_bf16"].with_(batch=3, context=(130, 700), seed=33),
}


def _decode(s, inp, **kw):
    kw.setdefault("kernel", qkn.KERNEL_TCGEN05)
    out, lse = s.decode(inp.block_table, inp.seq_lens, inp.wl.s_q, **kw)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name", sorted(CASES))
def test_wait_that_runs_out_is_reported_and_the_next_decode_is_correct(name):
    inp = make_inputs(CASES[name])
    s = session_from_inputs(inp)
    _decode(s, inp, wait_limit=SHORT_WAIT, test_withhold_ak=True)
    assert s.device_status() == qkn.ERR_TIMEOUT
    # the context is intact: clear the status and decode again on the same workspace
    s.clear_status()
    o, lse = _decode(s, inp)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o, lse, what=f"{name} after a timeout")


@pytest.mark.parametrize("name", ["large_mla_bf16", "grouped_mtp_bf16"])
def test_wait_that_runs_out_on_the_cta_pair_kernel(name):
    # 128-row tiles on CTA pairs: a timeout in one CTA of a pair must wind both down (the two
    # exchange data every page) and leave the context usable
    inp = make_inputs(CASES[name])
    s = session_from_inputs(inp)
    _decode(s, inp, head_tile=128, wait_limit=SHORT_WAIT, test_withhold_ak=True)
    assert s.device_status() == qkn.ERR_TIMEOUT
    s.clear_status()
    o, lse = _decode(s, inp, head_tile=128)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o, lse, what=f"{name} on CTA pairs after a timeout")


def test_timeout_twice_in_a_row_then_correct():
    inp = make_inputs(CASES["small_mla_bf16"])
    s = session_from_inputs(inp)
    for _ in range(2):
        _decode(s, inp, wait_limit=SHORT_WAIT, test_withhold_ak=True)
        assert s.device_status() == qkn.ERR_TIMEOUT
        s.clear_status()
    o, lse = _decode(s, inp)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o, lse, what="after two timeouts")


@pytest.mark.parametrize("kernel", [qkn.KERNEL_TCGEN05, qkn.KERNEL_SIMT])
def test_block_id_out_of_range_is_clamped_and_reported(kernel):
    inp = make_inputs(CASES["large_mla_bf16"])
    s = session_from_inputs(inp)
    bt = inp.block_table.copy()
    assert int(inp.seq_lens[0]) > 64           # sequence 0 has a second page
    bt[0, 1] = inp.num_blocks + 5              # outside the pool
    out, lse = s.decode(bt, inp.seq_lens, inp.wl.s_q, kernel=kernel)
    torch.cuda.synchronize()
    assert s.device_status() == qkn.ERR_BOUNDS
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    # the other sequences read only their own pages
    assert_close_to_oracle(inp, o, l, seqs=range(1, inp.wl.batch), what="sequences without the bad id")


@pytest.mark.parametrize("n_bad, scratch", [(4, True), (4, False), (300, True)],
                         ids=["one-launch", "three-launch", "gemm-path"])
def test_append_skips_slots_outside_the_pool(n_bad, scratch):
    # new tokens for the free slots at the end of each sequence's last page, mixed with tokens whose
    # slot ids lie outside the pool (negative, and past its end): those are skipped, nothing is
    # written outside the pool, and the valid tokens get their latent rows and a_k
    import oracle
    inp = make_inputs(CASES["grouped_mtp_bf16"])
    s = session_from_inputs(inp)
    if not scratch:
        s.cache.ak_scratch = None                       # the three-launch append
    pool = inp.num_blocks * 64
    free = []
    for b in range(inp.wl.batch):
        L = int(inp.seq_lens[b])
        last = int(inp.block_table[b, (L - 1) // 64])
        free += [last * 64 + t for t in range(L % 64, 64)] if L % 64 else []
    free = np.array(free[:6], dtype=np.int32)
    assert free.size > 0
    bad = np.array([-1 - k if k % 2 == 0 else pool + k for k in range(n_bad)], dtype=np.int32)
    slots = np.concatenate([free, bad])
    rng = np.random.default_rng(8)
    n = slots.size
    c = rng.standard_normal((n, inp.wl.r_kv)).astype(np.float32)
    kr = rng.standard_normal((n, inp.wl.d_rope)).astype(np.float32)
    pos = np.arange(n, dtype=np.int32)
    a_k_before = s.cache.a_k.clone()
    s.append(c, kr, slots, pos)
    torch.cuda.synchronize()
    a_k = s.cache.a_k.reshape(-1, inp.wl.groups).cpu().numpy()
    lat = s.cache.latent.reshape(pool, -1).float().cpu().numpy()
    c_bf16 = torch.from_numpy(c).to(torch.bfloat16).float().numpy()
    ref = oracle.key_inv_rms(c_bf16[:free.size].astype(np.float64), inp.w_k, inp.wl.eps)
    np.testing.assert_allclose(a_k[free], ref, rtol=2e-5)
    assert (lat[free] == c_bf16[:free.size]).all()
    # every other slot of the pool keeps its a_k
    others = torch.from_numpy(np.setdiff1d(np.arange(pool), free)).to(s.cache.a_k.device)
    assert torch.equal(s.cache.a_k.reshape(-1, inp.wl.groups)[others], a_k_before.reshape(-1, inp.wl.groups)[others])
