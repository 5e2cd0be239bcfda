"""The step-preparation paths (GPU): qkn_append_absorb in one launch against
qkn_append + qkn_absorb_query as separate launches, and the one-launch append
(cache with ak_scratch) against the three-launch append (without)."""
import numpy as np
import pytest
import torch

from qk_normed_latent_qkn_b200.session import session_from_inputs
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _step(inp):
    wl = inp.wl
    B, s_q, H = wl.batch, wl.s_q, wl.heads
    last = np.concatenate([np.arange(inp.tok_off[b + 1] - s_q, inp.tok_off[b + 1]) for b in range(B)])
    return (inp.c[last], inp.k_rope[last], inp.token_slots()[last], inp.token_positions()[last],
            inp.q.reshape(B * s_q, H, wl.d_h), inp.q_rope.reshape(B * s_q, H, wl.d_rope),
            inp.query_positions().reshape(-1))


def _slots(s, slots):
    flat = lambda t: t.reshape(-1, *t.shape[2:])
    idx = torch.as_tensor(slots, dtype=torch.long, device=s.device)
    return [flat(t)[idx].float().cpu().numpy() for t in (s.cache.latent, s.cache.k_rope, s.cache.a_k)]


@pytest.mark.parametrize("name", ["tiny_f32", "small_mla_bf16", "grouped_mtp_bf16"])
def test_prepare_matches_separate_calls(name):
    inp = make_inputs(WORKLOADS[name])
    c, kr, slot, pos, q, qr, qpos = _step(inp)
    a = session_from_inputs(inp)
    b = session_from_inputs(inp)
    # the step's tokens are written again with different values, so that stale entries cannot pass
    c2, kr2 = c[::-1].copy(), kr[::-1].copy()
    a.append(c2, kr2, slot, pos)
    a.absorb(q, qr, qpos)
    b.prepare(c2, kr2, slot, pos, q, qr, qpos)
    torch.cuda.synchronize()
    la, ra, aka = _slots(a, slot)
    lb, rb, akb = _slots(b, slot)
    assert np.array_equal(la, lb) and np.array_equal(ra, rb)
    np.testing.assert_allclose(akb, aka, rtol=1e-5, atol=0)    # fp32 atomics: order of the partial sums
    for x, y in ((a.q_tilde, b.q_tilde), (a.a_q, b.a_q), (a.q_rope_hat, b.q_rope_hat)):
        assert torch.equal(x, y)
    # every append leaves the accumulators and counts at zero
    assert int(b.cache.ak_scratch.abs().sum()) == 0 and int(a.cache.ak_scratch.abs().sum()) == 0


@pytest.mark.parametrize("name", ["tiny_f32", "grouped_mtp_bf16"])
def test_one_launch_append_matches_three_launch_append(name):
    inp = make_inputs(WORKLOADS[name])
    c, kr, slot, pos, *_ = _step(inp)
    a = session_from_inputs(inp)
    b = session_from_inputs(inp)
    b.cache.ak_scratch = None                     # three launches: copy, key statistic, finalize
    c2, kr2 = c[::-1].copy(), kr[::-1].copy()
    a.append(c2, kr2, slot, pos)
    b.append(c2, kr2, slot, pos)
    torch.cuda.synchronize()
    la, ra, aka = _slots(a, slot)
    lb, rb, akb = _slots(b, slot)
    assert np.array_equal(la, lb) and np.array_equal(ra, rb)
    np.testing.assert_allclose(akb, aka, rtol=1e-5, atol=0)


@pytest.mark.parametrize("name", ["tiny_f32", "small_mla_bf16", "grouped_mtp_bf16"])
def test_key_gram_matches_fp64(name):
    import qk_normed_latent_qkn_b200 as qkn
    inp = make_inputs(WORKLOADS[name])
    s = session_from_inputs(inp)
    torch.cuda.synchronize()
    w = inp.w_k.astype(np.float64)                          # [G, r, n_g d_h]
    ref = np.einsum("gik,gjk->gij", w, w)
    got = s.key_gram.cpu().numpy()
    # fp64 accumulation rounded once to fp32
    assert np.abs(got - ref).max() <= 2 ** -23 * np.abs(ref).max()
    assert np.array_equal(got, np.swapaxes(got, 1, 2))      # symmetric
    assert s.key_gram.shape == (inp.wl.groups, inp.wl.r_kv, inp.wl.r_kv)
    del qkn


@pytest.mark.parametrize("name", ["tiny_f32", "grouped_mtp_bf16"])
@pytest.mark.parametrize("scratch", [True, False])
def test_gram_and_direct_key_statistic_match_oracle(name, scratch):
    """qkn_append with key_gram (c G c^T) and without (sum of (c W)^2), in the one-launch and the
    three-launch append, against the oracle's key statistic from explicitly formed keys."""
    import oracle
    import qk_normed_latent_qkn_b200 as qkn
    inp = make_inputs(WORKLOADS[name])
    c, kr, slot, pos, *_ = _step(inp)
    s = session_from_inputs(inp)
    if not scratch:
        s.cache.ak_scratch = None
    ref = oracle.key_inv_rms(c, inp.w_k, inp.wl.eps)
    dev = lambda x, dt: torch.as_tensor(np.ascontiguousarray(x)).to(device=s.device, dtype=dt)
    args = (dev(c, s.dims.torch_dtype), dev(kr, s.dims.torch_dtype), dev(slot, torch.int32), dev(pos, torch.int32))
    for gram in (s.key_gram, None):
        s.cache.a_k.zero_()
        qkn.append(s.dims, s.cache, *args, s.w_k, gram, s.gamma_kr)
        torch.cuda.synchronize()
        ak = _slots(s, slot)[2]
        np.testing.assert_allclose(ak, ref, rtol=2e-5, atol=0)
