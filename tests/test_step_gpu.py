"""DecodeStep (one graph per step: copy-in, append + absorb, decode, copy-out)
against the eager session calls and the fp64 oracle (GPU)."""
import copy

import numpy as np
import pytest
import torch

import oracle
import qk_normed_latent_qkn_b200 as qkn
from gpu_common import LSE_TOL, REL_TOL
from qk_normed_latent_qkn_b200.session import session_from_inputs
from qk_normed_latent_qkn_b200.step import DecodeStep
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _step_inputs(inp):
    """The step appends the last s_q tokens of every sequence, with values that differ from the ones
    the cache was built with (so that a stale read of a page with new tokens cannot pass), and carries
    its queries.  Returns the step inputs and the problem as the oracle must see it."""
    wl = inp.wl
    B, s_q, H = wl.batch, wl.s_q, wl.heads
    last = np.concatenate([np.arange(inp.tok_off[b + 1] - s_q, inp.tok_off[b + 1]) for b in range(B)])
    inp2 = copy.copy(inp)
    inp2.c, inp2.k_rope = inp.c.copy(), inp.k_rope.copy()
    inp2.c[last] = inp.c[last][::-1] * 2.0            # exact in bf16
    inp2.k_rope[last] = -inp.k_rope[last][::-1]
    return last, inp2, {
        "c": inp2.c[last], "k_rope": inp2.k_rope[last], "slot": inp.token_slots()[last],
        "pos": inp.token_positions()[last], "q": inp.q.reshape(B * s_q, H, wl.d_h),
        "q_rope": inp.q_rope.reshape(B * s_q, H, wl.d_rope), "qpos": inp.query_positions().reshape(-1),
        "block_table": inp.block_table, "seq_lens": inp.seq_lens,
    }


@pytest.mark.parametrize("name", ["tiny_f32", "small_mla_bf16"])
def test_step_matches_eager_and_oracle(name):
    inp = make_inputs(WORKLOADS[name])
    wl = inp.wl
    s = session_from_inputs(inp)
    last, inp2, host = _step_inputs(inp)
    step = DecodeStep(s, wl.batch, wl.s_q, inp.block_table.shape[1], len(last))
    for k, v in host.items():
        step.host_in[k].copy_(torch.from_numpy(np.ascontiguousarray(v)).to(step.host_in[k].dtype))
    for _ in range(3):                      # replays are repeatable
        out, lse = step.run()
    assert s.device_status() == qkn.OK
    o = out.float().numpy().astype(np.float64)
    l = lse.numpy().astype(np.float64)

    eo, el = s.decode(inp.block_table, inp.seq_lens, wl.s_q)
    torch.cuda.synchronize()
    eo = eo.float().cpu().numpy().astype(np.float64)
    el = el.cpu().numpy().astype(np.float64)
    scale = np.abs(eo).max()
    # the key statistics of the re-appended tokens are summed with atomics: equal up to rounding
    assert np.abs(o - eo).max() <= 2 ** -7 * scale
    assert np.abs(l - el).max() <= LSE_TOL[wl.dtype]

    o_ref, l_ref = oracle.decode(inp2)
    assert np.abs(o - o_ref).max() <= REL_TOL[wl.dtype] * np.abs(o_ref).max()
    assert np.abs(l - l_ref).max() <= LSE_TOL[wl.dtype]


def test_step_byte_counts():
    """One copy each way: the packed buffers hold every field, 256-byte aligned."""
    inp = make_inputs(WORKLOADS["tiny_f32"])
    s = session_from_inputs(inp)
    last, _, host = _step_inputs(inp)
    step = DecodeStep(s, inp.wl.batch, inp.wl.s_q, inp.block_table.shape[1], len(last))
    field = lambda n: (n + 255) // 256 * 256
    assert step.h2d_bytes == sum(field(np.ascontiguousarray(v).astype(step.host_in[k].numpy().dtype).nbytes)
                                 for k, v in host.items())
    assert step.d2h_bytes == field(step.host_out[0].numel() * 4) + field(step.host_out[1].numel() * 4)
    for t in list(step.host_in.values()) + list(step.dev_in.values()):
        assert t.data_ptr() % 256 == 0
