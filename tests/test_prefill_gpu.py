"""Attention forward over whole sequences (prefill / training-time forward) through the absorbed
path (GPU).

With s_q equal to the context every token is a query, and query j sees the tokens t <= j (the
decode's causal limit t <= L - s_q + j); a chunk of s_q new tokens after a cached history is the
chunked form.  The outputs are compared with the oracle's explicit form (materialised, normalised
keys) under the decode's tolerances, at sizes that span many 64-row tiles and a ragged last page."""
import numpy as np
import pytest
import torch

import oracle
import qk_normed_latent_qkn_b200 as qkn
from gpu_common import assert_close_to_oracle, run_decode
from qkn_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    # full prefill: 300 queries over 300 tokens, 16 heads (75 row tiles per sequence)
    "full_16h": WORKLOADS["prefill_mla_bf16"].with_(batch=2, s_q=300, context=300, seed=101),
    # chunked prefill: 200 new tokens after 300 to 700 cached ones
    "chunk_16h": WORKLOADS["prefill_mla_bf16"].with_(batch=3, s_q=200, context=(500, 900), seed=102),
    # four KV groups of 16 heads
    "full_grouped": WORKLOADS["grouped_mtp_bf16"].with_(batch=2, s_q=130, context=130, seed=103),
    # fp32 storage through the CUDA-core decode
    "full_f32": WORKLOADS["tiny_f32"].with_(batch=2, s_q=150, context=150, seed=104),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_prefill_matches_oracle(name):
    inp = make_inputs(CASES[name])
    s, o, lse = run_decode(inp)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o, lse, what=name)


def test_first_query_sees_only_the_first_token():
    # full prefill: query 0 of a sequence attends to token 0 alone, so its output is c_0 (rounded
    # once to bf16) and its lse is that single logit
    inp = make_inputs(CASES["full_16h"])
    s, o, lse = run_decode(inp)
    for b in range(inp.wl.batch):
        c0 = np.asarray(inp.c[inp.sequence(b)][0], dtype=np.float64)
        assert np.abs(o[b, 0] - c0[None, :]).max() <= 2 ** -8 * np.abs(c0).max()
        l = oracle.sequence_logits(inp, b)[0, :, 0]
        assert np.abs(lse[b, 0] - l).max() <= 2e-2


@pytest.mark.parametrize("head_tile", [16, 128])
def test_prefill_other_tiles(head_tile):
    inp = make_inputs(CASES["chunk_16h"])
    s, o, lse = run_decode(inp, head_tile=head_tile)
    assert_close_to_oracle(inp, o, lse, what=f"head_tile={head_tile}")


def test_prefill_workload_full_size_sampled():
    # the prefill workload at full size (2 x 2048 tokens, all of them queries), one sequence
    # against the oracle
    inp = make_inputs("prefill_mla_bf16")
    s, o, lse = run_decode(inp)
    assert s.device_status() == qkn.OK
    assert_close_to_oracle(inp, o, lse, seqs=[1], what="prefill_mla_bf16 full size")
