"""The seeded input generator's layouts (CPU only): the tied-group weights of GQLA's
parameterisation and the sparse token selections."""
import numpy as np

from qkn_inputs import WORKLOADS, make_inputs, make_selection

SMALL_GQLA = WORKLOADS["gqla_gqa_bf16"].with_(batch=3, heads=12, groups=3, r_kv=64, d_h=16, d_rope=8, d_v=8,
                                              context=(5, 150), seed=41)


def test_tied_groups_lay_one_key_and_value_head_over_each_group():
    inp = make_inputs(SMALL_GQLA)
    wl = inp.wl
    ng = wl.heads_per_group
    w_uk, gamma_k, w_uv = inp.group_weights()
    assert w_uk.shape == (wl.groups, wl.r_kv, wl.d_h) and w_uv.shape == (wl.groups, wl.r_kv, wl.d_v)
    for g in range(wl.groups):
        for m in range(ng):
            h = g * ng + m
            assert np.array_equal(inp.w_k[g][:, m * wl.d_h:(m + 1) * wl.d_h], w_uk[g])
            assert np.array_equal(inp.gamma_k[h], gamma_k[g])
            assert np.array_equal(inp.w_uv[h], w_uv[g])
    # the groups' heads are distinct draws
    assert not np.array_equal(w_uk[0], w_uk[1]) and not np.array_equal(w_uv[0], w_uv[1])
    # bf16 workloads store W^UV in bf16: its values are bf16-exact
    assert ((np.ascontiguousarray(w_uv, np.float32).view(np.uint32) & 0xFFFF) == 0).all()


def test_untied_workloads_draw_the_same_values_as_before():
    # the tied option leaves per-head workloads alone: these values were drawn by the generator as it
    # was before the option existed (same workload, same seed)
    wl = WORKLOADS["grouped_mtp_bf16"].with_(batch=2, context=(64, 200), seed=42)
    a = make_inputs(wl)
    assert a.seq_lens.tolist() == [76, 170]
    assert a.w_k.shape == (wl.groups, wl.r_kv, wl.heads_per_group * wl.d_h)
    assert float(a.w_k[1, 7, 200]) == 0.04644552245736122
    assert float(a.gamma_k[37, 5]) == 0.9609049558639526
    assert float(a.w_uv[63, 511, 127]) == 0.1279296875
    assert float(a.c[10, 3]) == 1.2734375
    assert float(a.q[1, 1, 40, 9]) == 1.3359375


def test_selection_lists_distinct_visible_tokens():
    inp = make_inputs(SMALL_GQLA)
    wl = inp.wl
    k = 40
    sel = make_selection(inp, k, seed=43)
    assert sel.shape == (wl.batch, wl.s_q, wl.groups, k) and sel.dtype == np.int32
    qpos = inp.query_positions()
    for b in range(wl.batch):
        for j in range(wl.s_q):
            n = int(qpos[b, j]) + 1
            for g in range(wl.groups):
                row = sel[b, j, g]
                listed = row[row >= 0]
                assert len(listed) == min(k, n)
                assert len(set(listed.tolist())) == len(listed)          # distinct
                assert (listed <= qpos[b, j]).all()                      # visible to the query
                assert (row[len(listed):] == -1).all()                   # padding at the end
    # seeded: the same seed gives the same lists, another seed others
    assert np.array_equal(sel, make_selection(inp, k, seed=43))
    assert not np.array_equal(sel, make_selection(inp, k, seed=44))
