"""Roofline accounting against the figures the pages print (CPU only)."""
import json
import os

from qk_normed_latent_qkn_b200.roofline import (cache_bytes_per_token, decode_step_cost, flops_per_token_row,
                                                gqa_step_cost)

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def test_absorbed_mla_intensity_matches_gqla_figure():
    fig = GOLDEN["absorbed_mla_intensity_flop_per_byte"]
    sh = fig["shape"]
    per_token_flops = sh["heads"] * flops_per_token_row(sh["r_kv"], sh["d_rope"])
    per_token_bytes = cache_bytes_per_token(sh["r_kv"], sh["d_rope"], 1, sh["elem_bytes"], scalar_cache=False)
    ai = per_token_flops / per_token_bytes
    assert abs(ai - fig["value"]) < 1.0, ai          # 128 * 2176 / 1152 = 241.8


def test_long_context_step_intensity_approaches_per_token_figure():
    c = decode_step_cost([262144, 262144], 1, 128, 1, 512, 64, scalar_cache=False)
    assert abs(c.intensity - 241.8) < 0.5


def test_scalar_cache_overhead_is_consistent_with_printed_figures():
    # fp32 scalars for g = 4 groups over a 512-wide bf16 latent: 16 / 1024 = 1.5625 %
    assert abs(16 / (2 * 512) - GOLDEN["scalar_cache_overhead_tested_configs"]["value"]) < 5e-4
    # the same 16 bytes over a 288-wide bf16 latent+RoPE cache: 16 / 576 = 2.78 %
    assert abs(16 / (2 * 288) - GOLDEN["scalar_cache_overhead_total_per_layer"]["value"]) < 5e-4


def test_step_cost_counts_causal_pairs():
    c1 = decode_step_cost([10], 1, 2, 1, 8, 4)
    c2 = decode_step_cost([10], 2, 2, 1, 8, 4)
    # query 0 of a two-token step sees one token fewer than query 1
    assert c2.flops == (9 + 10) * 2 * flops_per_token_row(8, 4)
    assert c1.flops == 10 * 2 * flops_per_token_row(8, 4)
    assert c1.cache_bytes == 10 * (2 * 12 + 4)


def test_gqa_route_intensity_sits_at_the_printed_ridge():
    # the GQA route's g and s_q put a long-context step's intensity at about 37 FLOP/byte for both
    # configurations the page names
    fig = GOLDEN["gqa_route_intensity_h20_ridge_flop_per_byte"]
    sh = fig["shape"]
    for cfg in fig["configs"]:
        L = 1 << 18
        c = gqa_step_cost([L], cfg["s_q"], cfg["heads"], cfg["groups"], sh["d_h"], sh["d_rope"], sh["d_v"],
                          elem=sh["elem_bytes"])
        assert abs(c.intensity - fig["value"]) < 2.5, (cfg, c.intensity)


def test_gqa_step_cost_counts_causal_pairs_and_group_bytes():
    c = gqa_step_cost([10], 2, 4, 2, 8, 4, 6)
    assert c.cache_bytes == 10 * 2 * (2 * (8 + 6) + 4)
    assert c.flops == (9 + 10) * 4 * (2 * (8 + 4) + 2 * 6)

