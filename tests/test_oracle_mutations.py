"""Plant plausible mistakes in a copy of the oracle and confirm a pin catches each (CPU only).

Each mutation is a source-level replacement applied to a private copy of
``oracle/__init__.py``; the shipped oracle is never modified.
"""
import inspect
import types

import pytest

import oracle
import oracle_pins

MUTATIONS = {
    "causal_off_by_one": ("kpos[None, :] <= qpos[:, None]", "kpos[None, :] < qpos[:, None]"),
    "eps_outside_sqrt": ("np.sqrt(np.mean(x * x, axis=-1) + eps)", "(np.sqrt(np.mean(x * x, axis=-1)) + eps)"),
    "rotation_direction": ("x1 * cos - x2 * sin, x2 * cos + x1 * sin", "x1 * cos + x2 * sin, x2 * cos - x1 * sin"),
    "rope_pairs_interleaved": ("x1, x2 = x[..., :half], x[..., half:]", "x1, x2 = x[..., 0::2], x[..., 1::2]"),
    "dropped_gamma_k": ("k = rms_norm(cc @ w[g], gk, wl.eps)", "k = rms_norm(cc @ w[g], 1.0, wl.eps)"),
    "head_group_swapped": ("grp, m = divmod(h, ng)", "m, grp = divmod(h, ng)"),
    "key_slice_transposed": ("w_h = w[grp][:, m * d_h:(m + 1) * d_h]", "w_h = w[grp][:, m::ng][:, :d_h]"),
    "key_rms_half_width": ("out[t0:t0 + chunk, g] = inv_rms(cc @ w[g], eps)",
                           "out[t0:t0 + chunk, g] = inv_rms((cc @ w[g])[:, ::2], eps)"),
    "sigma_squared": ("logits *= sigma", "logits *= sigma * sigma"),
    "dropped_rope_block": ('logits += np.einsum("jhd,td->jht", qrh, krh)', "pass"),
    "query_rope_position": ("qpos[:, None], wl.rope_theta)", "qpos[:, None] + 1, wl.rope_theta)"),
    "key_rope_unnormalised": ("return rope(rms_norm(k_rope, gamma_kr, eps), pos, theta)",
                              "return rope(np.asarray(k_rope, np.float64) * gamma_kr, pos, theta)"),
    "values_normalised": ("return p @ c, lse", "return p @ (c / np.abs(c).max()), lse"),
    "row_scale_without_sigma": ("a_q = softmax_scale * inv_rms(q, eps)", "a_q = inv_rms(q, eps)"),
    "row_scale_half_width": ("a_q = softmax_scale * inv_rms(q, eps)",
                             "a_q = softmax_scale * inv_rms(q[..., ::2], eps)"),
    "up_projection_wrong_head": ("out[..., h, :] = o[..., h, :] @ w[h]",
                                 "out[..., h, :] = o[..., h, :] @ w[(h + 1) % w.shape[0]]"),
    "up_projection_rows_reversed": ("out[..., h, :] = o[..., h, :] @ w[h]",
                                    "out[..., h, :] = o[..., h, :] @ w[h][::-1]"),
    "gqa_key_group_of_head": ("qh[:, g * ng:(g + 1) * ng], k[:, g, :])", "qh[:, g * ng:(g + 1) * ng], k[:, (g + 1) % wl.groups, :])"),
    "gqa_value_group_shifted": ("v[:, g, :])", "v[:, (g + 1) % wl.groups, :])"),
    "gqa_key_gamma_dropped": ("rms_norm(c @ wk[g], np.asarray(gamma_k[g], np.float64), eps)",
                              "rms_norm(c @ wk[g], 1.0, eps)"),
    "gqa_key_unnormalised": ("rms_norm(c @ wk[g], np.asarray(gamma_k[g], np.float64), eps)",
                             "(c @ wk[g]) * np.asarray(gamma_k[g], np.float64)"),
    "gqa_values_from_keys_weight": ("np.stack([c @ wv[g] for g in range(wv.shape[0])], axis=1)",
                                    "np.stack([c @ wv[g][::-1] for g in range(wv.shape[0])], axis=1)"),
    "gqa_rope_dropped": ('logits = logits + np.einsum("jhd,td->jht", qrh, krh)', "pass"),
    "gqa_causal_off_by_one": ("visible = np.arange(L)[None, :] <= qpos[:, None]",
                              "visible = np.arange(L)[None, :] < qpos[:, None]"),
    "gqa_selection_of_group_zero": ("idx = np.asarray(selection[j, g])", "idx = np.asarray(selection[j, 0])"),
    "gqa_selection_ignored": ("mask &= listed[:, grp, :]", "pass"),
    "gqa_query_rope_position": ("pos=qpos[:, None], theta", "pos=qpos[:, None] + 1, theta"),
}


def _mutant(old, new):
    src = inspect.getsource(oracle)
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    mutant = _mutant(*MUTATIONS[name])
    monkeypatch.setattr(oracle_pins, "oracle", mutant)
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check()
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"no pin caught mutation {name}"
