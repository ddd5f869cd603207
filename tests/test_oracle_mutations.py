"""Planted-mistake check of the oracle pins (CPU only).

Each entry plants one plausible slip in a private copy of the oracle module and
asserts that at least one pin in ``test_oracle_pins`` fails on it.
"""

import importlib.util
import inspect
import os
import types

import pytest

import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "mla_oracle.py")

MUTATIONS = {
    "rope_rotation_sign": ("x1 * c - x2 * s, x2 * c + x1 * s", "x1 * c + x2 * s, x2 * c - x1 * s"),
    "rope_interleaved_pairs": ("x1, x2 = x[..., :h], x[..., h:]\n    return np.concat",
                               "x1, x2 = x[..., 0::2], x[..., 1::2]\n    return np.concat"),
    "rope_frequency_exponent": ("return base ** (-(2.0 * m) / d_r)", "return base ** (-(1.0 * m) / d_r)"),
    "scale_without_rope_dims": ("1.0 / math.sqrt(d_h + d_r)", "1.0 / math.sqrt(d_h)"),
    "shared_key_dropped": ("k = np.concatenate([k_c, k_r_rot], axis=1)",
                           "k = np.concatenate([k_c, 0 * k_r_rot], axis=1)"),
    "mask_off_by_one": ("visible = j_idx <= (T_k - T_q + t_idx)", "visible = j_idx < (T_k - T_q + t_idx)"),
    "value_uses_key_weight": ("v_c = c_kv @ wv.T", "v_c = c_kv @ wk.T"),
    "query_position_shift": ("qpos = np.arange(L - T_q, L)", "qpos = np.arange(L - T_q, L) - 1"),
    "merge_weights_linear": ("w = np.exp(lse_parts - m)", "w = (lse_parts - m + 1)"),
    "absorb_transposed": ("out[:, i, :] = q_c[:, i, :] @ w_uk[i]",
                          "out[:, i, :] = (q_c[:, i, :] @ w_uk[i])[:, ::-1]"),
    "up_v_feature_order": ("out[:, i, :] = latent[:, i, :] @ w_uv[i].T",
                           "out[:, i, :] = latent[:, i, :] @ w_uv[i][::-1].T"),
    "lse_without_max": ("lse[:, hi] = (m + np.log(z))[:, 0]", "lse[:, hi] = np.log(z)[:, 0]"),
    "rope_table_cos_sin_swapped": ("return np.concatenate([np.cos(theta), np.sin(theta)], axis=1).astype(np.float32)",
                                   "return np.concatenate([np.sin(theta), np.cos(theta)], axis=1).astype(np.float32)"),
    "rope_emulation_sign": ("a = (x1 * c) - (x2 * s)", "a = (x1 * c) + (x2 * s)"),
    # one rounding of the exact difference / sum instead of a rounding per step
    "rope_emulation_single_rounding": (
        "a = (x1 * c) - (x2 * s)\n    b = (x2 * c) + (x1 * s)",
        "a = ((x1.astype(np.float64) * c) - (x2.astype(np.float64) * s)).astype(np.float32)\n"
        "    b = ((x2.astype(np.float64) * c) + (x1.astype(np.float64) * s)).astype(np.float32)"),
    # a fused multiply-add: the first product is not rounded before the difference
    "rope_emulation_fused": (
        "a = (x1 * c) - (x2 * s)\n    b = (x2 * c) + (x1 * s)",
        "a = (x1.astype(np.float64) * c - (x2 * s)).astype(np.float32)\n"
        "    b = (x2.astype(np.float64) * c + (x1 * s)).astype(np.float32)"),
    "yarn_turns_without_two_pi": ("turns = orig_len * f / (2.0 * math.pi)", "turns = orig_len * f"),
    "yarn_ramp_reversed": ("return f * ((1.0 - gamma) / s + gamma)", "return f * (gamma / s + (1.0 - gamma))"),
    "yarn_temperature_not_squared": ("return yarn_sqrt_temperature(s, coeff) ** 2 / math.sqrt(d_h + d_r)",
                                     "return yarn_sqrt_temperature(s, coeff) / math.sqrt(d_h + d_r)"),
    "fold_q_uses_query_weight_twice": ('return np.einsum("hkc,hkd->hcd", w_uk, w_uq)',
                                       'return np.einsum("hkc,hkd->hcd", w_uq[..., :w_uk.shape[2]], w_uq)'),
    "fold_o_head_mismatch": ('return np.einsum("mhk,hkc->mhc", w_o, w_uv)',
                                  'return np.einsum("mhk,hkc->mhc", w_o, w_uv[::-1])'),
    "q_up_transposed_contraction": ('return np.einsum("hkd,nd->nhk", w_uq, c_q)',
                                    'return np.einsum("hkd,nd->nhk", w_uq[:, ::-1], c_q)'),
    "o_proj_head_order": ('return np.einsum("mhk,nhk->nm", w_o, o)',
                          'return np.einsum("mhk,nhk->nm", w_o, o[:, ::-1])'),
    "folded_q_wrong_axis": ('return np.einsum("hcd,nd->nhc", np.asarray(f, dtype=np.float64)',
                            'return np.einsum("hcd,nd->nhc", np.asarray(f[::-1], dtype=np.float64)'),
    "gather_wrong_slot": ("return int(block_table[b, pos // block_size]), pos % block_size",
                          "return int(block_table[b, pos // block_size]), (pos + 1) % block_size"),
}


def _mutated_module(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("mla_oracle_mutant")
    exec(compile(src.replace(old, new), "mla_oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    mod = _mutated_module(*MUTATIONS[name])
    monkeypatch.setattr(pins, "O", mod)
    failures = 0
    for fname, fn in inspect.getmembers(pins, inspect.isfunction):
        if not fname.startswith("test_"):
            continue
        try:
            fn()
        except Exception:
            failures += 1
    assert failures >= 1, f"no pin caught mutation {name}"


# Slips in the per-sequence evaluation that the GPU tests compare against; the
# brute force of whole workload cases must catch each.
import tests.test_oracle_brute_force as brute  # noqa: E402

EVAL_SRC = os.path.join(os.path.dirname(SRC), "evaluate.py")

EVAL_MUTATIONS = {
    "query_rows_of_next_token": ("sl = slice(b * T_q, (b + 1) * T_q)", "sl = slice(b * T_q + 1, (b + 1) * T_q + 1)"),
    "weights_swapped": ("_CACHE[key] = (O.bf16_to_f64(spec.w_uk()), O.bf16_to_f64(spec.w_uv()))",
                        "_CACHE[key] = (O.bf16_to_f64(spec.w_uv()), O.bf16_to_f64(spec.w_uk()))"),
    "rope_query_part_dropped": ("_CACHE[key] = (O.bf16_to_f64(spec.q_c()), O.bf16_to_f64(spec.q_r()))",
                                "_CACHE[key] = (O.bf16_to_f64(spec.q_c()), 0 * O.bf16_to_f64(spec.q_r()))"),
    "history_of_other_sequence": ("c = O.bf16_to_f64(spec.c_kv_rows(b, 0, L))",
                                  "c = O.bf16_to_f64(spec.c_kv_rows(b + 1, 0, L))"),
}


@pytest.mark.parametrize("name", sorted(EVAL_MUTATIONS))
def test_brute_force_catches_planted_evaluation_mistake(name, monkeypatch):
    old, new = EVAL_MUTATIONS[name]
    src = open(EVAL_SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.evaluate_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "evaluate_mutant", "exec"), mod.__dict__)
    monkeypatch.setattr(brute, "evaluate", mod)
    spec = brute.CaseSpec(n_h=2, d_c=16, d_h=8, d_r=8, seq_lens=brute.np.array([5, 23], brute.np.int32),
                          T_q=3, seed=4)
    with pytest.raises(Exception):
        brute._check(spec, 0)
        brute._check(spec, 1)
