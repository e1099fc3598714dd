"""Planted mistakes in the attention, rotary-embedding, e4m3 and cache-gate oracles (no GPU).

Each case builds a copy of one oracle module with one plausible mistake
planted in its source (a flipped sign, a wrong index, a dropped term, a
different rounding rule, a non-strict comparison ...), swaps the copy in for
the real module inside that module's committed pin tests, runs them, and
requires at least one pin to fail (an assertion, or an error a mutant raises).
The real oracle modules are never modified.
"""
import inspect
import types

import pytest

import test_oracle_attention as TA
import test_oracle_fp8_gate as T8
import test_oracle_rope as TR
from oracle import attention, fp8, gate, rope


def _mutant(module, edits):
    """A fresh module object holding module's source with each (old, new) edit applied once."""
    src = inspect.getsource(module)
    for old, new in edits:
        assert old in src, old
        src = src.replace(old, new, 1)
    m = types.ModuleType(module.__name__ + "_planted")
    m.__package__ = module.__package__
    exec(compile(src, f"<planted {module.__name__}>", "exec"), m.__dict__)
    return m


def _count_failing(pins):
    failed = 0
    for pin in pins:
        try:
            pin()
        except Exception:  # an assertion, or an error the mutant raises: the pin fails either way
            failed += 1
    return failed


ATTENTION_PINS = [
    TA.test_golden_hand_example,
    TA.test_zero_q_gives_mean_v_with_and_without_rope,
    TA.test_one_hot_scores_select_rows,
    TA.test_permutation_equivariance,
    TA.test_single_token_returns_v,
    TA.test_constant_v_gives_constant_output,
    TA.test_key_shift_invariance,
    TA.test_matches_torch_sdpa_float64,
    TA.test_brute_force_loops,
    TA.test_row_subset_matches_full,
    TA.test_rope_is_applied_to_q_and_k_not_v,
    TA.test_round_bf16_matches_torch_cast_of_float32,
    TA.test_round_bf16_ties_and_exact_values,
    TA.test_bf16_operand_reading_is_rounded_rotation,
]

_SIGMA = "sigma = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else float(scale)"
ATTENTION_MISTAKES = {
    "scale_argument_ignored": [(_SIGMA, "sigma = 1.0 / math.sqrt(d)")],
    "default_scale_one": [(_SIGMA, "sigma = 1.0 if scale is None or scale <= 0 else float(scale)")],
    "normalised_over_queries": [("/ e.sum(axis=1, keepdims=True)", "/ e.sum(axis=0, keepdims=True).T")],
    "last_key_left_out_of_the_sum": [("/ e.sum(axis=1, keepdims=True)", "/ e[:, :-1].sum(axis=1, keepdims=True)")],
    "v_rotated_too": [("    v = _f64(v)\n", "    v = rotate(v, pos, axes, theta)\n")],
    "k_not_rotated": [("k = rotate(k, pos, axes, theta)", "k = _f64(k)")],
    "bf16_operands_not_rounded": [("        q = round_bf16(q)\n        k = round_bf16(k)", "        q = q\n        k = k")],
    "bf16_rounding_truncates": [("np.round(ax / q) * q", "np.floor(ax / q) * q")],
    "bf16_one_bit_too_many": [("q = np.exp2(e - 7)", "q = np.exp2(e - 8)")],
    "selected_rows_ignored": [("s = sigma * (q[b, h, sel] @ kt)", "s = sigma * (q[b, h, r0:r0 + len(sel)] @ kt)")],
}


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(ATTENTION_MISTAKES))
def test_attention_pins_catch_planted_mistakes(name, monkeypatch):
    monkeypatch.setattr(TA, "A", _mutant(attention, ATTENTION_MISTAKES[name]))
    assert _count_failing(ATTENTION_PINS) >= 1, name


ROPE_PINS = [
    TR.test_golden_hand_values,
    TR.test_matches_complex_multiplication,
    TR.test_pair_norms_preserved,
    TR.test_position_zero_is_identity,
    TR.test_inverse_rotation,
    lambda: TR.test_scores_depend_only_on_relative_position((2, 9, 4)),
    TR.test_axes_are_independent,
    TR.test_angles_table_layout,
]

ROPE_MISTAKES = {
    "rotation_direction_reversed": [("x0 * c - x1 * s", "x0 * c + x1 * s"),
                                    ("x0 * s + x1 * c", "-x0 * s + x1 * c")],
    "one_sine_sign_flipped": [("x0 * c - x1 * s", "x0 * c + x1 * s")],
    "frequency_over_whole_head": [("-2.0 * p / da", "-2.0 * p / d")],
    "frequency_exponent_halved": [("-2.0 * p / da", "-1.0 * p / da")],
    "rotate_half_pairs": [("x0 = x[..., 0::2]", "x0 = x[..., : x.shape[-1] // 2]"),
                          ("x1 = x[..., 1::2]", "x1 = x[..., x.shape[-1] // 2:]"),
                          ("y[..., 0::2] =", "y[..., : x.shape[-1] // 2] ="),
                          ("y[..., 1::2] =", "y[..., x.shape[-1] // 2:] =")],
    "every_axis_uses_axis_0_position": [("pos[:, a] * freq", "pos[:, 0] * freq")],
    "pair_offset_dropped": [("out[:, off // 2 + p]", "out[:, p]")],
}


@pytest.mark.parametrize("name", sorted(ROPE_MISTAKES))
def test_rope_pins_catch_planted_mistakes(name, monkeypatch):
    monkeypatch.setattr(TR, "rope", _mutant(rope, ROPE_MISTAKES[name]))
    assert _count_failing(ROPE_PINS) >= 1, name


E4M3_PINS = [
    T8.test_code_table_round_trip,
    T8.test_ties_round_to_even_mantissa,
    T8.test_golden_e4m3,
    T8.test_matches_torch_float8_cast,
    T8.test_saturation,
    T8.test_block_scales_put_block_amax_on_448,
    T8.test_block_quantisation_within_e4m3_error_bound,
    T8.test_smoothing_leaves_exact_attention_unchanged,
]

E4M3_MISTAKES = {
    "ties_away_from_zero": [("np.round(ax / quantum)", "np.floor(ax / quantum + 0.5)")],
    "no_saturation": [("r = np.minimum(r, E4M3_MAX)", "r = r")],
    "subnormal_floor_one_binade_low": [("_MIN_NORMAL_EXP = -6", "_MIN_NORMAL_EXP = -7")],
    "two_mantissa_bits": [("_MANT_BITS = 3", "_MANT_BITS = 2")],
    "block_amax_mapped_to_240": [("a / E4M3_MAX, 1.0", "a / 240.0, 1.0")],
    "zero_block_scale_zero": [("a / E4M3_MAX, 1.0", "a / E4M3_MAX, 0.0")],
    "block_scales_shifted": [("rep = np.repeat(sc, block, axis=-1)[..., : x.shape[-2]]",
                              "rep = np.roll(np.repeat(sc, block, axis=-1)[..., : x.shape[-2]], 1, axis=-1)")],
    "smoothing_mean_over_channels": [("k.mean(axis=-2, keepdims=True)", "k.mean(axis=-1, keepdims=True)")],
}


@pytest.mark.parametrize("name", sorted(E4M3_MISTAKES))
def test_e4m3_pins_catch_planted_mistakes(name, monkeypatch):
    monkeypatch.setattr(T8, "fp8", _mutant(fp8, E4M3_MISTAKES[name]))
    assert _count_failing(E4M3_PINS) >= 1, name


INT8_PINS = [
    T8.test_int8_codes_round_trip_ties_to_even_and_clip,
    T8.test_int8_matches_torch_round_and_clamp,
    T8.test_int8_blocks_within_half_a_step,
    T8.test_simulated_int8_is_exact_where_every_step_is,
    T8.test_simulated_int8_keeps_an_integer_tie,
]

INT8_MISTAKES = {
    "ties_away_from_zero": [("np.clip(np.round(np.asarray(x, dtype=np.float64)), -INT8_MAX, INT8_MAX)",
                             "np.clip(np.trunc(np.asarray(x, dtype=np.float64) + np.copysign(0.5, x)), "
                             "-INT8_MAX, INT8_MAX)")],
    "no_clip": [("np.clip(np.round(np.asarray(x, dtype=np.float64)), -INT8_MAX, INT8_MAX)",
                 "np.round(np.asarray(x, dtype=np.float64))")],
    "clip_at_128": [("INT8_MAX = 127.0", "INT8_MAX = 128.0")],
    "amax_mapped_to_255": [("a / INT8_MAX, 1.0", "a / 255.0, 1.0")],
    "zero_block_scale_zero": [("a / INT8_MAX, 1.0", "a / INT8_MAX, 0.0")],
    "first_block_scale_for_all": [("quantize_int8(blk / sc[..., i, None, None])", "quantize_int8(blk / sc[..., 0, None, None])")],
    "k_left_in_e4m3": [("        k8, sk = quantize_int8_blocks(k, kv_block)", "        k8, sk = quantize_blocks(k, kv_block)")],
    "q_left_in_e4m3": [("        q8, sq = quantize_int8_blocks(q, q_block)", "        q8, sq = quantize_blocks(q, q_block)")],
}


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(INT8_MISTAKES))
def test_int8_pins_catch_planted_mistakes(name, monkeypatch):
    monkeypatch.setattr(T8, "fp8", _mutant(fp8, INT8_MISTAKES[name]))
    assert _count_failing(INT8_PINS) >= 1, name


GATE_PINS = [
    T8.test_golden_gate,
    T8.test_gate_brute_force_on_tiny_sweep,
    T8.test_gate_zero_denominator,
    T8.test_gate_strict_threshold,
    T8.test_gate_symmetric_scaling,
    T8.test_trace_decisions_follow_drift,
    T8.test_policy_consecutive_on_geometric_growth,
    T8.test_policy_last_computed_accumulates_until_threshold,
    T8.test_policy_warmup_forces_early_steps,
    T8.test_policy_last_computed_on_the_drift_trace,
]

GATE_MISTAKES = {
    "denominator_from_current_step": [("den = float(np.abs(b).sum())", "den = float(np.abs(a).sum())")],
    "squared_difference": [("num = float(np.abs(a - b).sum())", "num = float(((a - b) ** 2).sum())")],
    "threshold_not_strict": [("return rel < threshold", "return rel <= threshold")],
    "zero_denominator_always_inf": [('return 0.0 if num == 0.0 else float("inf")', 'return float("inf")')],
    "reference_never_moves": [("        if not s:\n            ref = t", "        if not s:\n            pass")],
    "reference_always_moves": [("        if not s:\n            ref = t", "        ref = t")],
    "warmup_off_by_one": [("and t >= warmup", "and t > warmup")],
    "policies_swapped": [('base = t - 1 if policy == "consecutive" else ref',
                          'base = ref if policy == "consecutive" else t - 1')],
}


@pytest.mark.parametrize("name", sorted(GATE_MISTAKES))
def test_gate_pins_catch_planted_mistakes(name, monkeypatch):
    monkeypatch.setattr(T8, "gate", _mutant(gate, GATE_MISTAKES[name]))
    assert _count_failing(GATE_PINS) >= 1, name


def test_unmutated_copies_pass_every_pin(monkeypatch):
    """The harness itself: copies built with no edit pass every pin."""
    monkeypatch.setattr(TA, "A", _mutant(attention, []))
    monkeypatch.setattr(TR, "rope", _mutant(rope, []))
    monkeypatch.setattr(T8, "fp8", _mutant(fp8, []))
    monkeypatch.setattr(T8, "gate", _mutant(gate, []))
    assert _count_failing(ATTENTION_PINS) == 0
    assert _count_failing(ROPE_PINS) == 0
    assert _count_failing(E4M3_PINS) == 0
    assert _count_failing(INT8_PINS) == 0
    assert _count_failing(GATE_PINS) == 0
