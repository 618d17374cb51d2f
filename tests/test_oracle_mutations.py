"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

Every mutation edits the oracle's source text, builds a throw-away module from
it, and swaps its functions into the ``oracle`` package for the duration of the
test.  The listed pins must then fail (raise AssertionError).  Nothing here
touches a GPU.
"""
import inspect
import types

import pytest

import oracle
import oracle.oracle as src_mod
import test_oracle as T
import test_oracle_int8 as T8
import test_oracle_chunk as TC
import test_oracle_transformed as TT

MUTATIONS = {
    # name: (original text, replacement, pins that must fail)
    "rope_rotates_backwards": (
        "out[..., :half] = a * c - b * s", "out[..., :half] = a * c + b * s",
        [T.test_rope_worked_example, T.test_rope_is_complex_rotation]),
    "rope_interleaved_pairs": (
        "a = x[..., :half]\n    b = x[..., half:rot_dim]",
        "a = x[..., 0:rot_dim:2]\n    b = x[..., 1:rot_dim:2]",
        [T.test_rope_worked_example]),
    "rope_frequency_uses_t_not_2t": (
        "theta ** (-2.0 * t / freq_dim)", "theta ** (-1.0 * t / freq_dim)",
        [T.test_rope_worked_example, T.test_rope_is_complex_rotation]),
    "norm_drops_one_plus": (
        "g = (1.0 + w) if mode == NORM_ONE_PLUS_W else w", "g = w",
        [T.test_rms_norm_worked_example]),
    "norm_sum_not_mean": (
        "ms = np.mean(x * x, axis=-1, keepdims=True)", "ms = np.sum(x * x, axis=-1, keepdims=True)",
        [T.test_rms_norm_worked_example]),
    "norm_eps_outside_root": (
        "return x / np.sqrt(ms + eps) * g", "return x / (np.sqrt(ms) + eps) * g",
        [T.test_rms_norm_worked_example]),
    "window_off_by_one": (
        "ok = ok & (i - j < window)", "ok = ok & (i - j <= window)",
        [T.test_mask_window_limits, T.test_mask_future_and_past_independence]),
    "scale_divides_by_scalar": (
        "scale=float(get(\"scalar\")) ** -0.5", "scale=1.0 / float(get(\"scalar\"))",
        [T.test_worked_three_tokens]),
    "softcap_drops_c": (
        "return c * np.tanh(s / c)", "return np.tanh(s / c)",
        [T.test_softcap_closed_form]),
    "gqa_heads_strided": (
        "            kv = h // G\n            valid", "            kv = h % Hkv\n            valid",
        [T.test_mqa_equals_replicated_gqa]),
    "keqv_values_are_normed_keys": (
        "vals_all = k if f[\"k_eq_v\"] else v",
        "vals_all = rms_norm(k, w_k, f[\"mode\"], f[\"eps\"]) if f[\"k_eq_v\"] else v",
        [T.test_k_eq_v_is_passing_v_equals_k]),
    "decode_query_one_past": (
        "np.array([L - 1]),\n                  f[\"rot\"]", "np.array([L]),\n                  f[\"rot\"]",
        [T.test_decode_equals_last_prefill_row]),
    "softmax_drops_normaliser": (
        "p = p / np.where(den > 0, den, 1.0)", "p = p",
        [T.test_softmax_of_constant_values, T.test_worked_three_tokens]),
    "padding_keys_not_masked": (
        "mask = mask & (k_idx[None, :] >= lo) & (q_idx[:, None] >= lo)",
        "mask = mask & (q_idx[:, None] >= lo)",
        [T.test_left_padding_equals_sequence_alone, T.test_padding_onehot_probe_counts]),
    "padding_rows_not_zeroed": (
        "& (q_idx[:, None] >= lo) & (q_idx[:, None] < hi)", "",
        [T.test_right_padding_rows_zero_and_rest_causal]),
    "int8_scale_over_128": (
        "amax / np.float32(127.0)", "amax / np.float32(128.0)",
        [T8.test_exact_on_codes_times_power_of_two]),
    "int8_codes_truncated": (
        "c = np.rint((x / safe[..., None]).astype(np.float32))",
        "c = np.trunc((x / safe[..., None]).astype(np.float32))",
        [T8.test_codes_are_nearest_integers_brute_force, T8.test_exact_halves_round_to_even]),
    "int8_ties_away_from_zero": (
        "c = np.rint((x / safe[..., None]).astype(np.float32))",
        "c = np.floor((x / safe[..., None]).astype(np.float32) + 0.5)",
        [T8.test_exact_halves_round_to_even]),
    "int8_dequant_drops_scale": (
        "return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]",
        "return np.asarray(codes, dtype=np.float64)",
        [T8.test_round_trip_within_half_step_and_extremes,
         T8.test_int8_decode_equals_float_decode_on_representable_cache]),
    "chunk_queries_at_local_positions": (
        "q_idx = P + rows                            # chunk token i: token P + i",
        "q_idx = rows",
        [TC.test_chunk_equals_rows_of_whole_prompt, TC.test_chunk_onehot_counts]),
    "chunk_sees_only_prefix": (
        "n = P + C                                   # cache rows the chunk can see", "n = max(P, 1)",
        [TC.test_chunk_equals_rows_of_whole_prompt]),
    "transformed_keys_normed_again": (
        """            assert not f["k_eq_v"], "tied values need the raw keys"
            kt = kc
        else:
            kt = rope(rms_norm(kc, w_k, f["mode"], f["eps"]), pos_k[:, None],""",
        """            assert not f["k_eq_v"], "tied values need the raw keys"
            kt = rms_norm(kc, w_k, f["mode"], f["eps"])
        else:
            kt = rope(rms_norm(kc, w_k, f["mode"], f["eps"]), pos_k[:, None],""",
        [TT.test_decode_over_transformed_keys_equals_raw]),
    "int8_values_from_key_codes": (
        "else deq(v_codes, v_scales)", "else deq(k_codes, v_scales)",
        [T8.test_int8_decode_equals_float_decode_on_representable_cache]),
}


def _mutated_module(old, new):
    text = inspect.getsource(src_mod)
    assert text.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(text.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _call(pin):
    params = inspect.signature(pin).parameters
    if not params:
        return pin()
    # parametrised pins: run their first parametrisation
    marks = [m for m in getattr(pin, "pytestmark", []) if m.name == "parametrize"]
    for m in marks:
        names = [n.strip() for n in m.args[0].split(",")]
        for values in m.args[1]:
            values = values if isinstance(values, tuple) else (values,)
            pin(**dict(zip(names, values)))
    return None


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    old, new, pins = MUTATIONS[name]
    mut = _mutated_module(old, new)
    for attr in oracle.__all__:
        monkeypatch.setattr(oracle, attr, getattr(mut, attr))
    for pin in pins:
        with pytest.raises(AssertionError):
            _call(pin)


def test_unmutated_pins_pass():
    for _, _, pins in MUTATIONS.values():
        for pin in pins:
            _call(pin)
