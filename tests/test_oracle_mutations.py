"""Pin strength (CPU only): plausible mistakes planted in a copy of the oracle
each make at least one of the pins that are meant to catch them fail.  The
oracle itself is never modified; each mutant is a fresh module built from the
oracle's source with one edit, handed to the pin tests in place of the real
one for the duration of the check."""
import importlib
import inspect
import os
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "oracle", "nvfp4_oracle.py")).read()
GOLDEN = os.path.join(ROOT, "tests", "golden")

# (what the mistake is, oracle function, text, replacement, pin module, pins)
MUTANTS = [
    ("E2M1 ties to the odd code", "e2m1_encode", "(hi % 2 == 0)", "(hi % 2 == 1)", "test_oracle_codecs",
     ["test_e2m1_rounding_golden", "test_e2m1_vs_exact_rational_sweep"]),
    ("E2M1 sign dropped", "e2m1_encode", "code + 8 * sign", "code + 0 * sign", "test_oracle_codecs",
     ["test_e2m1_roundtrip_all_codes", "test_e2m1_rounding_golden"]),
    ("E4M3 ties to the odd code", "e4m3_encode_nonneg", "(hi % 2 == 0)", "(hi % 2 == 1)", "test_oracle_codecs",
     ["test_e4m3_rounding_golden", "test_e4m3_roundtrip_and_midpoints"]),
    ("global scale amax / 448", "global_scale", "E2M1_MAX * E4M3_MAX", "E4M3_MAX", "test_oracle_quantize",
     ["test_global_scale_closed_form", "test_tensor_max_block_gets_448"]),
    ("block scale amax_b / 4", "quantize", "(amax_b / np.float32(6.0)) / g", "(amax_b / np.float32(4.0)) / g",
     "test_oracle_quantize", ["test_tensor_max_block_gets_448", "test_block_max_maps_to_the_top_code"]),
    ("element scale without g", "quantize", "denom = (S * g)", "denom = (S * np.float32(1.0))",
     "test_oracle_quantize", ["test_per_element_error_bound", "test_all_equal_blocks"]),
    ("nibbles swapped", "pack_codes", "c[:, 0::2] | (c[:, 1::2] << 4)", "c[:, 1::2] | (c[:, 0::2] << 4)",
     "test_oracle_quantize", ["test_pack_unpack_nibble_order"]),
    ("GEMM against reversed weight rows", "gemm", "acc = a @ w.T", "acc = a @ w[::-1].T", "test_oracle_gemm",
     ["test_gemm_exact_vs_brute_force", "test_gemm_is_not_transposed"]),
    ("magnitude sum without absolute values", "gemm", "mag = np.abs(a) @ np.abs(w).T", "mag = a @ w.T",
     "test_oracle_gemm", ["test_magnitude_sum_bounds_accumulation"]),
    ("sigmoid branches swapped", "sigmoid", "np.where(t >= 0, 1.0 / (1.0 + e), e / (1.0 + e))",
     "np.where(t >= 0, e / (1.0 + e), 1.0 / (1.0 + e))", "test_oracle_gemm", ["test_sigmoid_softplus_closed_forms"]),
    ("decay sign lost", "gdn_decay", "return -np.exp(", "return np.exp(", "test_oracle_gemm",
     ["test_gdn_decay_closed_form"]),
    ("SwiGLU without the gate factor", "swiglu", "gate * sigmoid(gate) *", "sigmoid(gate) *", "test_oracle_gemm",
     ["test_swiglu_closed_form"]),
    ("requantise with the new scale", "requantize", "vals.reshape(M, K) * g_rows", "vals.reshape(M, K) * np.float64(g_new)",
     "test_oracle_requant", ["test_rows_use_their_own_module_scale", "test_power_of_two_scale_change_halves_block_scales"]),
    ("KV encode multiplies by the scale", "kv_fp8_quantize", "inv = np.float32(1) / s", "inv = s", "test_oracle_kvfp8",
     ["test_every_code_round_trips_under_power_of_two_scales", "test_half_step_relative_error_in_the_normal_range"]),
    ("dominance on signed values", "activation_stats", "ab = np.abs(x64).reshape", "ab = x64.reshape",
     "test_oracle_actstats", ["test_tiny_tensor_by_hand", "test_dominated_blocks_and_exact_values"]),
    ("delta rule without the decay on the correction", "gdn_recurrence", "(v[t] - a[:, None] * Sk)", "(v[t] - Sk)",
     "test_oracle_gdn", ["test_scalar_closed_form", "test_chunked_form_agrees"]),
    ("state not decayed", "gdn_recurrence", "S = a[:, None, None] * S + u", "S = S + u", "test_oracle_gdn",
     ["test_pure_decay_closed_form", "test_chunked_form_agrees"]),
    ("output read with the key", 'gdn_recurrence', 'np.einsum("hvk,hk->hv", S, qh[t])', 'np.einsum("hvk,hk->hv", S, kh[t])',
     "test_oracle_gdn", ["test_pure_decay_closed_form", "test_orthonormal_keys_give_linear_attention"]),
    ("value heads mapped to q/k heads cyclically", "gdn_recurrence", "qh = np.repeat(q, rep, axis=1)",
     "qh = np.tile(q, (1, rep, 1))", "test_oracle_gdn", ["test_shared_query_key_heads"]),
    ("write strength not applied", "gdn_recurrence", "u = beta[t][:, None] * (", "u = (", "test_oracle_gdn",
     ["test_orthonormal_keys_give_linear_attention", "test_chunked_form_agrees"]),
    ("L2 norm without the square root", "l2_normalise", "np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)",
     "((x * x).sum(axis=-1, keepdims=True) + eps)", "test_oracle_gdn",
     ["test_write_overwrites_along_the_key", "test_pure_decay_closed_form"]),
    ("E2M1 exponent bias off by one", "e2m1_value", "2.0 ** (e - 1)", "2.0 ** e", "test_oracle_codecs",
     ["test_e2m1_values_match_golden", "test_e2m1_decode_table_vs_ml_dtypes"]),
    ("E4M3 exponent bias off by one", "e4m3_value", "2.0 ** (e - 7)", "2.0 ** (e - 8)", "test_oracle_codecs",
     ["test_e4m3_values_match_golden", "test_e4m3_decode_all_256_vs_torch"]),
    ("E4M3 subnormal step wrong", "e4m3_value", "(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7",
     "test_oracle_codecs", ["test_e4m3_values_match_golden", "test_e4m3_decode_all_256_vs_torch"]),
    ("dequantise without the global scale", "dequantize", "* np.float64(g)", "* 1.0", "test_oracle_quantize",
     ["test_per_element_error_bound", "test_quant_error_magnitude_sane"]),
    ("every segment takes the first segment's scale", "fused_projection", "np.float64(seg_scales[s])",
     "np.float64(seg_scales[0])", "test_oracle_gemm", ["test_fused_projection_equals_per_module_linears"]),
    ("SwiGLU paired with itself", "fused_projection", 'up = epilogues.index("swiglu_up")', "up = s",
     "test_oracle_gemm", ["test_swiglu_pairing_in_fused_projection"]),
    ("common scale is the largest", "common_global_scale", "np.min(", "np.max(", "test_oracle_gemm",
     ["test_common_scale_mismatch_closed_form"]),
    ("KV decode divides by the scale", "kv_fp8_dequantize", "v * np.float32(scale)", "v / np.float32(scale)",
     "test_oracle_kvfp8", ["test_bad_scale_gives_zeros_and_decoding_matches_torch",
                           "test_every_code_round_trips_under_power_of_two_scales"]),
    ("kurtosis over the variance", "activation_summary", "m4c / var ** 2", "m4c / var", "test_oracle_actstats",
     ["test_gaussian_and_heavy_tailed_moments"]),
    ("hot channel against the mean channel", "activation_summary", "col_rms.max() / med",
     "col_rms.max() / col_rms.mean()", "test_oracle_actstats", ["test_a4_error_within_the_half_step_bound_and_hot_channel"]),
    ("BF16 rounding truncates", "bf16_round", "np.round(y / q) * q", "np.floor(y / q) * q", "test_oracle_gemm",
     ["test_bf16_round_and_ulp"]),
]


def _mutant(func, old, new):
    start = SRC.index(f"\ndef {func}(")
    end = SRC.find("\ndef ", start + 1)
    end = len(SRC) if end < 0 else end
    body = SRC[start:end]
    assert body.count(old) >= 1, (func, old)
    src = SRC[:start] + body.replace(old, new, 1) + SRC[end:]
    mod = types.ModuleType("nvfp4_oracle_mutant")
    exec(compile(src, "nvfp4_oracle_mutant.py", "exec"), mod.__dict__)
    return mod


def _run(fn):
    kwargs = {}
    params = inspect.signature(fn).parameters
    if "golden_dir" in params:
        kwargs["golden_dir"] = GOLDEN
    if "seed" in params:
        kwargs["seed"] = 0
    fn(**kwargs)


@pytest.mark.parametrize("what,func,old,new,module,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(what, func, old, new, module, pins, monkeypatch):
    tests = importlib.import_module(f"tests.{module}")
    for name in pins:  # the pins pass on the real oracle
        _run(getattr(tests, name))
    monkeypatch.setattr(tests, "o", _mutant(func, old, new))
    caught = []
    for name in pins:
        try:
            _run(getattr(tests, name))
        except Exception:  # an assertion, or the mutant breaking a shape or range check
            caught.append(name)
    assert caught, f"no pin caught: {what}"
