"""Pins for the oracle's FP8 (E4M3) KV-cache codec (CPU only).

What fixes it, independently of its code:
  * every finite E4M3 value times a power-of-two scale encodes to its own code
    (and decodes back exactly);
  * each encoded value is the representable value nearest to x / scale, ties
    to the even code, by brute force over the whole E4M3 table;
  * values beyond 448 * scale saturate to +-448; the sign is symmetric and
    the sign of zero is kept;
  * the round trip of a value in the normal range errs by at most half an
    E4M3 step (2^-4 relative);
  * a non-positive scale gives all-zero codes; dequantisation agrees with
    torch's float8_e4m3fn decoding.
"""
import numpy as np
import torch

from oracle import nvfp4_oracle as o

FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_every_code_round_trips_under_power_of_two_scales():
    for s in (2.0 ** -7, 0.25, 1.0, 8.0):
        vals = np.array([o.e4m3_value(c) * s for c in FINITE], np.float32)
        codes = o.kv_fp8_quantize(vals, s)
        assert np.array_equal(codes, np.array(FINITE, np.uint8))
        back = o.kv_fp8_dequantize(codes, s, "f32")
        assert np.array_equal(back, vals.astype(np.float64))


def _nearest_code(y):
    """Brute force over all finite codes: nearest value, ties to the even code,
    saturation at +-448, sign kept for zero."""
    table = np.array([o.e4m3_value(c) for c in range(128) if c != 0x7F])
    mag = min(abs(float(y)), 448.0)
    d = np.abs(table - mag)
    best = np.flatnonzero(d == d.min())
    c = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
    return c | (0x80 if np.signbit(y) else 0)


def test_nearest_value_ties_to_even_by_brute_force():
    rng = np.random.default_rng(3)
    s = np.float32(0.37)
    x = np.concatenate([rng.standard_normal(3000) * 50, rng.standard_normal(1000) * 0.01,
                        np.array([0.0, -0.0, 1e-30, -1e30, 500 * 0.37, -465 * 0.37])]).astype(np.float32)
    codes = o.kv_fp8_quantize(x, s)
    y = (x * (np.float32(1) / s)).astype(np.float32)
    ref = np.array([_nearest_code(v) for v in y], np.uint8)
    assert np.array_equal(codes, ref)


def test_saturation_sign_and_zero():
    s = np.float32(0.5)
    x = np.array([224.0, 225.0, 1e6, -1e6, 0.0, -0.0], np.float32)
    c = o.kv_fp8_quantize(x, s)
    assert list(c) == [0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80]
    rng = np.random.default_rng(4)
    v = rng.standard_normal(2000).astype(np.float32)
    assert np.array_equal(o.kv_fp8_quantize(-v, s), o.kv_fp8_quantize(v, s) ^ 0x80)


def test_half_step_relative_error_in_the_normal_range():
    rng = np.random.default_rng(5)
    s = np.float32(0.01)
    x = (rng.uniform(2.0 ** -6, 440, 5000) * s * rng.choice([-1, 1], 5000)).astype(np.float32)
    back = o.kv_fp8_dequantize(o.kv_fp8_quantize(x, s), s, "f32")
    assert np.all(np.abs(back - x) <= 2.0 ** -4 * np.abs(x) * (1 + 1e-6))


def test_bad_scale_gives_zeros_and_decoding_matches_torch():
    x = np.linspace(-3, 3, 64, dtype=np.float32)
    for s in (0.0, -1.0, np.inf, np.nan):
        assert not o.kv_fp8_quantize(x, s).any()
    codes = np.array(FINITE, np.uint8)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    assert np.array_equal(o.kv_fp8_dequantize(codes, 1.0, "f32"), t)
    tb = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).mul(0.3).to(torch.bfloat16)
    assert np.array_equal(o.kv_fp8_dequantize(codes, np.float32(0.3), "bf16"), tb.to(torch.float64).numpy())
