"""Helpers shared by the GPU parity tests: reading the library's outputs back
into the oracle's logical layout, and the comparison rules.

Tolerances (the accumulation bound of 1e-5 * sum_k |a_k w_k| per output in
FP32, or one BF16 ulp after the epilogue):
  * FP32 pre-activations: |gpu - y| <= 1e-5 * mag, mag = sum_k |a_k w_k| g_a g_w.
  * BF16 results: |gpu - bf16(y)| <= 1 BF16 ulp, or, where the accumulation
    bound itself exceeds half an ulp, |gpu - y| <= ulp/2 + tol (counted).
  * sigmoid: |d beta| <= tol / 4 + 4 FP32 ulp.
  * decay -exp(A_log) softplus(t): |d| <= exp(A_log) sigmoid(t) (tol + ulp(t)) + 8 FP32 ulp.
  * SwiGLU: the BF16 rule with tol propagated through silu(g) * u.
"""
import numpy as np
import torch

from oracle import nvfp4_oracle as o

TOL_ACC = 1e-5


def unswizzle_sf(sf: np.ndarray, rows: int, K: int):
    """Scale bytes in the tcgen05 block-scale layout -> logical [rows_pad, KA*4]."""
    KA = (K + 63) // 64
    rows_pad = (rows + 127) // 128 * 128
    r = np.arange(rows_pad)[:, None]
    j = np.arange(KA * 4)[None, :]
    idx = ((r // 128) * KA + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    assert sf.size == rows_pad * KA * 4
    return sf[idx]


def operand_to_logical(op, rows: int, K: int):
    """(codes uint8[rows, K] one code per element, sf uint8[rows, K/16], sf_full)."""
    packed = op.codes.cpu().numpy()
    codes = o.unpack_codes(packed)[:rows, :K]
    full = unswizzle_sf(op.sf.cpu().numpy(), rows, K)
    return codes, full[:rows, : K // 16], full


def assert_quant_equal(op, g_gpu, x_np, g_in=None, rows=None):
    """Bit-exact comparison of a library quantisation with the oracle's."""
    M, K = x_np.shape
    codes, sf, full = operand_to_logical(op, M, K)
    oc, osf, og = o.quantize(x_np, g_in)
    g = float(g_gpu.cpu().numpy().reshape(-1)[0])
    assert np.float32(g).tobytes() == np.float32(og).tobytes(), (g, og)
    bad_sf = np.argwhere(sf != osf)
    assert bad_sf.size == 0, f"{len(bad_sf)} scale mismatches, first {bad_sf[:5].tolist()}"
    bad = np.argwhere(codes != oc)
    assert bad.size == 0, f"{len(bad)} code mismatches, first {bad[:5].tolist()} gpu {codes[tuple(bad[0])]} oracle {oc[tuple(bad[0])]}"
    # padding of the scale layout is zero
    pad = full.copy()
    pad[:M, : K // 16] = 0
    assert not pad.any()


def f32_ulp(v):
    v = np.abs(np.asarray(v, np.float64)).astype(np.float32)
    return np.spacing(np.maximum(v, np.float32(1.1754944e-38))).astype(np.float64)


def check_fp32(gpu, y, mag, label=""):
    gpu = np.asarray(gpu, np.float64)
    tol = TOL_ACC * mag + 1e-30
    err = np.abs(gpu - y)
    ratio = err / tol
    assert np.all(err <= tol), f"{label}: max err/tol {ratio.max():.3g} at {np.unravel_index(np.argmax(ratio), ratio.shape)}"
    return float(ratio.max())


def check_bf16(gpu, y, tol, label=""):
    """Returns (max ratio of |gpu - bf16(y)| to one ulp, elements that needed tol)."""
    gpu = np.asarray(gpu, np.float64)
    yb = o.bf16_round(y)
    ulp = o.bf16_ulp(yb)
    strict = np.abs(gpu - yb) <= ulp
    loose = np.abs(gpu - y) <= 0.5 * o.bf16_ulp(gpu) + tol
    ok = strict | loose
    assert np.all(ok), f"{label}: {np.count_nonzero(~ok)} BF16 mismatches, e.g. gpu {gpu[~ok][:4]} ref {y[~ok][:4]}"
    return float((np.abs(gpu - yb) / ulp).max()), int(np.count_nonzero(~strict))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)
