"""CPU oracle for the NVFP4 W4A4 linear layer — TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA library
and imports nothing from it.  Everything here is plain, slow numpy written from
the definitions, so that each step can be checked against the pages by eye.

What the pages fix (Paper summary page (ai.info), "Methodology in Plain
English"): NVFP4 stores 4-bit E2M1 values with one E4M3 scale per block of 16
consecutive elements, the largest value in a block fixes that block's scale,
and an outlier only affects its own block.  "Main Findings", fused-GEMM bullet:
one FP32 global scale per linear module; a fused GEMM over several modules must
keep each module's own global scale.  "Main Findings", gate-parameterisation
bullets: the write strength is a sigmoid of the b projection and the decay is
log-space, softplus then exponential, of the a projection.

Readings taken where the pages are silent:
  * global scale (dequantisation direction) g = amax(|x|) / (6 * 448), so the
    block holding the tensor maximum uses the full E4M3 range;
  * block scale byte = E4M3(RNE, saturating)((amax_block / 6) / g), FP32;
  * element codes = E2M1(RNE, saturating)(x * inv), inv = 1 / (S * g) in FP32
    (0 when S*g == 0, clamped to FLT_MAX), S the decoded block scale;
  * the sign of a value that rounds to magnitude 0 is kept (code 0x8);
  * g <= 0 (an all-zero tensor) gives all-zero codes and scale bytes;
  * GEMM and epilogues in FP64 on the dequantised operands;
  * decay gate: g = -exp(A_log[h]) * softplus(y + dt_bias[h]), head h = column
    within the segment; SwiGLU: silu(gate) * up;
  * delta-rule recurrence (the consumer of the projection's q, k, v, beta, g):
    one state S[d_v, d_k] per value head, alpha = exp(g),
    S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T and
    o_t = S_t q_t, with k and q L2-normalised per head (x / sqrt(sum x^2 + eps))
    and q scaled by d_k^-1/2; value head h reads query/key head h // (H / H_k).

Parity pins for every function live in tests/test_oracle_*.py.
"""
from __future__ import annotations


import numpy as np

FLT_MAX = np.float32(3.4028234663852886e38)
E2M1_MAX = 6.0
E4M3_MAX = 448.0
BLOCK = 16  # elements per block scale

# --------------------------------------------------------------------------
# E2M1 (FP4): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
# Codes 0..7 are the non-negative values, bit 3 is the sign.
# exponent field 0 is subnormal: value = m * 0.5; otherwise (1 + m/2) * 2^(e-1).
# --------------------------------------------------------------------------


def e2m1_value(code: int) -> float:
    """Decode one 4-bit E2M1 code from its bit fields."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


E2M1_GRID = np.array([e2m1_value(c) for c in range(8)], dtype=np.float64)  # 0,.5,1,1.5,2,3,4,6
E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Round float32 values to E2M1 codes: nearest grid value, ties to the even
    code (mantissa bit 0), magnitudes above 6 (and inf) saturate to 6, the sign
    bit is the sign of the input (so -0 and small negatives give 0x8)."""
    v = np.asarray(v, dtype=np.float32)
    mag = np.abs(v).astype(np.float64)
    # hi = index of the smallest grid value >= mag (clamped to the top code)
    hi = np.searchsorted(E2M1_GRID, mag, side="left")
    hi = np.minimum(hi, 7)
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - E2M1_GRID[lo]
    d_hi = E2M1_GRID[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= E2M1_GRID[7], 7, code)  # saturation, inf included
    code = np.where(mag == E2M1_GRID[hi], hi, code)  # exact grid hits
    sign = np.signbit(v).astype(np.int64)
    return (code + 8 * sign).astype(np.uint8)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_TABLE[np.asarray(codes, dtype=np.int64) & 15]


# --------------------------------------------------------------------------
# E4M3 (OCP FP8 "e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
# no infinities, 0x7F/0xFF are NaN, largest finite 448 (0x7E).
# exponent field 0 is subnormal: value = m/8 * 2^-6.
# --------------------------------------------------------------------------


def e4m3_value(code: int) -> float:
    s = (code >> 7) & 1
    e = (code >> 3) & 15
    m = code & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
E4M3_POS = E4M3_TABLE[:127]  # codes 0..126, increasing, all finite


def e4m3_encode_nonneg(v: np.ndarray) -> np.ndarray:
    """Round non-negative float32 values to E4M3 bytes: nearest finite value,
    ties to the even code, values above 448 (and inf) saturate to 0x7E."""
    mag = np.asarray(v, dtype=np.float32).astype(np.float64)
    if np.any(mag < 0) or np.any(np.isnan(mag)):
        raise ValueError("block scales are non-negative and finite or +inf")
    hi = np.searchsorted(E4M3_POS, mag, side="left")
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - E4M3_POS[lo]
    d_hi = E4M3_POS[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= E4M3_MAX, 126, code)
    code = np.where(mag == E4M3_POS[hi], hi, code)
    return code.astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.int64)]


# --------------------------------------------------------------------------
# Scales and quantisation
# --------------------------------------------------------------------------


def global_scale(x: np.ndarray) -> np.float32:
    """FP32 per-tensor (activations) or per-module (weights) global scale,
    dequantisation direction: g = amax / (6 * 448), in FP32."""
    amax = np.float32(np.max(np.abs(np.asarray(x, dtype=np.float32)))) if np.size(x) else np.float32(0)
    return np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX))


def quantize(x: np.ndarray, g=None):
    """Quantise x[M, K] (float32 values) into NVFP4 along K.

    Returns (codes uint8[M, K] one code per element, sf uint8[M, K/16], g float32).
    Steps (all FP32, IEEE round-to-nearest), per block of 16 along K:
      amax_b = max |x|;  s_raw = (amax_b / 6) / g;  sf = E4M3(s_raw);  S = dec(sf)
      denom = S * g;  inv = 1/denom (0 if denom == 0, at most FLT_MAX)
      code  = E2M1(x * inv)
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = global_scale(x) if g is None else np.float32(g)
    B = K // BLOCK
    if not (g > 0):
        return np.zeros((M, K), np.uint8), np.zeros((M, B), np.uint8), g
    xb = x.reshape(M, B, BLOCK)
    amax_b = np.max(np.abs(xb), axis=2)  # float32, exact
    with np.errstate(over="ignore"):
        s_raw = (amax_b / np.float32(6.0)) / g  # float32 divisions
    sf = e4m3_encode_nonneg(s_raw)
    S = e4m3_decode(sf).astype(np.float32)  # exact in float32
    denom = (S * g).astype(np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        inv = np.where(denom > 0, np.float32(1.0) / np.where(denom > 0, denom, np.float32(1)), np.float32(0))
    inv = np.minimum(inv.astype(np.float32), FLT_MAX)
    with np.errstate(over="ignore"):
        q = (xb * inv[:, :, None]).astype(np.float32)
    codes = e2m1_encode(q).reshape(M, K)
    return codes, sf, g


def dequantize(codes: np.ndarray, sf: np.ndarray, g) -> np.ndarray:
    """x_hat = e2m1(code) * S * g in FP64 (exact products)."""
    M, K = codes.shape
    vals = e2m1_decode(codes).reshape(M, K // BLOCK, BLOCK)
    S = e4m3_decode(sf)[:, :, None]
    return (vals * S).reshape(M, K) * np.float64(g)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte along K: element 2j in the low nibble, 2j+1 in the high."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


# --------------------------------------------------------------------------
# GEMM and epilogues
# --------------------------------------------------------------------------


def block_scaled_operand(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """e2m1(code) * S in FP64, without the global scale."""
    return dequantize(codes, sf, 1.0)


def gemm(a_codes, a_sf, w_codes, w_sf):
    """acc[m, n] = sum_k (e2m1(qa)*Sa)(e2m1(qw)*Sw) in FP64, plus the
    magnitude sum sum_k |.| |.| that scales the accumulation tolerance."""
    a = block_scaled_operand(a_codes, a_sf)
    w = block_scaled_operand(w_codes, w_sf)
    acc = a @ w.T
    mag = np.abs(a) @ np.abs(w).T
    return acc, mag


def sigmoid(t):
    t = np.asarray(t, dtype=np.float64)
    e = np.exp(-np.abs(t))
    return np.where(t >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def softplus(t):
    t = np.asarray(t, dtype=np.float64)
    return np.maximum(t, 0.0) + np.log1p(np.exp(-np.abs(t)))


def gdn_decay(y, a_log, dt_bias):
    """Decay gate in log space: -exp(A_log[h]) * softplus(y + dt_bias[h]);
    y[..., h] is head h."""
    return -np.exp(np.asarray(a_log, np.float64)) * softplus(np.asarray(y, np.float64) + np.asarray(dt_bias, np.float64))


def swiglu(gate, up):
    gate = np.asarray(gate, np.float64)
    return gate * sigmoid(gate) * np.asarray(up, np.float64)


def linear(x, w, g_a=None, g_w=None):
    """Full W4A4 linear of one module: quantise x and w, FP64 GEMM, global scales.
    Returns (y, mag_scaled, (a_codes, a_sf, g_a), (w_codes, w_sf, g_w))."""
    a_codes, a_sf, g_a = quantize(x, g_a)
    w_codes, w_sf, g_w = quantize(w, g_w)
    acc, mag = gemm(a_codes, a_sf, w_codes, w_sf)
    s = np.float64(g_a) * np.float64(g_w)
    return acc * s, mag * s, (a_codes, a_sf, g_a), (w_codes, w_sf, g_w)


def fused_projection(a_q, w_q_segments, seg_scales, epilogues, gate_params=None):
    """One GEMM over concatenated weight segments; segment s's columns are scaled
    by g_a * seg_scales[s] and then pass through that segment's epilogue.

    a_q = (codes, sf, g_a); w_q_segments = [(codes, sf), ...] in column order;
    epilogues[s] in {"identity", "sigmoid", "gdn_decay", "swiglu_gate", "swiglu_up"}.
    Returns (outputs, pre) where outputs maps segment index -> FP64 result (SwiGLU
    pairs produce one output under the gate's index) and pre maps segment index
    -> (pre-activation y, magnitude sum) both already scaled.
    """
    a_codes, a_sf, g_a = a_q
    pre = {}
    for s, (wc, ws) in enumerate(w_q_segments):
        acc, mag = gemm(a_codes, a_sf, wc, ws)
        scale = np.float64(g_a) * np.float64(seg_scales[s])
        pre[s] = (acc * scale, mag * scale)
    outputs = {}
    for s, epi in enumerate(epilogues):
        y = pre[s][0]
        if epi == "identity":
            outputs[s] = y
        elif epi == "sigmoid":
            outputs[s] = sigmoid(y)
        elif epi == "gdn_decay":
            a_log, dt_bias = gate_params
            outputs[s] = gdn_decay(y, a_log[None, :], dt_bias[None, :])
        elif epi == "swiglu_gate":
            up = epilogues.index("swiglu_up")
            outputs[s] = swiglu(y, pre[up][0])
        elif epi == "swiglu_up":
            pass
        else:
            raise ValueError(epi)
    return outputs, pre


def common_global_scale(seg_scales) -> np.float32:
    """The single scale a fused serving kernel applies when it takes the
    largest encode-direction scale of the fused modules (Paper summary page
    (ai.info), "Main Findings", fused-GEMM bullet).  In the dequantisation
    direction used here that is the smallest g."""
    return np.float32(np.min(np.asarray(seg_scales, np.float32)))


def requantize(codes: np.ndarray, sf: np.ndarray, g_rows, g_new):
    """Checkpoint-side harmonisation of fused modules' scales (Paper summary
    page (ai.info), "Methodology in Plain English": the fused modules' global
    scales are made to agree on the checkpoint side, so that a kernel applying
    one scale to the fused GEMM is correct).  Reading: every element is
    dequantised with its own module's scale, rounded once to FP32
    (x_hat = e2m1 * S * g_old; e2m1 * S is exact), and the result is quantised
    again with the common scale g_new exactly as quantize() does.  The common
    scale that clips nothing is the largest module scale, which is the scale
    of the fused (concatenated) weight; a smaller one makes the larger
    modules' block scales saturate.

    g_rows: the old global scale of each row (float32[M]) or one scalar.
    Returns (codes, sf, g_new) like quantize().
    """
    codes = np.asarray(codes, np.uint8)
    M, K = codes.shape
    g_rows = np.broadcast_to(np.asarray(g_rows, np.float64).reshape(-1, 1) if np.ndim(g_rows) else
                             np.float64(g_rows), (M, 1))
    vals = e2m1_decode(codes).reshape(M, K // BLOCK, BLOCK) * e4m3_decode(sf)[:, :, None]  # exact
    x_hat = (vals.reshape(M, K) * g_rows).astype(np.float32)  # one rounding to FP32
    return quantize(x_hat, np.float32(g_new))


def kv_fp8_quantize(x: np.ndarray, scale) -> np.ndarray:
    """FP8 (E4M3) KV-cache codec with a calibrated static per-tensor scale
    (Paper summary page (ai.info), "Main Findings", KV-cache bullet: an FP8
    KV cache whose scales are calibrated, not left at 1.0).  Reading, in FP32:
    inv = 1 / scale (once), y = x * inv, code = sign(y) | E4M3_rn_satfinite(|y|),
    the sign of zero kept; scale <= 0 (or not finite) gives all-zero codes."""
    x = np.asarray(x, dtype=np.float32)
    s = np.float32(scale)
    if not (np.isfinite(s) and s > 0):
        return np.zeros(x.shape, np.uint8)
    inv = np.float32(1) / s
    with np.errstate(over="ignore"):
        y = (x * inv).astype(np.float32)
    mag = e4m3_encode_nonneg(np.abs(y))
    return (mag | (np.signbit(y).astype(np.uint8) << 7)).astype(np.uint8)


def kv_fp8_dequantize(codes: np.ndarray, scale, out_dtype: str = "bf16") -> np.ndarray:
    """x_hat = e4m3(code) * scale rounded to FP32, then to BF16 when the output
    is BF16 (returned as float64 holding the rounded values)."""
    v = e4m3_decode(codes).astype(np.float32)
    y = (v * np.float32(scale)).astype(np.float32).astype(np.float64)
    return bf16_round(y) if out_dtype == "bf16" else y


def activation_stats(x: np.ndarray, g=None) -> dict:
    """Activation statistics at NVFP4 granularity (Paper summary page
    (ai.info), "Main Findings", activation bullet: max/RMS, kurtosis, hot
    channels against the median channel, the share of 16-element blocks
    dominated by a single value, and the per-token A4 quantisation error).
    Readings: a block is dominated when its largest magnitude exceeds the sum
    of the other fifteen; the A4 error of a token is ||x - x_hat|| / ||x||
    with x_hat the NVFP4 dequantisation under the tensor's global scale g (the
    quantiser's; computed from x when not given); moments in FP64."""
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    x64 = x.astype(np.float64)
    ab = np.abs(x64).reshape(M, K // BLOCK, BLOCK)
    amax_b = ab.max(axis=2)
    dominated = amax_b > (ab.sum(axis=2) - amax_b)
    codes, sf, gq = quantize(x, g)
    x_hat = dequantize(codes, sf, gq).astype(np.float32).astype(np.float64)
    return {
        "n": float(M * K), "sum": x64.sum(), "sum_sq": (x64 ** 2).sum(), "sum_cube": (x64 ** 3).sum(),
        "sum_4th": (x64 ** 4).sum(), "amax": np.abs(x64).max() if x.size else 0.0,
        "blocks": float(amax_b.size), "dominated": float(dominated.sum()),
        "row_err2": ((x64 - x_hat) ** 2).sum(axis=1), "row_norm2": (x64 ** 2).sum(axis=1),
        "col_sq": (x64 ** 2).sum(axis=0), "col_max": np.abs(x64).max(axis=0),
    }


def activation_summary(st: dict) -> dict:
    """Derived figures of activation_stats(): max/RMS, kurtosis (fourth central
    moment over the squared variance), dominated-block share, per-token A4
    error (mean, min, max) and the hot-channel ratio (largest channel RMS over
    the median channel RMS)."""
    n = st["n"]
    mean = st["sum"] / n
    m2 = st["sum_sq"] / n
    var = m2 - mean ** 2
    m4c = st["sum_4th"] / n - 4 * mean * st["sum_cube"] / n + 6 * mean ** 2 * m2 - 3 * mean ** 4
    norm = np.sqrt(st["row_norm2"])
    err = np.sqrt(st["row_err2"]) / np.where(norm > 0, norm, 1.0)
    col_rms = np.sqrt(np.asarray(st["col_sq"]) * (len(st["row_norm2"]) and 1.0 / len(st["row_norm2"])))
    med = np.median(col_rms)
    return {"max_over_rms": st["amax"] / np.sqrt(m2) if m2 > 0 else 0.0,
            "kurtosis": m4c / var ** 2 if var > 0 else 0.0,
            "dominated_share": st["dominated"] / st["blocks"] if st["blocks"] else 0.0,
            "a4_err_mean": float(err.mean()) if err.size else 0.0,
            "a4_err_min": float(err.min()) if err.size else 0.0,
            "a4_err_max": float(err.max()) if err.size else 0.0,
            "hot_channel_ratio": float(col_rms.max() / med) if med > 0 else 0.0}


# --------------------------------------------------------------------------
# Gated delta-rule recurrence (Paper summary page (ai.info), "Main Findings",
# recurrence bullet: a fixed-size state in which every write overwrites along
# the current key direction, with a decay alpha and a write strength beta;
# gate-parameterisation bullet: alpha comes from the log-space decay gate g,
# alpha = exp(g)).  The plain token-by-token definition, in FP64.
# --------------------------------------------------------------------------


def l2_normalise(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(sum(x^2) + eps) along the last axis, FP64."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def gdn_recurrence(q, k, v, beta, g, h0=None, scale=None, eps=1e-6, normalise=True, row_norms=False):
    """Run the gated delta rule over T tokens.

    q, k: [T, H_k, d_k]; v: [T, H, d_v]; beta, g: [T, H] (write strength and
    log-space decay, as the projection's epilogue emits them); h0: [H, d_v, d_k]
    or None (zeros).  Value head h uses query/key head h // (H / H_k).
    Returns (o [T, H, d_v], S_T [H, d_v, d_k]) and, with row_norms, also
    |S_t[i, :]|_2 for every token ([T, H, d_v]): the natural size of o_t[i],
    since |o_t[i]| <= |S_t[i, :]| * |q_t|.

    Per token, with alpha = exp(g_t):
        u   = beta_t * (v_t - alpha * S_{t-1} k_t)      (the correction written)
        S_t = alpha * S_{t-1} + u k_t^T
        o_t = S_t q_t
    which is S_t = alpha S_{t-1} (I - beta k k^T) + beta v k^T written out."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    T, H, dv = v.shape
    hk, dk = q.shape[1], q.shape[2]
    assert k.shape == q.shape and H % hk == 0 and beta.shape == (T, H) and g.shape == (T, H)
    rep = H // hk
    qh = np.repeat(q, rep, axis=1)
    kh = np.repeat(k, rep, axis=1)
    if normalise:
        qh = l2_normalise(qh, eps)
        kh = l2_normalise(kh, eps)
    qh = qh * (dk ** -0.5 if scale is None else scale)
    S = np.zeros((H, dv, dk)) if h0 is None else np.array(h0, dtype=np.float64)
    o = np.empty((T, H, dv))
    rn = np.empty((T, H, dv)) if row_norms else None
    for t in range(T):
        a = np.exp(g[t])
        Sk = np.einsum("hvk,hk->hv", S, kh[t])
        u = beta[t][:, None] * (v[t] - a[:, None] * Sk)
        S = a[:, None, None] * S + u[:, :, None] * kh[t][:, None, :]
        o[t] = np.einsum("hvk,hk->hv", S, qh[t])
        if row_norms:
            rn[t] = np.sqrt((S * S).sum(axis=2))
    if row_norms:
        return o, S, rn
    return o, S


def bf16_round(y) -> np.ndarray:
    """Round FP64 values to BF16 (8 significant bits, nearest, ties to even);
    returned as FP64.  y = m * 2^e with 0.5 <= |m| < 1, so y / 2^(e-8) has its
    8 significant bits in the integer part; np.round rounds halves to even."""
    y = np.asarray(y, dtype=np.float64)
    _, e = np.frexp(y)
    e = np.maximum(e, -125)  # BF16 subnormals share the quantum 2^-133
    q = np.ldexp(1.0, e - 8)
    return np.round(y / q) * q


def bf16_ulp(y) -> np.ndarray:
    """Spacing of BF16 values in the binade of |y|."""
    _, e = np.frexp(np.asarray(y, dtype=np.float64))
    return np.ldexp(1.0, np.maximum(e, -125) - 8)
