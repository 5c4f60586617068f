"""Seeded synthetic inputs for the NVFP4 W4A4 linear layer.

This module only draws random numbers and arranges them into the shapes of the
five workloads; it holds none of the quantisation or GEMM arithmetic, so both
the CUDA path and the CPU oracle can take their inputs from it.

The pages measure on captured activations of a 27B hybrid model, which are not
available; these inputs stand in for them.  They copy the statistics the pages
report for the residual stream (Paper summary page (ai.info), "Main Findings",
activation-statistics bullet: hot channels about 100x the median channel):
N(0,1) activations with a few outlier channels scaled by x50 or x100, and
N(0, 0.02) weights.

Recipe (every draw uses ``numpy.random.default_rng``):
  * X: ``rng = default_rng(seed)``; first the outlier channel indices
    (``rng.choice(K, n_outlier, replace=False)``, unless the workload fixes
    them), then ``rng.standard_normal((M, K), float32)``; outlier columns are
    multiplied by their factor; BF16 workloads round to BF16 (RNE).
  * Weight segment s (0-based): ``0.02 * default_rng(seed + 1000*(s+1))
    .standard_normal((n_s, K), float32)``, rounded to BF16 for BF16 workloads.
  * GDN gate parameters: ``default_rng(seed + 7)``: A_log ~ U(-1, 1) then
    dt_bias ~ N(0, 0.5) (0.5 read as the standard deviation), one per head.
  * Delta-rule recurrence inputs drawn directly (the parity cases; the
    benchmark feeds the recurrence from the GDN projection itself):
    ``default_rng(seed)``: q, k [T, H_k*64] and v [T, H*128] N(0,1) (BF16
    workloads round them), beta [T, H] ~ U(0, 1), and the log decay
    g = -exp(mu_h + 0.5 z) with one level mu_h ~ U(ln 1e-3, ln 2) per head and
    z ~ N(0, 1) per token, so heads range from slow (alpha ~ 0.999) to fast
    (alpha ~ 0.1) forgetting.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest BF16 value (ties to even); returns float32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


@dataclasses.dataclass(frozen=True)
class Segment:
    name: str
    width: int
    epilogue: str  # "identity", "sigmoid", "gdn_decay", "swiglu_gate", "swiglu_up"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    segments: tuple
    seed: int
    dtype: str  # "f32" or "bf16": input dtype of X and W
    outlier_channels: Optional[tuple] = None  # fixed channel indices, else drawn
    n_outlier: int = 0
    outlier_scale: float = 1.0
    out_dtype: str = "bf16"
    heads: int = 0

    @property
    def N(self) -> int:
        return sum(s.width for s in self.segments)

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K


def _seg(name, width, epi="identity"):
    return Segment(name, width, epi)


# Tiny NVFP4 W4A4 linear: X[64,512], W[256,512] in FP32, channels 7 and 300 x50.
TINY = Workload("tiny_64x256x512", 64, 512, (_seg("w", 256),), seed=0, dtype="f32",
                outlier_channels=(7, 300), outlier_scale=50.0, out_dtype="f32")
# Prefill o_proj-shaped dense projection: X[4096,5120], W[5120,5120], 16 channels x100.
OPROJ = Workload("oproj_prefill_4096x5120x5120", 4096, 5120, (_seg("o_proj", 5120),), seed=1,
                 dtype="bf16", n_outlier=16, outlier_scale=100.0)
# Prefill fused MLP gate+up: X[8192,5120], W_gate/W_up [17408,5120], 0.5% channels x50.
MLP = Workload("mlp_gate_up_8192x34816x5120", 8192, 5120,
               (_seg("gate", 17408, "swiglu_gate"), _seg("up", 17408, "swiglu_up")), seed=2,
               dtype="bf16", n_outlier=26, outlier_scale=50.0)
# Fused GDN input projection: X[32768,5120], segments q,k,v,z,b,a; 0.5% channels x100.
GDN = Workload("gdn_in_proj_32768x12352x5120", 32768, 5120,
               (_seg("q", 2048), _seg("k", 2048), _seg("v", 4096), _seg("z", 4096),
                _seg("b", 32, "sigmoid"), _seg("a", 32, "gdn_decay")), seed=3,
               dtype="bf16", n_outlier=26, outlier_scale=100.0, heads=32)


def decode_workload(M: int) -> Workload:
    """Decode-shaped down_proj: X[M,17408] N(0,1) (no outliers), W[5120,17408]."""
    return Workload(f"decode_down_proj_M{M}_5120x17408", M, 17408, (_seg("down_proj", 5120),),
                    seed=4, dtype="bf16")


DECODE = tuple(decode_workload(m) for m in (1, 8, 64))
# Standalone quantizer workload: X[32768,17408] BF16 N(0,1), seed 4.
QUANT_SHAPE = (32768, 17408)
QUANT_SEED = 4

ALL = {w.name: w for w in (TINY, OPROJ, MLP, GDN) + DECODE}


def make_x(w: Workload, rows: Optional[int] = None) -> np.ndarray:
    """Activations X[M, K] as float32 (BF16-representable for BF16 workloads).

    ``rows`` replaces M (a smaller seeded case of the same recipe)."""
    M = w.M if rows is None else rows
    rng = np.random.default_rng(w.seed)
    if w.outlier_channels is not None:
        ch = np.array(w.outlier_channels, dtype=np.int64)
    elif w.n_outlier > 0:
        ch = rng.choice(w.K, size=w.n_outlier, replace=False)
    else:
        ch = np.zeros(0, dtype=np.int64)
    x = rng.standard_normal((M, w.K), dtype=np.float32)
    if ch.size:
        x[:, ch] *= np.float32(w.outlier_scale)
    if w.dtype == "bf16":
        x = round_to_bf16(x)
    return x


def make_w_segment(w: Workload, s: int) -> np.ndarray:
    """Weight segment s as float32 [width_s, K]."""
    seg = w.segments[s]
    rng = np.random.default_rng(w.seed + 1000 * (s + 1))
    ws = np.float32(0.02) * rng.standard_normal((seg.width, w.K), dtype=np.float32)
    if w.dtype == "bf16":
        ws = round_to_bf16(ws)
    return ws


def make_w_segments(w: Workload) -> list:
    return [make_w_segment(w, s) for s in range(len(w.segments))]


def make_gate_params(w: Workload):
    """(A_log, dt_bias) float32 [heads] for the GDN decay gate."""
    rng = np.random.default_rng(w.seed + 7)
    a_log = rng.uniform(-1.0, 1.0, size=w.heads).astype(np.float32)
    dt_bias = (0.5 * rng.standard_normal(w.heads)).astype(np.float32)
    return a_log, dt_bias


def make_quant_input(rows: Optional[int] = None, cols: Optional[int] = None, seed: int = QUANT_SEED):
    """The standalone quantizer tensor: BF16 N(0,1) of shape QUANT_SHAPE (or a smaller one)."""
    M = QUANT_SHAPE[0] if rows is None else rows
    K = QUANT_SHAPE[1] if cols is None else cols
    rng = np.random.default_rng(seed)
    return round_to_bf16(rng.standard_normal((M, K), dtype=np.float32))


def sample_rows(M: int, n: int, seed: int = 12345) -> np.ndarray:
    """Sorted distinct row indices, always including 0 and M-1."""
    if n >= M:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    inner = rng.choice(np.arange(1, M - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, M - 1], inner])).astype(np.int64)


GDN_HEADS, GDN_DK, GDN_DV = 32, 64, 128  # the projection's q/k (2048 = 32 x 64) and v (4096 = 32 x 128)


def make_recurrence_inputs(T: int, H: int, H_k: int, seed: int, dtype: str = "bf16", slow: bool = False):
    """(q, k, v, beta, g) float32 arrays for the delta-rule recurrence.  With
    slow, every head decays slowly (mu_h ~ U(ln 1e-4, ln 1e-2))."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H_k * GDN_DK), dtype=np.float32)
    k = rng.standard_normal((T, H_k * GDN_DK), dtype=np.float32)
    v = rng.standard_normal((T, H * GDN_DV), dtype=np.float32)
    beta = rng.uniform(0.0, 1.0, size=(T, H)).astype(np.float32)
    lo, hi = (np.log(1e-4), np.log(1e-2)) if slow else (np.log(1e-3), np.log(2.0))
    mu = rng.uniform(lo, hi, size=H)
    g = (-np.exp(mu[None, :] + 0.5 * rng.standard_normal((T, H)))).astype(np.float32)
    if dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
    return q, k, v, beta, g
