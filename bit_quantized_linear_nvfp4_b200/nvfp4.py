"""ctypes binding of libnvfp4 (include/nvfp4.h).

Argument marshalling only: tensors are allocated with PyTorch (device memory
and streams are PyTorch's), every step of the computation runs in the CUDA
library.  There is no fallback: if the library cannot be loaded, or a call
returns a non-zero status, an exception is raised.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

DTYPE_BF16 = 0
DTYPE_F32 = 1
MAX_SEGMENTS = 8

EPI_IDENTITY_BF16 = 0
EPI_IDENTITY_F32 = 1
EPI_SIGMOID_F32 = 2
EPI_GDN_DECAY_F32 = 3
EPI_SWIGLU_GATE = 4
EPI_SWIGLU_UP = 5

EPILOGUES = {
    "identity": EPI_IDENTITY_BF16,
    "identity_bf16": EPI_IDENTITY_BF16,
    "identity_f32": EPI_IDENTITY_F32,
    "sigmoid": EPI_SIGMOID_F32,
    "gdn_decay": EPI_GDN_DECAY_F32,
    "swiglu_gate": EPI_SWIGLU_GATE,
    "swiglu_up": EPI_SWIGLU_UP,
}

# Names the header declares; tests check the shared library exports each one.
EXPORTED = (
    "nvfp4_status_string", "nvfp4_last_cuda_error", "nvfp4_sf_bytes",
    "nvfp4_quantize_workspace_bytes", "nvfp4_quantize", "nvfp4_quantize_segments",
    "nvfp4_gemm_workspace_bytes", "nvfp4_gemm", "nvfp4_fused_proj", "nvfp4_check",
    "nvfp4_quantize_noalloc", "nvfp4_linear", "nvfp4_requantize_segments",
    "nvfp4_kv_fp8_quantize", "nvfp4_kv_fp8_dequantize", "nvfp4_activation_stats",
    "nvfp4_activation_summary",
    "nvfp4_gdn_workspace_bytes", "nvfp4_gdn_recurrence", "nvfp4_selftest_bounded_wait",
)


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib().nvfp4_status_string(status).decode()
        if status == 4:
            msg += f" (cudaError {_lib().nvfp4_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [status {status}]")
        self.status = status


class _Operand(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sf", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("K", ctypes.c_int64)]


class _Segment(ctypes.Structure):
    _fields_ = [("n_begin", ctypes.c_int64), ("n_end", ctypes.c_int64),
                ("epilogue", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("out", ctypes.c_void_p), ("ld_out", ctypes.c_int64),
                ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libnvfp4.so is not built ({LIB_PATH}); run bit_quantized_linear_nvfp4_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        c = ctypes
        lib.nvfp4_status_string.restype = c.c_char_p
        lib.nvfp4_status_string.argtypes = [c.c_int]
        lib.nvfp4_last_cuda_error.restype = c.c_int
        lib.nvfp4_sf_bytes.restype = c.c_size_t
        lib.nvfp4_sf_bytes.argtypes = [c.c_int64, c.c_int64]
        lib.nvfp4_quantize_workspace_bytes.restype = c.c_size_t
        lib.nvfp4_quantize_workspace_bytes.argtypes = [c.c_int]
        lib.nvfp4_quantize.restype = c.c_int
        lib.nvfp4_quantize.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64,
                                       c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                       c.c_void_p, c.c_size_t, c.c_void_p]
        lib.nvfp4_quantize_segments.restype = c.c_int
        lib.nvfp4_quantize_segments.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64,
                                                c.POINTER(c.c_int64), c.c_int, c.c_void_p, c.c_void_p,
                                                c.c_void_p, c.c_void_p, c.c_void_p, c.c_size_t,
                                                c.c_void_p]
        lib.nvfp4_gemm_workspace_bytes.restype = c.c_size_t
        lib.nvfp4_gemm_workspace_bytes.argtypes = [c.c_int64, c.c_int64, c.c_int64]
        lib.nvfp4_gemm.restype = c.c_int
        lib.nvfp4_gemm.argtypes = [c.POINTER(_Operand), c.c_void_p, c.POINTER(_Operand), c.c_void_p,
                                   c.c_void_p, c.c_int, c.c_int64, c.c_void_p, c.c_size_t, c.c_void_p]
        lib.nvfp4_fused_proj.restype = c.c_int
        lib.nvfp4_fused_proj.argtypes = [c.POINTER(_Operand), c.c_void_p, c.POINTER(_Operand),
                                         c.c_void_p, c.POINTER(_Segment), c.c_int, c.c_void_p,
                                         c.c_size_t, c.c_void_p]
        lib.nvfp4_quantize_noalloc.restype = c.c_int
        lib.nvfp4_quantize_noalloc.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64,
                                               c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p]
        lib.nvfp4_linear.restype = c.c_int
        lib.nvfp4_linear.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_void_p,
                                     c.c_void_p, c.c_void_p, c.c_void_p, c.POINTER(_Operand), c.c_void_p,
                                     c.POINTER(_Segment), c.c_int, c.c_void_p, c.c_size_t, c.c_void_p]
        lib.nvfp4_requantize_segments.restype = c.c_int
        lib.nvfp4_requantize_segments.argtypes = [c.POINTER(_Operand), c.c_void_p, c.c_int, c.c_void_p, c.c_void_p,
                                                  c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p]
        lib.nvfp4_kv_fp8_quantize.restype = c.c_int
        lib.nvfp4_kv_fp8_quantize.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_void_p,
                                              c.c_void_p, c.c_int64, c.c_void_p]
        lib.nvfp4_kv_fp8_dequantize.restype = c.c_int
        lib.nvfp4_kv_fp8_dequantize.argtypes = [c.c_void_p, c.c_int64, c.c_int64, c.c_int64, c.c_void_p,
                                                c.c_void_p, c.c_int, c.c_int64, c.c_void_p]
        lib.nvfp4_activation_stats.restype = c.c_int
        lib.nvfp4_activation_stats.argtypes = [c.c_void_p, c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_void_p,
                                               c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                               c.c_void_p]
        lib.nvfp4_activation_summary.restype = c.c_int
        lib.nvfp4_activation_summary.argtypes = [c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64, c.c_void_p,
                                                 c.c_int64, c.c_void_p, c.c_void_p]
        lib.nvfp4_gdn_workspace_bytes.restype = c.c_size_t
        lib.nvfp4_gdn_workspace_bytes.argtypes = [c.c_int64, c.c_int64]
        lib.nvfp4_gdn_recurrence.restype = c.c_int
        lib.nvfp4_gdn_recurrence.argtypes = [c.c_void_p, c.c_void_p, c.c_void_p, c.c_int, c.c_int64, c.c_int64,
                                             c.c_int64, c.c_int64, c.c_int64, c.c_int64, c.c_int64, c.c_int64,
                                             c.c_void_p, c.c_int64, c.c_void_p, c.c_int64, c.c_float,
                                             c.c_void_p, c.c_void_p, c.c_void_p, c.c_int, c.c_int64,
                                             c.c_void_p, c.c_size_t, c.c_void_p]
        lib.nvfp4_selftest_bounded_wait.restype = c.c_int
        lib.nvfp4_selftest_bounded_wait.argtypes = [c.c_uint64, c.c_void_p]
        lib.nvfp4_check.restype = c.c_int
        lib.nvfp4_check.argtypes = [c.c_void_p]
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes library (raises ImportError if it is not built)."""
    return _lib()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _call(name: str, *args):
    st = getattr(_lib(), name)(*args)
    if st != 0:
        raise Nvfp4Error(st, name)


def nvfp4_sf_bytes(rows: int, K: int) -> int:
    return int(_lib().nvfp4_sf_bytes(rows, K))


def nvfp4_quantize_workspace_bytes(nseg: int = 1) -> int:
    return int(_lib().nvfp4_quantize_workspace_bytes(nseg))


def nvfp4_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib().nvfp4_gemm_workspace_bytes(M, N, K))


@dataclasses.dataclass
class Operand:
    """A quantised operand: packed E2M1 codes [rows, K/2] and E4M3 scales in the
    tcgen05 block-scale layout, both CUDA uint8 tensors."""
    codes: torch.Tensor
    sf: torch.Tensor
    rows: int
    K: int

    def _c(self) -> _Operand:
        return _Operand(self.codes.data_ptr(), self.sf.data_ptr(), self.rows, self.K)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"quantiser input must be bfloat16 or float32, not {t.dtype}")


def _check_2d(x: torch.Tensor):
    if not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("expected a CUDA 2-D tensor with unit column stride")


def nvfp4_quantize(x: torch.Tensor, g_in: Optional[torch.Tensor] = None, *, codes=None, sf=None,
                   g_out=None, workspace=None, stream=None):
    """Quantise activations x[M, K] (BF16/F32) -> (Operand, g_out[1])."""
    _check_2d(x)
    M, K = x.shape
    dev = x.device
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    sf = torch.empty(nvfp4_sf_bytes(max(M, 1), K), dtype=torch.uint8, device=dev) if sf is None else sf
    g_out = torch.empty(1, dtype=torch.float32, device=dev) if g_out is None else g_out
    if g_in is None and workspace is None:
        workspace = torch.empty(nvfp4_quantize_workspace_bytes(1), dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _call("nvfp4_quantize", _ptr(x), _dtype_code(x), M, K, x.stride(0), _ptr(g_in), _ptr(g_out),
          _ptr(codes), _ptr(sf), _ptr(workspace), ws_bytes, _stream(stream))
    return Operand(codes, sf, M, K), g_out


def nvfp4_quantize_segments(w: torch.Tensor, row_bounds: Sequence[int], g_in=None, *, codes=None,
                            sf=None, g_out=None, workspace=None, stream=None):
    """Quantise stacked modules w[N, K], one global scale per row range -> (Operand, g_out[nseg])."""
    _check_2d(w)
    N, K = w.shape
    nseg = len(row_bounds) - 1
    dev = w.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    sf = torch.empty(nvfp4_sf_bytes(N, K), dtype=torch.uint8, device=dev) if sf is None else sf
    g_out = torch.empty(nseg, dtype=torch.float32, device=dev) if g_out is None else g_out
    if g_in is None and workspace is None:
        workspace = torch.empty(nvfp4_quantize_workspace_bytes(nseg), dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    bounds = (ctypes.c_int64 * (nseg + 1))(*[int(b) for b in row_bounds])
    _call("nvfp4_quantize_segments", _ptr(w), _dtype_code(w), N, K, w.stride(0), bounds, nseg,
          _ptr(g_in), _ptr(g_out), _ptr(codes), _ptr(sf), _ptr(workspace), ws_bytes, _stream(stream))
    return Operand(codes, sf, N, K), g_out


def nvfp4_gemm(A: Operand, g_a: torch.Tensor, W: Operand, g_w: torch.Tensor, out=None,
               out_dtype=torch.bfloat16, workspace=None, stream=None):
    """out[M, N] = (A . W^T) * g_a * g_w, BF16 or F32."""
    if out is None:
        out = torch.empty((A.rows, W.rows), dtype=out_dtype, device=A.codes.device)
    code = DTYPE_BF16 if out.dtype == torch.bfloat16 else DTYPE_F32
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if workspace is None and nvfp4_gemm_workspace_bytes(A.rows, W.rows, A.K) > 0:
        workspace = torch.empty(nvfp4_gemm_workspace_bytes(A.rows, W.rows, A.K), dtype=torch.uint8,
                                device=A.codes.device)
        ws_bytes = workspace.numel()
    a, w = A._c(), W._c()
    _call("nvfp4_gemm", ctypes.byref(a), _ptr(g_a), ctypes.byref(w), _ptr(g_w), _ptr(out), code,
          out.stride(0), _ptr(workspace), ws_bytes, _stream(stream))
    return out


@dataclasses.dataclass
class Segment:
    """One module of a fused projection: W rows [n_begin, n_end)."""
    n_begin: int
    n_end: int
    epilogue: str
    out: Optional[torch.Tensor] = None
    A_log: Optional[torch.Tensor] = None
    dt_bias: Optional[torch.Tensor] = None


def _segment_array(segments: Sequence[Segment]):
    n = len(segments)
    arr = (_Segment * n)()
    for i, s in enumerate(segments):
        arr[i].n_begin = s.n_begin
        arr[i].n_end = s.n_end
        arr[i].epilogue = EPILOGUES[s.epilogue] if isinstance(s.epilogue, str) else int(s.epilogue)
        arr[i].reserved = 0
        arr[i].out = None if s.out is None else s.out.data_ptr()
        arr[i].ld_out = 0 if s.out is None else s.out.stride(0)
        arr[i].A_log = None if s.A_log is None else s.A_log.data_ptr()
        arr[i].dt_bias = None if s.dt_bias is None else s.dt_bias.data_ptr()
    return arr, n


def nvfp4_fused_proj(A: Operand, g_a: torch.Tensor, W: Operand, seg_global_scale: torch.Tensor,
                     segments: Sequence[Segment], workspace=None, stream=None):
    """One GEMM over the segments, each with its own global scale and epilogue;
    results go to each segment's `out` tensor."""
    arr, n = _segment_array(segments)
    need = nvfp4_gemm_workspace_bytes(A.rows, W.rows, A.K)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=A.codes.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a, w = A._c(), W._c()
    _call("nvfp4_fused_proj", ctypes.byref(a), _ptr(g_a), ctypes.byref(w), _ptr(seg_global_scale),
          arr, n, _ptr(workspace), ws_bytes, _stream(stream))


def nvfp4_linear(x: torch.Tensor, W: Operand, seg_global_scale: torch.Tensor, segments: Sequence[Segment],
                 g_in: Optional[torch.Tensor] = None, *, a_codes=None, a_sf=None, g_a=None, workspace=None,
                 stream=None):
    """Quantise x[M, K] and run the fused projection on it in one call (the GEMM
    may start streaming W while the quantiser runs).  Returns (A, g_a): the
    quantised activation left in a_codes / a_sf / g_a."""
    _check_2d(x)
    M, K = x.shape
    dev = x.device
    a_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if a_codes is None else a_codes
    a_sf = torch.empty(nvfp4_sf_bytes(max(M, 1), K), dtype=torch.uint8, device=dev) if a_sf is None else a_sf
    g_a = torch.empty(1, dtype=torch.float32, device=dev) if g_a is None else g_a
    if g_in is None and workspace is None:
        workspace = torch.empty(nvfp4_quantize_workspace_bytes(1), dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    arr, n = _segment_array(segments)
    w = W._c()
    _call("nvfp4_linear", _ptr(x), _dtype_code(x), M, K, x.stride(0), _ptr(g_in), _ptr(a_codes), _ptr(a_sf),
          _ptr(g_a), ctypes.byref(w), _ptr(seg_global_scale), arr, n, _ptr(workspace), ws_bytes,
          _stream(stream))
    return Operand(a_codes, a_sf, M, K), g_a


def nvfp4_requantize_segments(W: Operand, row_bounds: Sequence[int], g_old: torch.Tensor,
                              g_new: Optional[torch.Tensor] = None, *, codes=None, sf=None, g_out=None,
                              in_place: bool = False, stream=None):
    """Re-encode W (modules = row ranges with scales g_old) under one common
    global scale (g_new, or the largest of g_old) -> (Operand, g_out[nseg])."""
    nseg = len(row_bounds) - 1
    dev = W.codes.device
    if in_place:
        codes, sf = W.codes, W.sf
    codes = torch.empty_like(W.codes) if codes is None else codes
    sf = torch.empty_like(W.sf) if sf is None else sf
    g_out = torch.empty(nseg, dtype=torch.float32, device=dev) if g_out is None else g_out
    bounds = (ctypes.c_int64 * (nseg + 1))(*[int(b) for b in row_bounds])
    w = W._c()
    _call("nvfp4_requantize_segments", ctypes.byref(w), bounds, nseg, _ptr(g_old), _ptr(g_new), _ptr(codes),
          _ptr(sf), _ptr(g_out), _stream(stream))
    return Operand(codes, sf, W.rows, W.K), g_out


def nvfp4_gdn_workspace_bytes(T: int, H: int) -> int:
    return int(_lib().nvfp4_gdn_workspace_bytes(T, H))


GDN_DK, GDN_DV = 64, 128


def nvfp4_gdn_recurrence(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, beta: torch.Tensor, g: torch.Tensor,
                         h0: Optional[torch.Tensor] = None, scale: float = 0.0, *, d_k: int = GDN_DK,
                         d_v: int = GDN_DV, out=None, out_dtype=None, h_out=None, workspace=None, stream=None):
    """Gated delta rule over one sequence: q, k [T, H_k*64], v [T, H*128]
    (BF16/F32, same dtype), beta, g [T, H] FP32 -> o [T, H*128] (v's dtype
    unless out/out_dtype says otherwise).  h0 / h_out: FP32 [H, 128, 64]
    entering / final state (h_out may be h0).  scale 0 selects 64^-1/2."""
    for t in (q, k, v, beta, g):
        _check_2d(t)
    if q.dtype != v.dtype or k.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    if beta.dtype != torch.float32 or g.dtype != torch.float32:
        raise TypeError("beta and g must be float32")
    T = v.shape[0]
    H = v.shape[1] // d_v
    H_k = q.shape[1] // d_k
    dev = v.device
    if out is None:
        out = torch.empty((T, H * GDN_DV), dtype=out_dtype or v.dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(max(1, nvfp4_gdn_workspace_bytes(T, H)), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    in_code = _dtype_code(v)
    out_code = DTYPE_BF16 if out.dtype == torch.bfloat16 else DTYPE_F32
    _call("nvfp4_gdn_recurrence", _ptr(q), _ptr(k), _ptr(v), in_code, T, H, H_k, d_k, d_v, q.stride(0),
          k.stride(0), v.stride(0), _ptr(beta), beta.stride(0), _ptr(g), g.stride(0), float(scale), _ptr(h0),
          _ptr(h_out), _ptr(out), out_code, out.stride(0), _ptr(workspace), ws_bytes, _stream(stream))
    return out


def nvfp4_kv_fp8_quantize(x: torch.Tensor, scale: torch.Tensor, *, out=None, stream=None) -> torch.Tensor:
    """FP8 (E4M3) codes of x[rows, cols] (BF16/F32) under the static scale (a
    device float tensor); returns uint8 codes [rows, cols]."""
    _check_2d(x)
    rows, cols = x.shape
    out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if out is None else out
    _call("nvfp4_kv_fp8_quantize", _ptr(x), _dtype_code(x), rows, cols, x.stride(0), _ptr(scale), _ptr(out),
          out.stride(0), _stream(stream))
    return out


def nvfp4_kv_fp8_dequantize(codes: torch.Tensor, scale: torch.Tensor, out_dtype=torch.bfloat16, *, out=None,
                            stream=None) -> torch.Tensor:
    """Decode FP8 (E4M3) codes [rows, cols] with the static scale."""
    _check_2d(codes)
    rows, cols = codes.shape
    out = torch.empty((rows, cols), dtype=out_dtype, device=codes.device) if out is None else out
    code = DTYPE_BF16 if out.dtype == torch.bfloat16 else DTYPE_F32
    _call("nvfp4_kv_fp8_dequantize", _ptr(codes), rows, cols, codes.stride(0), _ptr(scale), _ptr(out), code,
          out.stride(0), _stream(stream))
    return out


def nvfp4_activation_stats(x: torch.Tensor, g: Optional[torch.Tensor] = None, *, into: Optional[dict] = None,
                           stream=None) -> dict:
    """Accumulate NVFP4-granularity statistics of x[M, K] into `into` (a dict of
    device tensors from a previous call, or fresh zeros): moments (float64[8]),
    row_err2 / row_norm2 (float32[M], A4 error needs g), col_sq / col_max
    (float32[K])."""
    _check_2d(x)
    M, K = x.shape
    dev = x.device
    if into is None:
        into = {"moments": torch.zeros(8, dtype=torch.float64, device=dev),
                "row_err2": torch.zeros(M, dtype=torch.float32, device=dev) if g is not None else None,
                "row_norm2": torch.zeros(M, dtype=torch.float32, device=dev),
                "col_sq": torch.zeros(K, dtype=torch.float32, device=dev),
                "col_max": torch.zeros(K, dtype=torch.float32, device=dev)}
    _call("nvfp4_activation_stats", _ptr(x), _dtype_code(x), M, K, x.stride(0), _ptr(g), _ptr(into["moments"]),
          _ptr(into["row_err2"]), _ptr(into["row_norm2"]), _ptr(into["col_sq"]), _ptr(into["col_max"]),
          _stream(stream))
    return into


SUMMARY_FIELDS = ("max_over_rms", "kurtosis", "dominated_share", "a4_err_mean", "a4_err_min", "a4_err_max",
                  "hot_channel_ratio", "channel_rms_median")


def nvfp4_activation_summary(stats: dict, *, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Device float64[8] of derived figures from nvfp4_activation_stats'
    accumulators (nvfp4_activation_summary; the order is SUMMARY_FIELDS)."""
    dev = stats["moments"].device
    out = torch.empty(8, dtype=torch.float64, device=dev) if out is None else out
    M = stats["row_norm2"].numel()
    K = stats["col_sq"].numel()
    _call("nvfp4_activation_summary", _ptr(stats["moments"]), _ptr(stats.get("row_err2")), _ptr(stats["row_norm2"]),
          M, _ptr(stats["col_sq"]), K, _ptr(out), _stream(stream))
    return out


def activation_summary(stats: dict, stream=None) -> dict:
    """The derived figures as a dict (computed by the library on the device;
    the A4 error fields are absent when the statistics had no global scale)."""
    vals = nvfp4_activation_summary(stats, stream=stream).cpu().tolist()
    out = dict(zip(SUMMARY_FIELDS, vals))
    if stats.get("row_err2") is None:
        for k in ("a4_err_mean", "a4_err_min", "a4_err_max"):
            del out[k]
    return out


def nvfp4_check(stream=None):
    """Synchronise the stream and raise if a device-side wait timed out."""
    _call("nvfp4_check", _stream(stream))
