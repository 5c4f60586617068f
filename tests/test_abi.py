"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/nvfp4.h declares, and rejects bad arguments on the host before
any CUDA call (CPU only: pointers below are never dereferenced)."""
import ctypes
import os
import re

import pytest

from bit_quantized_linear_nvfp4_b200 import build as nvbuild
from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    nvbuild.build(verbose=False)
    return nv.library()


def _declared():
    text = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(nv.EXPORTED)


def test_status_strings(lib):
    for s in range(8):
        assert nv.library().nvfp4_status_string(s)
    assert b"unknown" in nv.library().nvfp4_status_string(99)


def test_sf_bytes_padding(lib):
    assert nv.nvfp4_sf_bytes(1, 16) == 128 * 4
    assert nv.nvfp4_sf_bytes(128, 64) == 512
    assert nv.nvfp4_sf_bytes(129, 64) == 1024
    assert nv.nvfp4_sf_bytes(4096, 5120) == 4096 * 320
    assert nv.nvfp4_sf_bytes(12352, 5120) == 97 * 128 * 320
    assert nv.nvfp4_sf_bytes(0, 16) == 0
    assert nv.nvfp4_quantize_workspace_bytes(1) >= 4
    assert nv.nvfp4_quantize_workspace_bytes(8) >= 32


FAKE = 0x10000  # aligned, never dereferenced: validation fails first
STREAM = None


def _q(lib, x=FAKE, dtype=0, M=4, K=32, ld=32, g_in=FAKE, g_out=FAKE, codes=FAKE, sf=FAKE, ws=None, wsb=0):
    v = ctypes.c_void_p
    return lib.nvfp4_quantize(v(x) if x else None, dtype, M, K, ld, v(g_in) if g_in else None,
                              v(g_out) if g_out else None, v(codes) if codes else None,
                              v(sf) if sf else None, v(ws) if ws else None, wsb, None)


def test_quantize_rejects_bad_arguments(lib):
    assert _q(lib, K=24) == 2          # K % 16
    assert _q(lib, dtype=7) == 1       # dtype
    assert _q(lib, x=0) == 1           # null input
    assert _q(lib, g_out=0) == 1       # null g_out
    assert _q(lib, M=-1) == 1
    assert _q(lib, ld=16) == 1         # ld < K
    assert _q(lib, x=FAKE + 2) == 3    # misaligned input
    assert _q(lib, ld=36) == 3         # row stride not a multiple of 16 bytes
    assert _q(lib, codes=FAKE + 8) == 3
    assert _q(lib, g_in=0) == 6        # dynamic scale without workspace
    assert _q(lib, g_in=0, ws=FAKE, wsb=2) == 6


def _op(codes=FAKE, sf=FAKE, rows=128, K=256):
    return nv._Operand(codes, sf, rows, K)


def _fp(lib, A=None, W=None, segs=None, nseg=None, g_a=FAKE, sc=FAKE):
    A = A or _op()
    W = W or _op(rows=256)
    if segs is None:
        segs = [nv._Segment(0, 256, 0, 0, FAKE, 256, None, None)]
    arr = (nv._Segment * len(segs))(*segs)
    v = ctypes.c_void_p
    return lib.nvfp4_fused_proj(ctypes.byref(A), v(g_a) if g_a else None, ctypes.byref(W),
                                v(sc) if sc else None, arr, len(segs) if nseg is None else nseg,
                                None, 0, None)


def test_fused_proj_rejects_bad_arguments(lib):
    S = nv._Segment
    assert _fp(lib, A=_op(K=48)) == 2                         # K % 32
    assert _fp(lib, A=_op(K=512)) == 1                        # K mismatch
    assert _fp(lib, A=_op(codes=FAKE + 4)) == 3
    assert _fp(lib, g_a=0) == 1
    assert _fp(lib, nseg=0) == 1
    assert _fp(lib, nseg=9) == 1
    # segments must tile [0, N)
    assert _fp(lib, segs=[S(0, 100, 0, 0, FAKE, 256, None, None)]) == 1
    assert _fp(lib, segs=[S(0, 100, 0, 0, FAKE, 256, None, None), S(120, 256, 0, 0, FAKE, 256, None, None)]) == 1
    assert _fp(lib, segs=[S(0, 256, 9, 0, FAKE, 256, None, None)]) == 1     # epilogue kind
    assert _fp(lib, segs=[S(0, 256, 0, 0, None, 256, None, None)]) == 1     # null out
    assert _fp(lib, segs=[S(0, 256, 0, 0, FAKE + 2, 256, None, None)]) == 3  # misaligned out
    assert _fp(lib, segs=[S(0, 256, 0, 0, FAKE, 260, None, None)]) == 3     # ld not multiple of 8
    assert _fp(lib, segs=[S(0, 256, 3, 0, FAKE, 256, None, None)]) == 1     # decay without params
    # SwiGLU needs gate then up of equal width, 128-row aligned
    assert _fp(lib, segs=[S(0, 128, 4, 0, FAKE, 128, None, None), S(128, 256, 0, 0, FAKE, 128, None, None)]) == 1
    assert _fp(lib, W=_op(rows=200), segs=[S(0, 100, 4, 0, FAKE, 104, None, None), S(100, 200, 5, 0, None, 0, None, None)]) == 2


def test_segmented_quantize_rejects_bad_bounds(lib):
    v = ctypes.c_void_p
    def call(bounds, N=256):
        b = (ctypes.c_int64 * len(bounds))(*bounds)
        return lib.nvfp4_quantize_segments(v(FAKE), 0, N, 64, 64, b, len(bounds) - 1, v(FAKE), v(FAKE),
                                           v(FAKE), v(FAKE), None, 0, None)
    assert call([0, 100, 90, 256]) == 1
    assert call([1, 256]) == 1
    assert call([0, 200]) == 1
    assert call([0] + list(range(10, 256, 30)) + [256]) == 1   # more than 8 segments


def _lin(lib, x=FAKE, M=4, K=256, ld=256, g_in=FAKE, ac=FAKE, asf=FAKE, ga=FAKE, W=None, sc=FAKE,
         segs=None, ws=None, wsb=0):
    v = ctypes.c_void_p
    W = W or _op(codes=0x400000, sf=0x800000, rows=256)
    if segs is None:
        segs = [nv._Segment(0, 256, 0, 0, 0x900000, 256, None, None)]
    arr = (nv._Segment * len(segs))(*segs)
    return lib.nvfp4_linear(v(x) if x else None, 0, M, K, ld, v(g_in) if g_in else None,
                            v(ac) if ac else None, v(asf) if asf else None, v(ga) if ga else None,
                            ctypes.byref(W), v(sc) if sc else None, arr, len(segs), v(ws) if ws else None,
                            wsb, None)


def test_linear_rejects_bad_arguments(lib):
    assert _lin(lib, K=24, ld=32) == 2                        # K % 16
    assert _lin(lib, x=0) == 1
    assert _lin(lib, ga=0) == 1                               # g_a receives the scale
    assert _lin(lib, W=_op(codes=0x400000, sf=0x800000, rows=256, K=512)) == 1   # K mismatch
    assert _lin(lib, g_in=0) == 6                             # dynamic scale without workspace
    # nothing the quantiser writes may overlap W (the GEMM streams W early)
    assert _lin(lib, ac=0x400000 + 64) == 1
    assert _lin(lib, asf=0x800000) == 1
    assert _lin(lib, ga=0x400010) == 1
    assert _lin(lib, g_in=0, ws=0x800000 + 1024, wsb=4096) == 1
    assert _lin(lib, segs=[nv._Segment(0, 100, 0, 0, 0x900000, 256, None, None)]) == 1   # segments
    assert _lin(lib, M=0) == 0                                # empty: nothing enqueued


def test_requantize_rejects_bad_arguments(lib):
    v = ctypes.c_void_p
    W = _op(codes=0x400000, sf=0x800000, rows=256, K=256)

    def call(bounds=(0, 100, 256), g_old=FAKE, codes=0x900000, sf=0xA00000, g_out=FAKE, W=W):
        b = (ctypes.c_int64 * len(bounds))(*bounds)
        return lib.nvfp4_requantize_segments(ctypes.byref(W), b, len(bounds) - 1, v(g_old) if g_old else None, None,
                                             v(codes) if codes else None, v(sf) if sf else None,
                                             v(g_out) if g_out else None, None)
    assert call(bounds=(0, 100, 200)) == 1            # bounds must end at W->rows
    assert call(bounds=(0, 120, 100, 256)) == 1       # increasing
    assert call(g_old=0) == 1
    assert call(codes=0) == 1
    assert call(g_out=FAKE + 2) == 3
    assert call(codes=0x900000 + 8) == 3
    assert call(codes=0x400000 + 64) == 1             # partial overlap with W's codes
    assert call(sf=0x800000 + 16) == 1                # partial overlap with W's scales
    assert call(W=_op(codes=0x400000, sf=0x800000, rows=256, K=48)) == 2


def test_kv_fp8_rejects_bad_arguments(lib):
    v = ctypes.c_void_p

    def enc(x=FAKE, dtype=0, rows=4, cols=64, ld_x=64, scale=FAKE, out=FAKE, ld_out=64):
        return lib.nvfp4_kv_fp8_quantize(v(x) if x else None, dtype, rows, cols, ld_x, v(scale) if scale else None,
                                         v(out) if out else None, ld_out, None)

    def dec(c=FAKE, rows=4, cols=64, ld_c=64, scale=FAKE, out=FAKE, dtype=0, ld_out=64):
        return lib.nvfp4_kv_fp8_dequantize(v(c) if c else None, rows, cols, ld_c, v(scale) if scale else None,
                                           v(out) if out else None, dtype, ld_out, None)
    assert enc(cols=60, ld_x=64, ld_out=64) == 2      # cols % 8
    assert enc(dtype=3) == 1
    assert enc(scale=0) == 1
    assert enc(x=FAKE + 8) == 3                        # rows 16-byte aligned
    assert enc(ld_x=68) == 3                           # BF16 row stride not a multiple of 16 bytes
    assert enc(out=FAKE + 4) == 3
    assert enc(ld_out=60) == 1                         # ld_out < cols
    assert enc(rows=0) == 0 and enc(cols=0, ld_x=0, ld_out=0) == 0
    assert dec(c=FAKE + 4) == 3
    assert dec(out=FAKE + 8) == 3
    assert dec(dtype=1, ld_out=66) == 3
    assert dec(ld_c=32) == 1


def test_activation_stats_rejects_bad_arguments(lib):
    v = ctypes.c_void_p

    def call(x=FAKE, dtype=0, M=4, K=64, ld=64, g=FAKE, mom=FAKE, re=FAKE, rn=FAKE, cs=FAKE, cm=FAKE):
        p = lambda a: v(a) if a else None
        return lib.nvfp4_activation_stats(p(x), dtype, M, K, ld, p(g), p(mom), p(re), p(rn), p(cs), p(cm), None)
    assert call(K=40) == 2
    assert call(dtype=5) == 1
    assert call(mom=0) == 1
    assert call(g=0) == 1                   # A4 error requested without a global scale
    assert call(x=FAKE + 8) == 3
    assert call(mom=FAKE + 4) == 3
    assert call(cs=FAKE + 2) == 3
    assert call(ld=32) == 1
    assert call(M=0) == 0


def test_activation_summary_rejects_bad_arguments(lib):
    v = ctypes.c_void_p

    def call(mom=FAKE, re=FAKE, rn=FAKE, M=4, cs=FAKE, K=64, out=FAKE):
        p = lambda a: v(a) if a else None
        return lib.nvfp4_activation_summary(p(mom), p(re), p(rn), M, p(cs), K, p(out), None)
    assert call(mom=0) == 1 and call(rn=0) == 1 and call(cs=0) == 1 and call(out=0) == 1
    assert call(M=0) == 1 and call(K=0) == 1 and call(M=-3) == 1
    assert call(M=1 << 31) == 2 and call(K=(1 << 30) + 1) == 2
    assert call(mom=FAKE + 4) == 3 and call(out=FAKE + 4) == 3
    assert call(re=FAKE + 2) == 3 and call(rn=FAKE + 1) == 3 and call(cs=FAKE + 2) == 3


def test_gdn_recurrence_rejects_bad_arguments(lib):
    v = ctypes.c_void_p
    T, H, Hk = 100, 4, 2
    Q, K, V, B, G, O, WS = (FAKE + i * 0x1000000 for i in range(7))

    def call(q=Q, k=K, vv=V, dt=0, T=T, H=H, Hk=Hk, dk=64, dv=128, ldq=Hk * 64, ldk=Hk * 64, ldv=H * 128,
             beta=B, ldb=H, g=G, ldg=H, scale=0.0, h0=0, hout=0, o=O, odt=0, ldo=H * 128, ws=WS, wsb=1 << 40):
        p = lambda a: v(a) if a else None
        return lib.nvfp4_gdn_recurrence(p(q), p(k), p(vv), dt, T, H, Hk, dk, dv, ldq, ldk, ldv, p(beta), ldb, p(g),
                                        ldg, scale, p(h0), p(hout), p(o), odt, ldo, p(ws), wsb, None)
    assert lib.nvfp4_gdn_workspace_bytes(T, H) == 2 * H * 3 * 128 * 64 * 4  # two chunks of 64 tokens
    assert lib.nvfp4_gdn_workspace_bytes(0, H) == 0
    assert call(dt=2) == 1 and call(odt=7) == 1
    assert call(Hk=3) == 1                    # H_k must divide H
    assert call(dk=128) == 2 and call(dv=64) == 2
    assert call(scale=-1.0) == 1 and call(scale=float("nan")) == 1
    assert call(q=0) == 1 and call(beta=0) == 1 and call(o=0) == 1
    assert call(ldq=64) == 1 and call(ldv=500) == 1 and call(ldb=2) == 1
    assert call(q=Q + 8) == 3 and call(o=O + 4) == 3
    assert call(ldk=Hk * 64 + 4) == 3         # BF16 row of k not a multiple of 16 bytes
    assert call(beta=B + 2) == 3
    assert call(ws=0) == 6 and call(wsb=1000) == 6 and call(ws=WS + 8) == 6
    assert call(o=V + 256) == 1               # output overlapping v
    assert call(ws=O) == 1                    # workspace overlapping the output
    assert call(h0=FAKE + 0x9000000, hout=FAKE + 0x9000000 + 64) == 1  # partial state overlap
    assert call(T=0) == 0                     # nothing to do without h_out


def test_bounded_wait_selftest_rejects_bad_limits(lib):
    assert lib.nvfp4_selftest_bounded_wait(0, None) == 1
    assert lib.nvfp4_selftest_bounded_wait(999_999, None) == 1          # below 1 ms
    assert lib.nvfp4_selftest_bounded_wait(2_000_000_001, None) == 1    # above 2 s
