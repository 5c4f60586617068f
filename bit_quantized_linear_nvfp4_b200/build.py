"""Build libnvfp4.so in-tree for sm_100a with nvcc (no JIT cache, no torch build)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4.so")
SOURCES = ["libnvfp4.cu", "quantize.cu", "gemm.cu", "gemm_decode.cu", "api.cu", "noalloc.cu", "kv_fp8.cu", "act_stats.cu", "gdn.cu", "selftest.cu", "ptx.cuh",
           "internal.h"]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES]
    deps.append(os.path.join(HERE, "..", "include", "nvfp4.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = True, extra=()) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
        "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v",
        "-I", os.path.join(HERE, "..", "include"),
        os.path.join(CSRC, "libnvfp4.cu"), "-o", LIB + ".tmp",
    ] + list(extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libnvfp4.so")
    if verbose:
        for line in (r.stdout + r.stderr).splitlines():
            if "registers" in line or "spill" in line or "error" in line.lower():
                print(line)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv)
