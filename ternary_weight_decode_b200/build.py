"""Builds the CUDA libraries in-tree for B200 (sm_100a) with nvcc.

libtern.so        -- the C-ABI library (include/tern.h): kernels + boundary.
libtern_synth.so  -- the device side of the seeded input generator.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-rdc=true",
                "-I" + os.path.join(ROOT, "include")]

LIBS = {
    "libtern.so": ["csrc/tern_api.cu", "csrc/tern_format.cu", "csrc/tern_quant.cu",
                   "csrc/tern_gemv.cu", "csrc/tern_gemv_tc.cu", "csrc/tern_gemv_stream.cu",
                   "csrc/tern_noalloc.cu", "csrc/tern_gemm.cu", "csrc/tern_tcdebug.cu",
                   "csrc/tern_debug.cu", "csrc/tern_ternarize.cu", "csrc/tern_attention.cu"],
    "libtern_synth.so": ["synth_csrc/tern_synth.cu"],
}
HEADERS = ["csrc/tern_common.cuh", "csrc/tern_internal.h", "csrc/tern_tc.cuh",
           "csrc/tern_gemv_common.cuh", "csrc/tern_gemv_stream.cuh"]


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose_ptxas: bool) -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    deps = [src] + [os.path.join(PKG, h) for h in HEADERS] + [os.path.join(ROOT, "include", "tern.h")]
    if os.path.exists(obj) and os.path.getmtime(obj) >= _newest(deps):
        return obj
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose_ptxas else []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose_ptxas: bool = False) -> list[str]:
    os.makedirs(BUILD, exist_ok=True)
    out = []
    for lib, srcs in LIBS.items():
        srcs = [os.path.join(PKG, s) for s in srcs]
        with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
            objs = list(ex.map(lambda s: _compile(s, verbose_ptxas), srcs))
        target = os.path.join(PKG, lib)
        if not os.path.exists(target) or os.path.getmtime(target) < _newest(objs):
            tmp = target + f".tmp{os.getpid()}"
            cmd = [NVCC] + ARCH + ["-shared", "-rdc=true", "-Xcompiler", "-fPIC", "-o", tmp] + objs
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc link failed for {lib}:\n{r.stdout}\n{r.stderr}")
            os.replace(tmp, target)
        out.append(target)
    return out


if __name__ == "__main__":
    for p in build(verbose_ptxas="-v" in sys.argv):
        print(p)
