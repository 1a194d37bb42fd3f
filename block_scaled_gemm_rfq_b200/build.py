"""Build the sm_100a CUDA library ``librfq.so`` in-tree with nvcc.

    python -m block_scaled_gemm_rfq_b200.build          # or __graft_entry__.build()

The library is the C ABI of include/rfq.h.  Sources: csrc/*.cu.  Flags: sm_100a
only, -O3, -lineinfo, IEEE fp32 (no fast-math: the quantizer relies on exact
power-of-two scaling and on subnormals not being flushed).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "librfq.so")
BUILD_DIR = os.path.join(PKG, "_build")

SOURCES = ["rfq_api.cu", "rfq_quantize.cu", "rfq_gemm.cu", "rfq_static_ws.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-ftz=false", "-prec-div=true",
              "-prec-sqrt=true", "-fmad=true", "--expt-relaxed-constexpr", "-Wno-deprecated-declarations"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build librfq.so")
    return path


def _deps(src: str):
    heads = [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".h", ".cuh"))]
    return [src] + heads + [os.path.join(INCLUDE, "rfq.h")]


def _compile(src_name: str, verbose_ptxas: bool) -> str:
    src = os.path.join(CSRC, src_name)
    obj = os.path.join(BUILD_DIR, src_name.replace(".cu", ".o"))
    newest = max(os.path.getmtime(d) for d in _deps(src))
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest and not verbose_ptxas:
        return obj
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src_name}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile csrc/*.cu for sm_100a and link librfq.so next to this file."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    if force:
        for f in os.listdir(BUILD_DIR):
            os.remove(os.path.join(BUILD_DIR, f))
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas), SOURCES))
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(o) for o in objs)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
