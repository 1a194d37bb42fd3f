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

SOURCES = ["rfq_api.cu", "rfq_quantize.cu", "rfq_gemm.cu", "rfq_linear_fused.cu", "rfq_static_ws.cu"]
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


def _compile(src_name: str, verbose_ptxas: bool, build_dir: str = BUILD_DIR, extra_flags=()) -> str:
    src = os.path.join(CSRC, src_name)
    obj = os.path.join(build_dir, src_name.replace(".cu", ".o"))
    newest = max(os.path.getmtime(d) for d in _deps(src))
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest and not verbose_ptxas and not extra_flags:
        return obj
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src_name}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, out_lib: str = LIB, extra_flags=()) -> str:
    """Compile csrc/*.cu for sm_100a and link librfq.so next to this file (or to
    `out_lib`, with `extra_flags` such as -D overrides of the kernels' tuning knobs)."""
    build_dir = BUILD_DIR if out_lib == LIB else os.path.join(os.path.dirname(out_lib), "_build")
    os.makedirs(build_dir, exist_ok=True)
    if force:
        for f in os.listdir(build_dir):
            os.remove(os.path.join(build_dir, f))
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, build_dir, tuple(extra_flags)), SOURCES))
    if (not force and not extra_flags and os.path.exists(out_lib)
            and os.path.getmtime(out_lib) >= max(os.path.getmtime(o) for o in objs)):
        return out_lib
    LIB_ = out_lib
    tmp = LIB_ + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB_)
    return LIB_


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
