"""Build libm3.so (the CUDA C-ABI library) in-tree for sm_100a.

Each .cu translation unit is compiled by its own nvcc process (in parallel),
then linked into autoregressive_audio_token_b200/libm3.so with the CUDA
runtime linked statically.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libm3.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]

SOURCES = ["m3.cu", "attention.cu", "gemv_tile.cu", "gemv_bf16.cu", "gemv_i8row.cu",
           "gemv_i8g128.cu", "gemm_tc.cu", "dit.cu", "dit_gemm.cu", "depth.cu"]


def _deps_mtime() -> float:
    files = ([os.path.join(CSRC, f) for f in os.listdir(CSRC)] +
             [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)] + [os.path.abspath(__file__)])
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, extra: list[str], bdir: str = BUILD) -> str:
    obj = os.path.join(bdir, os.path.splitext(src)[0] + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, out: str | None = None,
          defines: tuple = (), build_dir: str | None = None) -> str:
    """Compile libm3.so; `defines` (e.g. ("M3_STAGES=4",)) and `out` build a
    variant elsewhere for tuning sweeps."""
    lib = out or LIB
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _deps_mtime():
        return lib
    bdir = build_dir or BUILD
    os.makedirs(bdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    extra += [f"-D{d}" for d in defines]
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, bdir), SOURCES))
    tmp = lib + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-Xcompiler", "-fPIC"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas" in sys.argv))
