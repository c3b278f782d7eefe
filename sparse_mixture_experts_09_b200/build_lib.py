"""Build step: compile csrc/*.cu for sm_100a into the in-tree shared library libmoe.so.

    python -m sparse_mixture_experts_09_b200.build_lib [--verbose-ptxas]

nvcc cross-compiles without a GPU. The library links the CUDA runtime statically and
reaches the driver's tensor-map encoder through cudaGetDriverEntryPointByVersion, so it
needs no libcuda at link time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe.so")
SOURCES = ["moe_api.cu", "routing.cu", "gemm_sm100.cu", "gemm_w8.cu", "combine.cu", "moe_noalloc.cu",
           "gather_rows.cu", "ep_peer.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "moe.h")]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose_ptxas: bool = False, extra_flags=(), out: str = LIB) -> str:
    """Compile into ``out`` (default: the in-tree libmoe.so) unless it is up to date."""
    if not force and out == LIB and not _stale():
        return LIB
    objdir = os.path.join(ROOT, "_build", os.path.basename(os.path.dirname(os.path.abspath(out))))
    os.makedirs(objdir, exist_ok=True)
    objs = []
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                    "-I", os.path.join(ROOT, "include")]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    flags += list(extra_flags)
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [nvcc()] + flags + ["-c", os.path.join(CSRC, src), "-o", obj]
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = out + ".tmp"
    subprocess.run([nvcc()] + ARCH + ["-shared", "-o", tmp] + objs, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
