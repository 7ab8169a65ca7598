"""Builds libqattn.so in-tree with nvcc for sm_100a (no GPU needed to compile), and with
``--checked`` (or QATTN_DEBUG=1 in the environment) also the checked build libqattn_checked.so:
the same sources compiled with QATTN_CHECKED, whose kernels test the global-memory indices they
compute against their buffers' extents and record QATTN_ERR_BOUNDS instead of trapping.  The
binding loads the checked library when QATTN_DEBUG=1 is set.

    python -m precision_quantized_attention_b200.build [--checked] [-v]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libqattn.so")
LIB_CHECKED = os.path.join(HERE, "libqattn_checked.so")
SOURCES = ["qattn_api.cu", "quant.cu", "attn_fwd.cu", "attn_pair.cu", "attn_debug.cu", "noalloc.cu",
           "gemm_fp8.cu", "gemm_fp4.cu"]
HEADERS = ["sm100_ptx.cuh", "softmax_sm100.cuh", "launch.h", "device_once.h", "quant_math.cuh",
           "tensor_map.h"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def flags(verbose_ptxas: bool = False) -> list[str]:
    f = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE,
         "--expt-relaxed-constexpr"]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    return f


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "qattn.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    """Builds libqattn.so (checked=False) or libqattn_checked.so (checked=True) if stale."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *flags(verbose_ptxas), *(["-DQATTN_CHECKED"] if checked else []), "-shared",
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    v = "-v" in sys.argv
    print(build(force=True, verbose_ptxas=v))
    if "--checked" in sys.argv or os.environ.get("QATTN_DEBUG") == "1":
        print(build(force=True, verbose_ptxas=v, checked=True))
