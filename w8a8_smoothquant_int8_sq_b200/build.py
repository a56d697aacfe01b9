"""Build libsq.so in-tree for sm_100a with nvcc.

    python -m w8a8_smoothquant_int8_sq_b200.build [--verbose-ptxas]

The shared library lands next to this file (``libsq.so``) so that it travels
with the source tree.  cudart is linked statically; the driver API entry point
used for tensor maps is resolved at run time through cudart, so the library
needs no link-time libcuda.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsq.so")
SOURCES = ["sq_api.cu", "sq_quant.cu", "sq_gemm.cu", "sq_weight_only.cu", "sq_ste.cu", "sq_aux.cu"]
HEADERS = ["sq_device.cuh", "sq_internal.h", "sq_gemm_small.cuh", "sq_gemm_splitk.cuh", "sq_gemm_pair.cuh", "sq_gemm_prologue.cuh", os.path.join("..", "..", "include", "sq.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [os.path.join(CSRC, h) for h in HEADERS]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose_ptxas: bool = False, out: str = LIB, defines=()) -> str:
    """Compile every CUDA source into a shared library for sm_100a (libsq.so
    next to this file by default).  ``defines`` are extra -D tuning macros.
    Returns the library path."""
    if out == LIB and not defines and not force and not verbose_ptxas and not _stale():
        return LIB
    tmp = out + ".tmp"
    cmd = [nvcc()] + ARCH + FLAGS + [f"-D{d}" for d in defines] + ["-shared", "-o", tmp] + \
        [os.path.join(CSRC, s) for s in SOURCES]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose_ptxas:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
