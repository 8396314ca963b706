"""Builds libsparselora.so in-tree with nvcc for sm_100a (no GPU needed).

    python -m contextual_sparsity_lora_b200.build [--debug] [-v]

--debug builds libsparselora_debug.so instead: the same sources compiled with -DSL_DEBUG_BOUNDS,
whose kernels check every index read from a channel set, row permutation or gather list against the
extent it indexes before using it (a failing check skips the access and records a code in the error
word; see sl_debug_bounds_enabled in include/sparselora.h). Objects go to _build/ (release) and
_build_debug/ (debug).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsparselora.so")
DEBUG_LIB = os.path.join(HERE, "libsparselora_debug.so")
SOURCES = ["sl_api.cu", "sl_gemm.cu", "sl_estimator.cu", "sl_select.cu", "sl_aux.cu", "sl_lora.cu", "sl_noalloc.cu", "sl_est_tc.cu", "sl_criteria.cu", "sl_layer.cu", "sl_attention.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def build(verbose: bool = False, extra: list[str] | None = None, debug: bool = False) -> str:
    """Compile every CUDA source and link the shared library (the debug build with debug=True).
    The sources compile in parallel. Returns the library's path."""
    objdir = os.path.join(HERE, "_build_debug" if debug else "_build")
    out = DEBUG_LIB if debug else LIB
    os.makedirs(objdir, exist_ok=True)
    common = [nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "-I" + os.path.join(ROOT, "include")] + (["-DSL_DEBUG_BOUNDS"] if debug else []) + (extra or [])
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = common + ["-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.append("-Xptxas=-v")
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)))
        objs.append(obj)
    for src, p in procs:
        _, err = p.communicate()
        if p.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{err}")
        if verbose and err:
            print(err, file=sys.stderr)
    # the driver API (tensor-map encoding) is reached through the runtime's entry-point query: no -lcuda
    cmd = [nvcc(), *ARCH, "-shared", "-o", out, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, debug="--debug" in sys.argv))
