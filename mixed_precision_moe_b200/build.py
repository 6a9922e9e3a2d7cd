"""Build libmoe.so (the library's compute path) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe.so")
LIB_TRACE = os.path.join(HERE, "libmoe_trace.so")  # profiling build, see ffn_trace.py
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    """Compile csrc/moe_lib.cu (which includes every kernel) into libmoe.so, or
    with trace=True into the profiling build libmoe_trace.so (-DMOE_FFN_TRACE:
    the grouped FFN records a per-unit timeline, see ffn_trace.py)."""
    out = LIB_TRACE if trace else LIB
    newest = max(os.path.getmtime(p) for p in sources() +
                 [os.path.join(HERE, "..", "include", "moe.h")])
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, "-std=c++17", "-O3", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xptxas", "-v" if verbose else "-O3"]
    if trace:
        cmd.append("-DMOE_FFN_TRACE")
    cmd += ["-o", tmp, os.path.join(CSRC, "moe_lib.cu")]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv))
