"""Build librecsa.so in-tree for sm_100a with nvcc.

Usage: python -m long_context_recsa_b200.build   (or build() from Python)
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "librecsa.so")
SOURCES = ["recsa_api.cu", "tree_kernels.cu", "select_attend.cu", "prefill_tc.cu", "noalloc.cu",
           "gated.cu", "offload.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found")


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


OUT_BOUNDS = os.path.join(HERE, "librecsa_bounds.so")


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile the library (librecsa.so), or with debug_bounds the bounds-checked
    variant (librecsa_bounds.so: every gather row and selection rank is range-checked
    on the device and a failure is recorded in the status word)."""
    out = OUT_BOUNDS if debug_bounds else OUT
    deps = [os.path.join(CSRC, s) for s in SOURCES]
    deps += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(HERE, "..", "include", "recsa.h"))
    if not force and not _stale(out, deps):
        return out
    cmd = [nvcc_path(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-o", out + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    if debug_bounds:
        cmd.insert(1, "-DRECSA_DEBUG_BOUNDS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug_bounds="--bounds" in sys.argv))
