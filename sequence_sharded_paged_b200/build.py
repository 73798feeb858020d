"""Build libdcp.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

Each .cu under csrc/ is compiled separately (objects cached under
_build/) and linked into ``libdcp.so`` next to this file.  Also builds
``synth/libsynth.so`` (device fill of the seeded inputs).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdcp.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "synth_fill.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libsynth.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "dcp.h")]
    return max(os.path.getmtime(f) for f in files)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"build failed: {' '.join(cmd[:4])} ...")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return r


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    dep_t = _deps_mtime()
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    objs = []
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    for src in srcs:
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or ptxas_info or not os.path.exists(obj) or os.path.getmtime(obj) < dep_t:
            _run([NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj], verbose or ptxas_info)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        _run([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs], verbose)
    if force or not os.path.exists(SYNTH_LIB) or os.path.getmtime(SYNTH_LIB) < max(
            os.path.getmtime(SYNTH_SRC), os.path.getmtime(os.path.join(ROOT, "synth", "synth_hash.h"))):
        _run([NVCC, *ARCH, *FLAGS, "-shared", "-cudart", "static", "-o", SYNTH_LIB, SYNTH_SRC], verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
