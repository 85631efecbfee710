"""Build step for the CUDA libraries (sm_100a, in-tree).

``python -m bit_w4a4_quantized_svdq_b200.build`` compiles every ``csrc/*.cu``
with nvcc for ``sm_100a`` into ``bit_w4a4_quantized_svdq_b200/libsvdq.so``
(release) and ``libsvdq_debug.so`` (the same source with SVDQ_DEBUG_CHECKS=1:
pointer checks on the host, store bounds checks in the kernels).  The two are
compiled concurrently.  nvcc cross-compiles, so this runs on machines without
a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libsvdq.so")
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libsvdq_debug.so")
VARIANT_FLAGS = {LIB_PATH: [], DEBUG_LIB_PATH: ["-DSVDQ_DEBUG_CHECKS=1"]}
INCLUDE = os.path.join(os.path.dirname(PKG_DIR), "include")

SOURCES = ["abi.cu", "calib.cu", "quantize.cu", "linear.cu", "score.cu", "residual.cu", "proxy.cu", "grid.cu", "mxfp8.cu"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the sm_100a library cannot be built")


def needs_build(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "svdq.h")]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Compile the release library (and, with ``debug``, the debug one) where a
    source is newer than it (or ``force``); return the release library's path."""
    targets = [p for p in ([LIB_PATH, DEBUG_LIB_PATH] if debug else [LIB_PATH]) if force or needs_build(p)]
    procs = []
    for path in targets:
        cmd = [nvcc_path(), *NVCC_FLAGS, *VARIANT_FLAGS[path], "-I", INCLUDE, "-o", path + ".tmp"] + \
              [os.path.join(CSRC, s) for s in SOURCES]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((path, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)))
    failed = []
    for path, proc in procs:
        out, err = proc.communicate()
        if proc.returncode != 0:
            failed.append(f"{os.path.basename(path)}: nvcc failed ({proc.returncode}):\n{out}\n{err}")
        else:
            os.replace(path + ".tmp", path)
    if failed:
        raise RuntimeError("\n".join(failed))
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
