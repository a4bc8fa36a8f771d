"""Build libmoe.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m expert_dispatch_gate_b200.build [--force]``. Objects go to ``_build/`` next
to this file; the shared library lands at ``expert_dispatch_gate_b200/libmoe.so``. ptxas
resource usage (registers, spills, shared memory) is written to ``_build/ptxas.log``.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmoe.so")
# Debug variant (-DMOE_DEBUG): every slot, token-row and group-table index a kernel reads from
# device data is checked before use; a failure is recorded in the workspace error word.
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libmoe_debug.so")
SOURCES = ["moe_api.cu", "route.cu", "route_tc.cu", "align.cu", "combine.cu", "ffn_simt.cu",
           "ffn_tc.cu", "quant.cu", "probe.cu", "ep.cu"]
# every header under csrc/: a change to any of them rebuilds every object
HEADERS = sorted(f for f in os.listdir(CSRC) if f.endswith((".cuh", ".h")))

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
                "--expt-relaxed-constexpr", "-Xptxas", "-v", "-I", INCLUDE]


def nvcc():
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe.so")
    return p


def _deps_mtime():
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "moe.h"), __file__]
    return max(os.path.getmtime(p) for p in paths)


def _compile(src, force, debug=False):
    obj = os.path.join(BUILD_DEBUG if debug else BUILD, src.replace(".cu", ".o"))
    srcp = os.path.join(CSRC, src)
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(srcp), _deps_mtime())):
        return obj, ""
    cmd = [nvcc()] + FLAGS + (["-DMOE_DEBUG"] if debug else []) + ["-c", srcp, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    bdir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, len(SOURCES))) as ex:
        results = list(ex.map(lambda s: _compile(s, force, debug), SOURCES))
    objs = [o for o, _ in results]
    logs = "".join(l for _, l in results)
    if logs:
        with open(os.path.join(bdir, "ptxas.log"), "w") as f:
            f.write(logs)
    if (force or not os.path.exists(lib)
            or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs)):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if verbose:
        print(logs)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true",
                    help="build libmoe_debug.so with the device-side bounds checks")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))
    sys.exit(0)
