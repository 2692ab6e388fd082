"""Build libqmoe.so (the CUDA library behind the C ABI) and libqmoe_synth.so.

Both are compiled in-tree for sm_100a with nvcc: one object per .cu file
(rebuilt only when a source or header is newer), then one shared library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "quantised_expert_decode_b200")
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libqmoe.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "csrc", "synth_fill.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libqmoe_synth.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
BASE_FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC"] + ARCH
FLAGS = BASE_FLAGS + ["-Xcompiler", "-fvisibility=hidden"]


def _newest(paths):
    return max((os.path.getmtime(p) for p in paths), default=0.0)


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return r.stdout + r.stderr


def _compile(src, headers, obj, extra):
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), _newest(headers)):
        return obj
    _run([NVCC] + FLAGS + extra + ["-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj])
    return obj


def build_qmoe(verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    objs = [os.path.join(BUILD, os.path.basename(s) + ".o") for s in srcs]
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        list(ex.map(lambda so: _compile(so[0], headers, so[1], ["-DQMOE_BUILD"]), zip(srcs, objs)))
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < _newest(objs):
        _run([NVCC] + ARCH + ["-shared", "-o", LIB] + objs)
    if verbose:
        print("built", LIB)
    return LIB


def build_synth(verbose: bool = False) -> str:
    if not os.path.exists(SYNTH_LIB) or os.path.getmtime(SYNTH_LIB) < os.path.getmtime(SYNTH_SRC):
        _run([NVCC] + BASE_FLAGS + ["-shared", SYNTH_SRC, "-o", SYNTH_LIB])
    if verbose:
        print("built", SYNTH_LIB)
    return SYNTH_LIB


def build(verbose: bool = False):
    return build_qmoe(verbose), build_synth(verbose)


if __name__ == "__main__":
    build(verbose=True)
    sys.exit(0)
