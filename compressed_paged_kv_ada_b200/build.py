"""Build libsphkv.so (all CUDA kernels + the C ABI) in-tree for sm_100a.

    python -m compressed_paged_kv_ada_b200.build [--force] [--verbose]

It also builds two variants that only the tests load; the product library is
built without their flags:
- libsphkv_testhooks.so: decode.cu compiled with -DSPHKV_TEST_HOOKS (the tests
  use it to make a bounded device wait run out without any fault);
- libsphkv_debug.so: decode.cu compiled with -DSPHKV_DEBUG (every shared-memory
  table address checked against its table, a canary past each shorter page
  copy, and a stream synchronisation after every call).

encode.cu and rdr.cu are compiled with -fmad=false: their fp64 arithmetic must
not be contracted into fused multiply-adds (codes and tier decisions are
compared bit for bit with a plain fp64 reference).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsphkv.so")
TEST_LIB = os.path.join(HERE, "libsphkv_testhooks.so")
DEBUG_LIB = os.path.join(HERE, "libsphkv_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
SOURCES = {
    "api.cu": [],
    "encode.cu": ["-fmad=false"],
    "rdr.cu": ["-fmad=false"],
    "decode.cu": [],
    "splitkv.cu": [],
    "keep.cu": [],
}


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(ROOT, "include", "sphkv.h"))
    files.append(os.path.abspath(__file__))
    return files


def _link(objs, out):
    tmp = out + ".tmp"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"])
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    newest = max(os.path.getmtime(f) for f in _deps())
    if not force and all(os.path.exists(f) and os.path.getmtime(f) >= newest for f in (LIB, TEST_LIB, DEBUG_LIB)):
        return LIB
    objs = {}
    variants = [("decode.cu#hooks", ["-DSPHKV_TEST_HOOKS"]), ("decode.cu#debug", ["-DSPHKV_DEBUG"])]
    for src, extra in list(SOURCES.items()) + variants:
        name = src.split("#")[0]
        obj = os.path.join(BUILD, src.replace(".cu", "").replace("#", "_") + ".o")
        cmd = [NVCC, *ARCH, *COMMON, *extra, "-c", os.path.join(CSRC, name), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        objs[src] = obj
    _link([objs[s] for s in SOURCES], LIB)
    _link([objs[s] for s in SOURCES if s != "decode.cu"] + [objs["decode.cu#hooks"]], TEST_LIB)
    _link([objs[s] for s in SOURCES if s != "decode.cu"] + [objs["decode.cu#debug"]], DEBUG_LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
