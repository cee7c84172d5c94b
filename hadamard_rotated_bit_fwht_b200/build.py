"""Build the sm_100a shared library libkvq.so in-tree with nvcc.

    python -m hadamard_rotated_bit_fwht_b200.build
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkvq.so")
# the same sources compiled with KVQ_DEBUG_BOUNDS: every computed cache,
# slot and scale-row address is checked against its buffer, and a violation
# is recorded in the device error word (kvq_device_errors) instead of accessed
LIB_DEBUG = os.path.join(PKG, "libkvq_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "kvq.h")]
    return any(os.path.getmtime(p) > t for p in deps)


OBJ_DIR = os.path.join(ROOT, "_build", "kvq")


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every .cu to an object in parallel (relocatable device code is
    not needed: no kernel calls across files), then link libkvq.so (or, with
    debug=True, libkvq_debug.so with the bounds checks compiled in)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    from concurrent.futures import ThreadPoolExecutor
    os.makedirs(OBJ_DIR, exist_ok=True)
    compile_flags = [f for f in FLAGS if f not in ("--shared",)]
    if debug:
        compile_flags += ["-DKVQ_DEBUG_BOUNDS"]
    tag = f".{'dbg' if debug else 'rel'}{os.getpid()}"

    def compile_one(src):
        obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + tag + ".o")
        cmd = [NVCC, *compile_flags, "-I", INCLUDE, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
            print(" ".join(cmd))
        subprocess.check_call(cmd)
        return obj

    srcs = sources()
    with ThreadPoolExecutor(min(len(srcs), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "--shared",
                           "-Xcompiler", "-fPIC", "-o", tmp, *objs])
    os.replace(tmp, lib)
    for o in objs:
        os.remove(o)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
