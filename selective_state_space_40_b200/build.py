"""Build libmambascan.so in-tree with nvcc for sm_100a (B200).

    python -m selective_state_space_40_b200.build [--verbose]

The library links the CUDA runtime statically, so it loads on a machine
without a GPU (every entry point then returns MS_ERR_CUDA).
"""
from __future__ import annotations

import glob
import hashlib
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmambascan.so")
# the same sources with MS_DEBUG: device bounds checks record MS_ERR_BOUNDS
LIB_DEBUG = os.path.join(PKG, "libmambascan_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]
LINK_FLAGS = [*ARCH, "-shared", "-cudart", "static"]
# kept for callers that want the one-shot command line
NVCC_FLAGS = [*COMPILE_FLAGS, "-shared", "-cudart", "static"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    """Every header the sources include: csrc/*.h, csrc/*.cuh and include/*.h.
    An edit to any of them rebuilds every object (they key the object cache)."""
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    mt = os.path.getmtime(LIB)
    deps = sources() + headers()
    return any(os.path.getmtime(p) > mt for p in deps)


def _run(cmd):
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    return res.stdout + res.stderr


def build_debug(force: bool = False) -> str:
    """The MS_DEBUG variant of the library (a test artefact, never loaded by
    the product path)."""
    if not force and os.path.exists(LIB_DEBUG):
        mt = os.path.getmtime(LIB_DEBUG)
        deps = sources() + headers()
        if all(os.path.getmtime(p) <= mt for p in deps):
            return LIB_DEBUG
    return build(force=True, defines=("MS_DEBUG",), out=LIB_DEBUG)


def build(force: bool = False, verbose: bool = False, defines=(), out: str = LIB) -> str:
    """Compile every .cu under csrc/ to an object (in parallel), then link the
    shared library. ``defines`` are extra -D flags (a separate ``out`` path
    must be given for a variant build)."""
    if defines and os.path.abspath(out) == os.path.abspath(LIB):
        raise ValueError("a variant build must not overwrite the product library")
    if not force and out == LIB and not needs_build():
        return LIB
    tag = f"{os.getpid()}"
    # objects are cached under _build/ by a hash of their inputs (source,
    # every header, flags), so an edit recompiles only what it touches
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = [*COMPILE_FLAGS, *(f"-D{d}" for d in defines), "-I", INCLUDE, "-I", CSRC]
    if verbose:
        flags.insert(0, "-Xptxas=-v")
    common = hashlib.sha256(" ".join(flags).encode())
    for h in headers():
        with open(h, "rb") as f:
            common.update(f.read())
    srcs = sources()

    def obj_for(src):
        h = common.copy()
        with open(src, "rb") as f:
            h.update(f.read())
        return os.path.join(objdir, os.path.basename(src)[:-3] + "." + h.hexdigest()[:16] + ".o")

    objs = [obj_for(s) for s in srcs]
    todo = [(s, o) for s, o in zip(srcs, objs) if verbose or not os.path.exists(o)]

    def compile_one(so):
        tmp_o = so[1] + f".tmp{tag}"
        log = _run([nvcc(), *flags, "-c", so[0], "-o", tmp_o])
        os.replace(tmp_o, so[1])
        return log

    with ThreadPoolExecutor(max_workers=max(1, min(len(todo) or 1, os.cpu_count() or 1))) as pool:
        logs = list(pool.map(compile_one, todo))
    tmp = out + f".tmp{tag}"
    _run([nvcc(), *LINK_FLAGS, *objs, "-o", tmp])
    if verbose:
        sys.stdout.write("".join(logs))
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
    if "--debug" in sys.argv:
        print(build_debug(force=True))
