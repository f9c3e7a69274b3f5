"""Build libkq.so in-tree with nvcc for sm_100a (no JIT cache, no torch
extension machinery: the library exports a plain C ABI), and beside it
libkq_debug.so, the same sources built with KQ_DEBUG (device bounds checks
that set the error word, short bounded waits; include/kq_debug.h)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkq.so")
LIB_DEBUG = os.path.join(HERE, "libkq_debug.so")
# Rounds of one bounded wait in the debug build: milliseconds, so that a test
# can make a wait run out (the release build's limit is seconds).
DEBUG_SPIN_LIMIT = 16384
# variant -> (library, object folder, extra nvcc flags)
VARIANTS = {
    "release": (LIB, os.path.join(HERE, "_build"), []),
    "debug": (LIB_DEBUG, os.path.join(HERE, "_build", "debug"),
              ["-DKQ_DEBUG=1", f"-DKQ_SPIN_LIMIT={DEBUG_SPIN_LIMIT}u"]),
}
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(
        os.path.join(ROOT, "include", "*.h")) + [os.path.abspath(__file__)]


def stale(variant: str = "release") -> bool:
    lib = VARIANTS[variant][0]
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False, variants=("release", "debug")) -> str:
    """Compile the stale variants (all their sources at once) and link them;
    returns the release library's path."""
    todo = [v for v in variants if force or stale(v)]
    procs = []
    for v in todo:
        objdir, extra = VARIANTS[v][1], VARIANTS[v][2]
        os.makedirs(objdir, exist_ok=True)
        for s in sources():
            o = os.path.join(objdir, os.path.basename(s) + ".o")
            cmd = [NVCC, *FLAGS, *extra, "-rdc=false", "-c", s, "-o", o]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), file=sys.stderr)
            procs.append((s, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for s, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode:
            sys.stderr.write(out.decode(errors="replace"))
        if p.returncode:
            failed.append(s)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    for v in todo:
        lib, objdir = VARIANTS[v][0], VARIANTS[v][1]
        objs = [os.path.join(objdir, os.path.basename(s) + ".o") for s in sources()]
        tmp = lib + f".tmp{os.getpid()}"
        # -shared through nvcc links the static CUDA runtime; the driver library
        # is loaded at run time, so the .so also loads on a machine without a GPU.
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                               "-Xcompiler", "-fPIC", *objs, "-o", tmp])
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
