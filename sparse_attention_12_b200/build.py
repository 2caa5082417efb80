"""Build the in-tree C-ABI library libdsa.so for sm_100a with nvcc.

    python -m sparse_attention_12_b200.build [--force] [--ptxas-v]

Every .cu file is compiled to an object on its own (in parallel), then linked into one shared
library. The library links the CUDA runtime statically and reaches the driver only through the
runtime's entry-point query, so it loads on a machine without a GPU driver (for symbol checks) and
runs on a B200.

build(out=..., extra=[...]) builds a variant under another name with extra flags; the tests use
that for a fault-injection build (-DDSA_TEST_FAULTS), which is never the product library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libdsa.so")
FAULTS_LIB = os.path.join(PKG, "libdsa_testfaults.so")
FAULTS_FLAGS = ("-DDSA_TEST_FAULTS", "-DDSA_WAIT_LIMIT_NS=20000000ull")  # waits give up after 20 ms
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O3",
          "-I", os.path.join(ROOT, "include")]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "dsa.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return r.stdout + r.stderr


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB) -> str:
    if not force and not _stale(out):
        return out
    srcs = sources()
    with tempfile.TemporaryDirectory(prefix="dsa_build_") as tmp:
        objs = [os.path.join(tmp, os.path.basename(s) + ".o") for s in srcs]
        cmds = [[NVCC, *ARCH_FLAGS, *CFLAGS, *extra, "-c", s, "-o", o] for s, o in zip(srcs, objs)]
        workers = max(1, min(len(cmds), len(os.sched_getaffinity(0))))
        with ThreadPoolExecutor(workers) as ex:
            logs = list(ex.map(_run, cmds))
        tmp_out = out + ".tmp"
        logs.append(_run([NVCC, *ARCH_FLAGS, "-shared", "-cudart", "static", "-o", tmp_out, *objs]))
        if verbose:
            print("\n".join(" ".join(c) for c in cmds))
            print("".join(logs))
        os.replace(tmp_out, out)
    return out


def build_faults(force: bool = False) -> str:
    """The fault-injection variant used by the bounded-wait test (not the product library)."""
    return build(force=force, extra=FAULTS_FLAGS, out=FAULTS_LIB)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    print(LIB)
