"""Build ``libgqa.so`` (the CUDA kernels behind the C ABI of include/gqa.h).

The library is compiled in-tree for sm_100a only, with nvcc:

    python -m kv_cache_bandwidth_b200.build [--force] [--verbose]

The ptxas resource report (registers, spills, shared memory per kernel) is kept
in ``kv_cache_bandwidth_b200/_build/ptxas.log``.

A second library, ``libgqa_test_hooks.so``, is the same sources built for the
bounded-wait tests: every wait gives up after ~10 ms instead of ~2 s, and an
extra entry point (gqa_test_skip_tile) makes one block's producer leave one
K/V tile out so that a wait runs out.  Nothing but those tests loads it.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgqa.so")
TEST_LIB = os.path.join(PKG, "libgqa_test_hooks.so")
BUILD_DIR = os.path.join(PKG, "_build")
# the test library's wait limit: ~10 ms at the B200's clocks
TEST_FLAGS = ["-DGQA_TEST_HOOKS", "-DGQA_WAIT_LIMIT_CYCLES=20000000ll"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH_FLAGS + [
    "-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
    "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC,
]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgqa")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "gqa.h"), __file__]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Build libgqa.so and libgqa_test_hooks.so (two nvcc runs in parallel);
    returns the path of libgqa.so."""
    jobs = [(lib, extra, log) for lib, extra, log in ((LIB, [], "ptxas.log"),
                                                      (TEST_LIB, TEST_FLAGS, "ptxas_test_hooks.log"))
            if force or not up_to_date(lib)]
    if not jobs:
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    procs = []
    for lib, extra, log in jobs:
        tmp = lib + ".tmp.%d" % os.getpid()
        cmd = [nvcc()] + NVCC_FLAGS + extra + ["-o", tmp] + sources()
        procs.append((lib, tmp, log, cmd,
                      subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)))
    failed = None
    for lib, tmp, log, cmd, proc in procs:
        out, err = proc.communicate()
        with open(os.path.join(BUILD_DIR, log), "w") as f:
            f.write(" ".join(cmd) + "\n" + out + err)
        if proc.returncode != 0:
            sys.stderr.write(out + err)
            failed = failed or "nvcc failed building %s (exit %d)" % (os.path.basename(lib), proc.returncode)
            continue
        if verbose:
            sys.stderr.write(err)
        os.replace(tmp, lib)
    if failed:
        raise RuntimeError(failed)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
