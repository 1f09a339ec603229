"""Build the sm_100a shared library ``libfp4q.so`` in-tree with nvcc.

    python -m fp4_micro_block_b200.build [--force]

The library is a plain C ABI (``include/fp4q.h``); nothing here links against
torch.  ``-gencode arch=compute_100a,code=sm_100a`` targets B200 only; no
fast-math, so IEEE division and square root stay correctly rounded.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfp4q.so")
HEADER = os.path.join(ROOT, "include", "fp4q.h")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-Xptxas", "-v",
    "-shared",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")))


TEST_LIB = os.path.join(PKG, "libfp4q_test.so")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources() + [HEADER])


def build(force: bool = False, verbose: bool = False, test_hooks: bool = False,
          defines: tuple = (), out: str | None = None) -> str:
    """Builds libfp4q.so, or with test_hooks the test build libfp4q_test.so
    (bounded waits cut short and a hook that withholds one tile, so that a
    test can drive the kernels' timeout path).  `defines` (NAME=VALUE) and
    `out` build a variant of the library elsewhere, e.g.
    FP4Q_REGISTER_FWHT_MAX=64 (rotations up to 64 on the register path)."""
    lib = out or (TEST_LIB if test_hooks else LIB)
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    extra = (["-DFP4Q_TEST_HOOKS"] if test_hooks else []) + [f"-D{d}" for d in defines]
    cmd = [nvcc(), *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), os.path.join(CSRC, "fp4q.cu"),
           "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    with open(os.path.join(PKG, "build_test.log" if test_hooks else "build.log"), "w") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + log[-8000:])
    if verbose:
        print(log)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import argparse

    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", action="store_true")
    ap.add_argument("--test", action="store_true", help="the test build (libfp4q_test.so)")
    ap.add_argument("--define", action="append", default=[], help="NAME=VALUE for a library variant")
    ap.add_argument("--out", default=None, help="output path of a library variant")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.v, test_hooks=a.test, defines=tuple(a.define), out=a.out))
