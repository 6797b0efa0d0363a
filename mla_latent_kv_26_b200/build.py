"""Build ``libmla.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m mla_latent_kv_26_b200.build [--force] [--verbose]``.
The library links the CUDA runtime statically and exports only the C ABI of
``include/mla.h``.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmla.so")
SOURCES = ["mla_api.cu", "mla_decode.cu", "mla_plan_combine.cu", "mla_insert.cu", "mla_absorb.cu",
           "mla_indexer.cu"]
HEADERS = ["common.cuh", "sm100.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "mla.h"))
    files.append(os.path.abspath(__file__))
    return files


# A test build in which the indexer kernel's pipeline waits give up after
# 200 ns, so that the bounded-wait error path runs (tests/test_timeout.py).
SHORT_WAIT_LIB = os.path.join(HERE, "libmla_shortwait.so")
SHORT_WAIT_DEFINES = ["-DMLA_WAIT_LIMIT_NS=200ull"]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _compile(lib: str, defines, verbose: bool) -> str:
    cmd = [
        nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
        "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC, *defines,
        *[os.path.join(CSRC, f) for f in SOURCES], "-o", lib + ".tmp",
    ]
    if verbose:
        cmd.insert(-2, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date(LIB):
        _compile(LIB, [], verbose)
    return LIB


def build_short_wait(force: bool = False) -> str:
    """The test build with 200 ns pipeline waits in the indexer kernel."""
    if force or not up_to_date(SHORT_WAIT_LIB):
        _compile(SHORT_WAIT_LIB, SHORT_WAIT_DEFINES, False)
    return SHORT_WAIT_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
    if "--short-wait" in sys.argv:
        print(build_short_wait(force="--force" in sys.argv))
