"""Builds libpariskv.so in-tree for sm_100a with nvcc (no JIT cache, no torch extension).

    python -m long_context_kv_srht_b200.build [--force] [--verbose] [--check]

Objects go to ``long_context_kv_srht_b200/_build/``; the library to
``long_context_kv_srht_b200/_lib/libpariskv.so``. ``--check`` builds the checked variant
``libpariskv_check.so`` instead (objects in ``_build_check/``): the same kernels compiled with
PKV_CHECK=1, whose extra device-side checks record ST_BADINDEX in the index's status word and
skip the access (they never trap). The binding loads it when PARISKV_LIBRARY=check.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG, "_build")
LIB_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIB_DIR, "libpariskv.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc" if os.path.exists(
    "/usr/local/cuda/bin/nvcc") else "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
                "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.hpp")) + glob.glob(os.path.join(INCLUDE, "*.h"))


CHECK_OBJ_DIR = os.path.join(PKG, "_build_check")
CHECK_LIB = os.path.join(LIB_DIR, "libpariskv_check.so")


def _compile(src: str, verbose: bool, check: bool = False) -> str:
    obj = os.path.join(CHECK_OBJ_DIR if check else OBJ_DIR, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *FLAGS, *(["-DPKV_CHECK=1"] if check else []), "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    """Compile every kernel source for sm_100a and link libpariskv.so (or, with check, the
    checked libpariskv_check.so); skipped when current."""
    lib = CHECK_LIB if check else LIB
    if not force and up_to_date(lib):
        return lib
    os.makedirs(CHECK_OBJ_DIR if check else OBJ_DIR, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, check), sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "--cudart", "static", *objs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                check="--check" in sys.argv))
