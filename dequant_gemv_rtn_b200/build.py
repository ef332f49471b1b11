"""Build libqnt.so in-tree: hand-written CUDA for sm_100a plus the C ABI.

    python -m dequant_gemv_rtn_b200.build [-v] [--force]
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libqnt.so")
TEST_OBJ = os.path.join(PKG, "_build_test")
TEST_LIB = os.path.join(PKG, "libqnt_test.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC,
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(lib: str = None) -> bool:
    lib = lib or LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, verbose: bool, ptxas_v: bool, objdir: str = None, extra=()) -> str:
    obj = os.path.join(objdir or OBJ, os.path.basename(src) + ".o")
    cmd = ["nvcc", *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if ptxas_v and src.endswith(".cu"):
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if ptxas_v:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False, test: bool = False) -> str:
    """Build libqnt.so; with test=True the test library libqnt_test.so instead
    (the same sources compiled with QNT_TEST_FAULTS: fault injection for the
    tests of the bounded waits; the product library never contains it)."""
    lib, obj, extra = (TEST_LIB, TEST_OBJ, ["-DQNT_TEST_FAULTS"]) if test else (LIB, OBJ, [])
    if not force and up_to_date(lib):
        return lib
    os.makedirs(obj, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, ptxas_v, obj, extra), _sources()))
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib, *objs, "-lcudart"]
    if test:   # its own calls bind to its own definitions, even beside libqnt.so
        cmd += ["-Xlinker", "-Bsymbolic"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, ptxas_v="--ptxas-v" in sys.argv,
                test="--test" in sys.argv))
