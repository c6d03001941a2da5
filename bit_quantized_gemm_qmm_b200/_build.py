"""Build the CUDA library in-tree: csrc/*.cu -> libqmm_b200.so (sm_100a only), and the small
CPython module _qmm_call that hands each qmm() call to the library's C ABI.

Each translation unit is compiled on its own (in parallel) and linked into one shared
library with the CUDA runtime linked statically, so the .so loads on a host without a GPU
(the C ABI can be inspected there) and carries no JIT step at run time.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys
import sysconfig

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libqmm_b200.so")
CALL_SRC = os.path.join(HERE, "_qmm_call.c")
CALL_LIB = os.path.join(HERE, "_qmm_call" + (sysconfig.get_config_var("EXT_SUFFIX") or ".so"))
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(srcs, target) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + [os.path.join(HERE, "..", "include", "qmm.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build_call_module(force: bool = False) -> str:
    """gcc the CPython hand-off module (plain C against the interpreter's headers)."""
    if not force and os.path.exists(CALL_LIB) and os.path.getmtime(CALL_LIB) >= max(
            os.path.getmtime(CALL_SRC), os.path.getmtime(__file__)):
        return CALL_LIB
    cc = os.environ.get("CC") or shutil.which("gcc") or shutil.which("cc")
    if not cc:
        raise RuntimeError("no C compiler for the _qmm_call module")
    tmp = CALL_LIB + ".tmp"
    subprocess.check_call([cc, "-O2", "-shared", "-fPIC", "-Wall", "-Werror",
                           "-I" + sysconfig.get_paths()["include"], CALL_SRC, "-o", tmp])
    os.replace(tmp, CALL_LIB)
    return CALL_LIB


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    build_call_module(force)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if not force and not _stale(srcs, LIB):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(compile_one, srcs))
    if verbose or ptxas_info:
        for _, log in results:
            if log.strip():
                print(log, file=sys.stderr)
    objs = [o for o, _ in results]
    tmp = LIB + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
