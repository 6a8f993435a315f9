"""Build libsge.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python -m activation_sparse_gated_epilogue_b200.build [--force] [--debug]

Objects are compiled in parallel into ``_build/`` next to this file and
linked into ``libsge.so`` beside the Python binding.  The CUDA runtime is
linked statically, so the library needs only the driver at run time.
``--debug`` also builds ``libsge_debug.so`` (objects in ``_build_debug/``):
the same sources compiled with SGE_DEBUG, whose kernels check every
data-driven index (``sge_debug_flags``); the binding loads it when the
environment sets SGE_DEBUG=1.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsge.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libsge_debug.so")
# the test-only self-test library (failure handling of the GEMM engines)
SELFTEST_SRC = os.path.join(CSRC, "selftest", "selftest.cu")
SELFTEST_LIB = os.path.join(HERE, "libsge_selftest.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE,
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, inputs):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in inputs)


def _compile(src, verbose, obj=None, extra=()):
    obj = obj or os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    deps = _deps()
    todo = [s for s in srcs if force or _stale(os.path.join(BUILD, os.path.basename(s)[:-3] + ".o"), [s, *deps])]
    logs = []
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            for obj, log in ex.map(lambda s: _compile(s, verbose), todo):
                logs.append(log)
    objs = [os.path.join(BUILD, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if force or todo or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               "-Xcompiler", "-fPIC", *objs, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    _build_selftest(force, verbose)
    if verbose:
        for log in logs:
            sys.stderr.write(log)
    return LIB


def _build_selftest(force: bool, verbose: bool) -> str:
    """libsge_selftest.so: the self-test kernels plus the host helpers."""
    obj = os.path.join(BUILD, "selftest.o")
    host = os.path.join(BUILD, "host.o")
    if force or _stale(obj, [SELFTEST_SRC, *_deps()]):
        _compile(SELFTEST_SRC, verbose, obj)
    if force or _stale(SELFTEST_LIB, [obj, host]):
        tmp = SELFTEST_LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               "-Xcompiler", "-fPIC", obj, host, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, SELFTEST_LIB)
    return SELFTEST_LIB


def build_debug(force: bool = False) -> str:
    """libsge_debug.so: every source compiled with SGE_DEBUG."""
    os.makedirs(BUILD_DEBUG, exist_ok=True)
    srcs = _sources()
    deps = _deps()
    objs = [os.path.join(BUILD_DEBUG, os.path.basename(s)[:-3] + ".o") for s in srcs]
    todo = [(s, o) for s, o in zip(srcs, objs) if force or _stale(o, [s, *deps])]
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            list(ex.map(lambda so: _compile(so[0], False, so[1], ("-DSGE_DEBUG",)), todo))
    if force or todo or _stale(LIB_DEBUG, objs):
        tmp = LIB_DEBUG + f".tmp{os.getpid()}"
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               "-Xcompiler", "-fPIC", *objs, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB_DEBUG)
    return LIB_DEBUG


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
    if "--debug" in sys.argv:
        print(build_debug(force="--force" in sys.argv))
