"""Build libmq.so (all CUDA sources, sm_100a) in-tree with nvcc.

Objects are rebuilt only when their source or a header is newer; the
translation units compile in parallel.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden,-ffp-contract=off",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _headers_mtime() -> float:
    # this script too: a change of its flags rebuilds every object
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return max([os.path.getmtime(h) for h in hs] + [os.path.getmtime(os.path.abspath(__file__))])


def _compile(src: str, hdr_mtime: float, verbose: bool, obj_dir: str = OBJ, extra=()) -> str:
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_mtime):
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(obj + ".tmp", obj)
    return obj


def _build_lib(lib: str, obj_dir: str, extra: list, verbose: bool) -> str:
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hm = _headers_mtime()
    with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        objs = list(ex.map(lambda s: _compile(s, hm, verbose, obj_dir, extra), srcs))
    if not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        tmp = lib + ".tmp%d" % os.getpid()
        subprocess.check_call([NVCC, *ARCH, "-shared", "--cudart", "static", "-Xlinker",
                               "--exclude-libs,ALL", "-o", tmp, *objs])
        os.replace(tmp, lib)
    return lib


def build(verbose: bool = False) -> str:
    return _build_lib(LIB, OBJ, [], verbose)


# Test-hook build (tests only, never loaded by the package): every bounded
# wait gives up after 5 ms instead of about a second, and
# mq_test_drop_x_arrivals() makes a GEMM CTA drop one arrival, so a test can
# run the timeout path on a GPU without a fault or a trap.
HOOKS_LIB = os.path.join(HERE, "libmq_testhooks.so")
HOOKS_OBJ = os.path.join(HERE, "_build_hooks")


def build_test_hooks(verbose: bool = False) -> str:
    return _build_lib(HOOKS_LIB, HOOKS_OBJ, ["-DMQ_TEST_HOOKS", "-DMQ_WAIT_NS=5000000ull"], verbose)


if __name__ == "__main__":
    print(build(verbose=os.environ.get("MQ_VERBOSE") == "1"))
    print(build_test_hooks())
