"""Build ``libgdn_b200.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m linear_attention_recurrent_chunked_b200.build [--force] [--verbose] [--debug]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel),
then linked into ``linear_attention_recurrent_chunked_b200/libgdn_b200.so``.
Objects are rebuilt when their source or any ``csrc`` header / ``include/gdn.h``
is newer. ``--ptxas-v`` prints register / spill / shared-memory usage.
``--debug`` builds the index-checking variant instead: the same sources with
``-DGDN_DEBUG_CHECKS`` (objects under ``_build/debug/``) into
``libgdn_b200_debug.so``, whose kernels check their indices into the
workspace and the outputs and report a failed check as GDN_ERR_BOUNDS
(the binding loads it when the environment sets GDN_DEBUG_CHECKS=1).
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libgdn_b200.so")
LIB_DEBUG = os.path.join(PKG, "libgdn_b200_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    hdrs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "gdn.h")]
    return max(os.path.getmtime(h) for h in hdrs)


def _compile(src: str, obj: str, extra) -> str:
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), r.stderr))
    return r.stderr


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False, debug: bool = False) -> str:
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib_path = LIB_DEBUG if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    dep_t = _deps_mtime()
    extra = (["-Xptxas", "-v"] if ptxas_v else []) + (["-DGDN_DEBUG_CHECKS"] if debug else [])
    jobs = {}
    objs = []
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for s in srcs:
            o = os.path.join(bdir, os.path.basename(s)[:-3] + ".o")
            objs.append(o)
            stale = force or ptxas_v or not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), dep_t)
            if stale:
                jobs[ex.submit(_compile, s, o, extra)] = s
        for f in cf.as_completed(jobs):
            log = f.result()
            if (verbose or ptxas_v) and log:
                print("==", os.path.basename(jobs[f]), "\n" + log, file=sys.stderr)
    if jobs or force or not os.path.exists(lib_path) or os.path.getmtime(lib_path) < max(os.path.getmtime(o) for o in objs):
        tmp = lib_path + ".tmp%d" % os.getpid()
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (" ".join(cmd), r.stderr))
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, ptxas_v="--ptxas-v" in sys.argv,
                debug="--debug" in sys.argv))
