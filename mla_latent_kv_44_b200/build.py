"""Build libmla.so in-tree with nvcc for sm_100a.

    python -m mla_latent_kv_44_b200.build [--force] [--verbose]

Each csrc/*.cu compiles to an object under _build/ (recompiled when it or a header is newer),
then the objects link into mla_latent_kv_44_b200/libmla.so with the CUDA runtime linked
statically, so the library loads on a machine without a GPU (calls then fail with
MLA_ERR_CUDA) and needs nothing at run time but the NVIDIA driver. A second library,
libmla_testhook.so, differs only in a test define of the attention kernel (one K-slab load of
the first work range is left out); only the tests load it.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmla.so")
# Test build: the same library with one K-slab load of the first work range left out
# (MLA_TEST_DROP_ARRIVE), so that the tests can watch a bounded wait run out.
TEST_LIB = os.path.join(PKG, "libmla_testhook.so")
TEST_DEFINE = "-DMLA_TEST_DROP_ARRIVE"
TEST_SOURCES = ("decode_tc.cu",)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
            glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    jobs = []
    objs = []
    test_objs = []
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or ptxas_info or _stale(obj, [src] + headers):
            cmd = [cc, *ARCH, *FLAGS, "-c", src, "-o", obj]
            if ptxas_info:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append(cmd)
        if os.path.basename(src) in TEST_SOURCES:
            tobj = os.path.join(BUILD, os.path.basename(src) + ".testhook.o")
            test_objs.append(tobj)
            if force or _stale(tobj, [src] + headers):
                jobs.append([cc, *ARCH, *FLAGS, TEST_DEFINE, "-c", src, "-o", tobj])
        else:
            test_objs.append(obj)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        p = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, p

    failed = []
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for cmd, p in ex.map(run, jobs):
            if p.returncode != 0 or ptxas_info or verbose:
                sys.stderr.write(p.stdout + p.stderr)
            if p.returncode != 0:
                failed.append(cmd[-3])
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    for lib, parts in ((LIB, objs), (TEST_LIB, test_objs)):
        if force or jobs or _stale(lib, parts):
            cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", lib, *parts]
            if verbose:
                print(" ".join(cmd), flush=True)
            p = subprocess.run(cmd, capture_output=True, text=True)
            if p.returncode != 0:
                raise RuntimeError("link failed:\n" + p.stdout + p.stderr)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills/smem")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    main()
