"""Build the in-tree CUDA library ``libtq.so`` for sm_100a with nvcc.

Usage: ``python kv_cache_vector_04_b200/build.py [--force] [--verbose]`` (run it by path:
importing the package itself needs the library).
The shared library is written next to this file so that it travels with the
source tree; nothing is installed into site-packages.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libtq.so")
SOURCES = ["api.cu", "quantize.cu", "attend.cu", "attend_d64.cu", "attend_d128.cu",
           "attend_d256.cu", "noalloc.cu", "tables.cpp"]
HEADERS = ["device_common.cuh", "kernels.h", "tables.h", "attend_impl.cuh", "attend_cc.cuh",
           "quantize_fast.cuh"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the TurboQuant CUDA library cannot be built")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "tq.h"))
    files.append(os.path.abspath(__file__))
    return files


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object (in parallel: the kernel templates are
    instantiated for every format), then link libtq.so."""
    if not force and not is_stale():
        return LIB
    import concurrent.futures
    import tempfile
    nvcc = nvcc_path()
    flags = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-ffp-contract=off",
             "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-I", INCLUDE, "-I", CSRC]
    if verbose:
        flags += ["-Xptxas", "-v"]
    with tempfile.TemporaryDirectory(prefix="tq_build_") as tmpdir:
        def compile_one(src):
            obj = os.path.join(tmpdir, src + ".o")
            r = subprocess.run([nvcc] + flags + ["-c", os.path.join(CSRC, src), "-o", obj],
                               stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
            return src, obj, r.returncode, r.stdout
        workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
            results = list(ex.map(compile_one, SOURCES))
        failed = [r for r in results if r[2] != 0]
        for src, _, rc, out in results:
            if out and (verbose or rc != 0):
                sys.stdout.write(out)
        if failed:
            raise subprocess.CalledProcessError(failed[0][2], "nvcc -c " + failed[0][0])
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.run([nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp]
                       + [r[1] for r in results] + ["-lcudart"], check=True)
        os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose))
    return 0


if __name__ == "__main__":
    sys.exit(main())
