"""Build libqknorm.so in-tree with nvcc for sm_100a (B200).

Usage: ``python qk_norm_attention_b200/csrc/build_lib.py [--force] [--verbose]``.
This script does not import the package (whose import loads the library).
``--verbose`` passes ``-Xptxas -v`` (registers, spills, shared memory per kernel).
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

CSRC = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(CSRC)
ROOT = os.path.dirname(PKG)
LIBRARY = os.path.join(PKG, "libqknorm.so")
HEADER = os.path.join(ROOT, "include", "qknorm.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _inputs():
    files = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                         if f.endswith((".cuh", ".h"))] + [HEADER, __file__]
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIBRARY):
        return False
    t = os.path.getmtime(LIBRARY)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


DECODE_BENCH = os.path.join(PKG, "decode_bench")
COPY_FLOOR = os.path.join(PKG, "copy_floor")


def _compile_objects(verbose: bool) -> list:
    """Each .cu to its own object, in parallel (in _build/ under the package)."""
    from concurrent.futures import ThreadPoolExecutor
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = [f for f in NVCC_FLAGS if f not in ("-shared", "-cudart", "static")]
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *flags, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        jobs.append((cmd, obj))
    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as ex:
        for r in ex.map(lambda j: subprocess.run(j[0]), jobs):
            if r.returncode != 0:
                raise subprocess.CalledProcessError(r.returncode, r.args)
    return [obj for _, obj in jobs]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ into libqknorm.so (skipped when up to date),
    the C++ decode timing program linked against it, and the copy/read
    yardstick (copy_floor, standalone)."""
    if force or verbose or not up_to_date():
        tmp = LIBRARY + ".tmp"
        objs = _compile_objects(verbose)
        subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                        "-cudart", "static", "-o", tmp, *objs], check=True)
        os.replace(tmp, LIBRARY)
    src = os.path.join(CSRC, "decode_bench.cpp")
    if (force or not os.path.exists(DECODE_BENCH) or
            os.path.getmtime(DECODE_BENCH) < max(os.path.getmtime(src), os.path.getmtime(LIBRARY))):
        tmp = DECODE_BENCH + ".tmp"
        subprocess.run([nvcc(), "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", os.path.join(ROOT, "include"), "-o", tmp, src,
                        "-L", PKG, "-lqknorm", "-Xlinker", "-rpath,$ORIGIN"], check=True)
        os.replace(tmp, DECODE_BENCH)
    src = os.path.join(CSRC, "copy_floor.cpp")
    if force or not os.path.exists(COPY_FLOOR) or os.path.getmtime(COPY_FLOOR) < os.path.getmtime(src):
        tmp = COPY_FLOOR + ".tmp"
        subprocess.run([nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-x", "cu", "-o", tmp, src], check=True)
        os.replace(tmp, COPY_FLOOR)
    return LIBRARY


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose))


if __name__ == "__main__":
    sys.exit(main())
