"""Builds libhils.so (all CUDA sources under csrc/) for sm_100a with nvcc.

Usage: python -m chunk_wise_hierarchical_b200.build [--force]
Each source is compiled to its own object, in parallel; decode_slice.cu is compiled once
per (element type, head dim, group size) slice of the decode kernels.  The objects are
then linked into one shared library, written next to this file so that it travels with
the package.  The stamp beside it hashes the sources by their paths relative to the
package, so a copy of the tree at another path reuses the library.
"""
from __future__ import annotations

import glob
import hashlib
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libhils.so")
STAMP = os.path.join(HERE, ".libhils.stamp")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "--std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
]
SLICED = "decode_slice.cu"
# (element type: 0 fp32 / 1 bf16, head dim, group size) of each decode slice
DECODE_SLICES = [(t, d, g) for t in (1, 0) for d in (64, 128) for g in (1, 2, 4, 8)]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _digest():
    h = hashlib.sha256()
    files = _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "hils.h")]
    for f in files:
        h.update(os.path.relpath(f, os.path.dirname(HERE)).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    h.update(repr(DECODE_SLICES).encode())
    return h.hexdigest()


def nvcc_path():
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the HiLS CUDA library cannot be built")
    return p


def build(force: bool = False, verbose: bool = False) -> str:
    dig = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == dig:
                return LIB
    tmp = LIB + ".tmp"
    with tempfile.TemporaryDirectory(prefix="hils_build_") as objdir:
        jobs = []
        for src in _sources():
            name = os.path.splitext(os.path.basename(src))[0]
            if os.path.basename(src) == SLICED:
                for t, d, g in DECODE_SLICES:
                    defs = [f"-DHILS_DECODE_T={t}", f"-DHILS_DECODE_D={d}", f"-DHILS_DECODE_G={g}"]
                    jobs.append((src, defs, os.path.join(objdir, f"{name}_{t}_{d}_{g}.o")))
            else:
                jobs.append((src, [], os.path.join(objdir, name + ".o")))

        def compile_one(job):
            src, defs, obj = job
            cmd = [nvcc_path(), *NVCC_FLAGS, *defs, "-I", INCLUDE, "-c", "-o", obj, src]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            return subprocess.run(cmd).returncode, src, defs

        # the decode slices (bf16 ones first) are the slowest objects: start them first
        jobs.sort(key=lambda j: os.path.basename(j[0]) != SLICED)
        with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as pool:
            results = list(pool.map(compile_one, jobs))
        failed = [(src, defs) for rc, src, defs in results if rc != 0]
        if failed:
            raise RuntimeError(f"nvcc failed on {failed}")
        link = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                "-o", tmp, *[obj for _, _, obj in jobs]]
        subprocess.run(link, check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(dig)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
