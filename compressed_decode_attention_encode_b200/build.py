"""Builds the in-tree C-ABI library ``libtq.so`` for sm_100a with nvcc.

``python -m compressed_decode_attention_encode_b200.build`` (or
``__graft_entry__.build()``) compiles every CUDA source under ``csrc/`` into
one shared library next to this file.  It rebuilds only when a source or
header is newer than the library.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtq.so")
SOURCES = ["tq_host.cu", "tq_encode.cu", "tq_decode.cu", "tq_gate.cu", "tq_tcache.cu", "tq_search.cu",
           "tq_promote.cu", "tq_attend_64_64.cu", "tq_attend_64_128.cu", "tq_attend_128_64.cu", "tq_attend_128_128.cu"]
HEADERS = ["tq_internal.cuh", "tq_encode_core.cuh", "tq_attend.cuh", os.path.join("..", "..", "include", "tq.h")]

NVCC_FLAGS = [
    "-O3", "-lineinfo", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile each source to an object (in parallel, under _build/ at the
    repository root), then link them into libtq.so."""
    if not force and not _stale():
        return LIB
    from concurrent.futures import ThreadPoolExecutor

    obj_dir = os.path.join(ROOT, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    jobs = []
    for src in SOURCES:
        obj = os.path.join(obj_dir, os.path.splitext(src)[0] + ".o")
        jobs.append((obj, [nvcc_path(), *compile_flags, "-I", os.path.join(ROOT, "include"),
                           "-c", "-o", obj, os.path.join(CSRC, src)]))

    def run(job):
        if verbose:
            print(" ".join(job[1]), file=sys.stderr)
        subprocess.run(job[1], check=True)

    with ThreadPoolExecutor(max_workers=len(jobs)) as pool:
        list(pool.map(run, jobs))
    tmp = LIB + ".tmp"
    link = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
            "-Xcompiler", "-fPIC", "-o", tmp, *[o for o, _ in jobs]]
    if verbose:
        print(" ".join(link), file=sys.stderr)
    subprocess.run(link, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
