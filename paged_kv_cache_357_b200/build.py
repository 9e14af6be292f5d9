"""Build libpa.so in-tree for B200 (sm_100a) with nvcc.

    python -m paged_kv_cache_357_b200.build [--force] [--verbose]

Each CUDA source compiles to an object under ``_build/`` (in parallel), then
the objects link into ``paged_kv_cache_357_b200/libpa.so`` with the CUDA
runtime linked statically, so the library only needs the driver at run time.
Nothing is JIT-compiled; the built file travels with the source tree.
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
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(HERE, "libpa.so")
SOURCES = [
    "pa_decode.cu",
    "pa_decode_tc.cu",
    "pa_decode_tc_blocks.cu",
    "pa_attn_tc_multi.cu",
    "pa_attn_tc_multi_b8.cu",
    "pa_attn_tc_multi_b32.cu", "pa_attn_tc_prefill.cu", "pa_attn_tc_prefill_b8.cu", "pa_attn_tc_prefill_b32.cu",
    "pa_attn_tc_group.cu", "pa_attn_tc_group_b8.cu", "pa_attn_tc_group_b32.cu",
    "pa_kv_ops.cu",
    "pa_merge.cu",
    "pa_block_manager.cpp",
    "pa_step.cpp",
]
HEADERS = ["pa_device.cuh", "pa_internal.h", "pa_decode_common.cuh", "pa_decode_host.h", "pa_attn_tc.cuh",
           "pa_attn_tc_group.cuh", "pa_attn_tc_prefill.cuh"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON_FLAGS = ARCH_FLAGS + [
    "-O3",
    "-lineinfo",
    "-std=c++17",
    "-Xcompiler",
    "-fPIC,-fvisibility=hidden",
    "-I" + os.path.join(ROOT, "include"),
]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; libpa needs the CUDA toolkit to build")
    return cand


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "pa.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    """Compile libpa.so if any input is newer than it; return its path."""
    if not force and up_to_date():
        return LIB_PATH
    nvcc = nvcc_path()
    os.makedirs(BUILD_DIR, exist_ok=True)
    flags = COMMON_FLAGS + list(extra_flags or [])
    procs = []
    objs = []
    for src in SOURCES:
        obj = os.path.join(BUILD_DIR, os.path.splitext(src)[0] + ".o")
        objs.append(obj)
        cmd = [nvcc, *flags, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for cmd, p in procs:
        out, _ = p.communicate()
        if verbose and out:
            print(out, flush=True)
        if p.returncode != 0:
            failed.append((cmd, out))
    if failed:
        msg = "\n".join(f"$ {' '.join(c)}\n{o}" for c, o in failed)
        raise RuntimeError(f"nvcc failed:\n{msg}")
    tmp = LIB_PATH + ".tmp"
    link = [nvcc, *ARCH_FLAGS, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(link), flush=True)
    r = subprocess.run(link, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true", help="print registers/spills/smem per kernel")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_verbose else []
    path = build(force=a.force or a.ptxas_verbose, verbose=a.verbose or a.ptxas_verbose, extra_flags=extra)
    print(path)
    return 0


if __name__ == "__main__":
    sys.exit(main())
