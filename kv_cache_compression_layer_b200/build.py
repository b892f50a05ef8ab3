"""Builds libkvcomp.so in-tree from csrc/*.cu for sm_100a (nvcc, no GPU needed).

    python -m kv_cache_compression_layer_b200.build [--force] [--verbose-ptxas] [--debug]

--debug builds libkvcomp_debug.so instead: the same sources with
-DKV_DEBUG_CHECKS, whose kernels check their data-dependent indices and
report a failed check in the library's check word (kv_debug_check_word).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkvcomp.so")
DEBUG_LIB = os.path.join(HERE, "libkvcomp_debug.so")
BUILD_DIR = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(os.path.dirname(HERE), "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(os.path.dirname(HERE), "include", "*.h")))


def build(force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    """Compile every kernel file and link libkvcomp.so (debug: libkvcomp_debug.so); returns its path."""
    build_dir = os.path.join(BUILD_DIR, "debug") if debug else BUILD_DIR
    lib_path = DEBUG_LIB if debug else LIB
    flags = FLAGS + (["-DKV_DEBUG_CHECKS"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = _sources()
    newest_hdr = max([os.path.getmtime(h) for h in _headers()] + [0])
    jobs = []
    objs = []
    for src in srcs:
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), newest_hdr):
            cmd = [NVCC, *ARCH, *flags, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = []
    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for cmd, r in ex.map(run, jobs):
            if r.returncode != 0 or ptxas_verbose:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                failed.append(cmd[-3])
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    if force or jobs or not os.path.exists(lib_path):
        tmp = lib_path + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs])
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv, debug="--debug" in sys.argv))
