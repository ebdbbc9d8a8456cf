"""Build the CUDA library in-tree: every csrc/*.cu for sm_100a -> libcsa_attn.so.

    python causal_softmax_attention_b200/build.py [-v] [--debug]   # or __graft_entry__.build()

The shared library lands next to this file so that it travels with the
source tree; object files go to _build/ (git-ignored). `--debug` builds the
same sources with ATTN_DEBUG (device-side bounds checks that report
ATTN_ERR_BOUNDS instead of trapping, outputs filled with NaN before each
call) into libcsa_attn_debug.so, objects in _build_debug/; the package loads
it instead of the release library when CSA_ATTN_DEBUG=1.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB_NAME = "libcsa_attn.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
DEBUG_BUILD = os.path.join(HERE, "_build_debug")
DEBUG_LIB_PATH = os.path.join(HERE, "libcsa_attn_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
    "--expt-relaxed-constexpr", "-diag-suppress", "177",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build the library")
    return path


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _needs_rebuild(obj: str, deps) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    """Compile (incrementally) and link the library (the ATTN_DEBUG variant
    with debug=True); returns its path."""
    build_dir = DEBUG_BUILD if debug else BUILD
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    extra = ["-DATTN_DEBUG"] if debug else []
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(ROOT, "include", "attn.h"))
    objs, jobs = [], []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if _needs_rebuild(obj, [src] + headers) or ptxas_verbose:
            cmd = [nvcc()] + NVCC_FLAGS + extra + (["-Xptxas", "-v"] if ptxas_verbose else []) + [
                "-c", src, "-o", obj]
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        return r.stdout + r.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 4))) as ex:
        for out in ex.map(run, jobs):
            if verbose or ptxas_verbose:
                sys.stdout.write(out)
    if jobs or not os.path.exists(lib_path) or _needs_rebuild(lib_path, objs):
        tmp = lib_path + ".tmp"
        run([nvcc()] + ARCH + ["-shared", "-o", tmp] + objs)
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(verbose=True, ptxas_verbose="-v" in sys.argv, debug="--debug" in sys.argv))
