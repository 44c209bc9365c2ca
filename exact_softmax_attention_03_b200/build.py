"""Compile the CUDA library ``libattn.so`` in-tree for sm_100a.

Usage: ``python -m exact_softmax_attention_03_b200.build [--verbose] [--debug]``
(``--debug``: the bounds-checking debug build, ``libattn_debug.so``).
The shared object is written next to this file, so it travels with the
source tree; nothing is installed elsewhere.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "attn_api.cu")
DEPS = [os.path.join(HERE, "csrc", f) for f in
        ("attn_api.cu", "sm100_ptx.cuh", "decode_kernels.cuh", "prefill_kernel.cuh",
         "backward_kernels.cuh", "merge_kernel.cuh")] + \
       [os.path.join(ROOT, "include", "attn.h")]
LIB = os.path.join(HERE, "libattn.so")
# the bounds-checking debug build (never the default): every kernel checks its
# computed global indices and its roles' stage counts (include/attn.h,
# attn_debug_checks)
LIB_DEBUG = os.path.join(HERE, "libattn_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in DEPS if os.path.exists(f))


def build(force: bool = False, verbose: bool = False, debug: bool | None = None) -> str:
    """Compile the release library, or the bounds-checking debug build with
    ``debug=True`` (default: the variant ATTN_LIBRARY selects)."""
    if debug is None:
        debug = os.environ.get("ATTN_LIBRARY", "release") == "debug"
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    # a private temporary name: ranks of one job that build at once each write
    # their own file, and the atomic rename leaves one complete library
    tmp = f"{lib}.{os.getpid()}.tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", tmp, SRC]
    if debug:
        cmd += ["-DATTN_DEBUG_BOUNDS=1"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        if os.path.exists(tmp):
            os.remove(tmp)
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
