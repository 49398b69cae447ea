"""Builds the sm_100a shared library in-tree: head_attention_streaming_b200/libattn_sm100.so,
and its debug build libattn_sm100_debug.so (-DATTN_DEBUG: every kernel checks the
global, shared- and tensor-memory indices it computes before using them; see
attn_debug_fault_site in include/attn.h).

    python -m head_attention_streaming_b200.build [--force] [--debug]

nvcc cross-compiles for sm_100a without a GPU. The CUDA runtime is linked
statically, so the library needs only the NVIDIA driver at run time.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(os.path.dirname(PKG_DIR), "include")
SO_PATH = os.path.join(PKG_DIR, "libattn_sm100.so")
DEBUG_SO_PATH = os.path.join(PKG_DIR, "libattn_sm100_debug.so")
SOURCES = [os.path.join(CSRC, "attn_fwd_sm100.cu"), os.path.join(CSRC, "qk_prologue.cu"),
           os.path.join(CSRC, "fp8_pack.cu")]
DEPS = SOURCES + [os.path.join(CSRC, "sm100_ptx.cuh"), os.path.join(CSRC, "tmem_ldst.inc"),
                  os.path.join(INCLUDE, "attn.h")]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(path: str) -> bool:
    if not os.path.exists(path):
        return True
    built = os.path.getmtime(path)
    return any(os.path.getmtime(p) > built for p in DEPS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile the library (or its debug build) if it is missing or older than
    its sources; return its path."""
    path = DEBUG_SO_PATH if debug else SO_PATH
    if not force and not _stale(path):
        return path
    tmp = path + ".tmp"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-std=c++17", "-lineinfo", "-Xptxas", "-v",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-o", tmp, *SOURCES]
    if debug:
        cmd.insert(1, "-DATTN_DEBUG")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
