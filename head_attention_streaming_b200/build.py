"""Builds the sm_100a shared library in-tree: head_attention_streaming_b200/libattn_sm100.so.

    python -m head_attention_streaming_b200.build [--force]

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


def _stale() -> bool:
    if not os.path.exists(SO_PATH):
        return True
    built = os.path.getmtime(SO_PATH)
    return any(os.path.getmtime(p) > built for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources; return its path."""
    if not force and not _stale():
        return SO_PATH
    tmp = SO_PATH + ".tmp"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-std=c++17", "-lineinfo", "-Xptxas", "-v",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-o", tmp, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, SO_PATH)
    return SO_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
