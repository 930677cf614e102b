"""Builds libattn_b200.so (all CUDA sources, sm_100a) next to this file.

Usage: python -m attention_causal_gqa_b200.build [--verbose]
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libattn_b200.so")
SOURCES = ["api.cu", "rope.cu", "prefill.cu", "decode.cu", "decode_fp8.cu", "mla.cu", "merge.cu", "chunk.cu", "dsa.cu", "dsa_fp8.cu", "noalloc.cu"]
HEADERS = ["sm100.cuh", "kernels.h"]  # shared by every kernel
PROLOGUE_HEADERS = ["prologue.h", "dsa.h", "dsa_fp8.h"]  # included by their own kernels only (not in every fingerprint)
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _fingerprint() -> str:
    h = hashlib.sha256()
    for name in SOURCES + HEADERS + PROLOGUE_HEADERS:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(INCLUDE, "attn_b200.h"), "rb") as f:
        h.update(f.read())
    h.update(" ".join(ARCH).encode())
    return h.hexdigest()


# The file that defines each main kernel; with the shared headers and the arch
# flags it fixes that kernel's code (profile figures are keyed by this).
KERNEL_SOURCES = {"prefill_kernel": "prefill.cu", "decode_kernel": "decode.cu", "decode_fp8_kernel": "decode_fp8.cu",
                  "mla_kernel": "mla.cu", "dsa_index_kernel": ("dsa.cu", "dsa.h")}


def kernel_fingerprint(kernel: str) -> str:
    h = hashlib.sha256()
    srcs = KERNEL_SOURCES[kernel]
    for name in ([srcs] if isinstance(srcs, str) else list(srcs)) + HEADERS:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    h.update(" ".join(ARCH).encode())
    return h.hexdigest()[:16]


def build(verbose: bool = False, force: bool = False) -> str:
    stamp = LIB + ".sha256"
    fp = _fingerprint()
    if not force and os.path.exists(LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == fp:
                return LIB
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-o", LIB + ".tmp"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    with open(stamp, "w") as f:
        f.write(fp)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
