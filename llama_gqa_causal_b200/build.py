"""Build libllama_attn.so in-tree with nvcc for sm_100a.

    python -m llama_gqa_causal_b200.build [--force] [--verbose-ptxas]

One translation unit (csrc/llama_attn.cu) holds every kernel and the C ABI;
the CUDA runtime is linked statically and the driver entry point for TMA
descriptors is looked up at run time, so the library loads on machines
without a GPU driver (its compute calls then fail with LLAMA_ERR_CUDA).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libllama_attn.so")
# Written beside the library by build(): the source hash it was compiled from.
HASH_FILE = LIB + ".srchash"
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def source_hash() -> str:
    """sha256 over every CUDA source and public header (names and contents)."""
    h = hashlib.sha256()
    for s in sources():
        h.update(os.path.relpath(s, ROOT).encode())
        with open(s, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def built_hash() -> str | None:
    """Source hash recorded when the in-tree library was built (None if unknown)."""
    try:
        with open(HASH_FILE) as f:
            return f.read().strip()
    except OSError:
        return None


def needs_build() -> bool:
    return not os.path.exists(LIB) or built_hash() != source_hash()


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not needs_build() and not verbose_ptxas:
        return LIB
    cmd = [NVCC, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", LIB,
           os.path.join(CSRC, "llama_attn.cu")]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    digest = source_hash()
    if os.path.exists(HASH_FILE):
        os.remove(HASH_FILE)
    subprocess.check_call(cmd)
    with open(HASH_FILE, "w") as f:
        f.write(digest + "\n")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
    sys.exit(0)
