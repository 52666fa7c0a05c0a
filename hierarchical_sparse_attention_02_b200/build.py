"""Builds libzha.so (CUDA sm_100a) in-tree with nvcc.

Usage: python -m hierarchical_sparse_attention_02_b200.build [-v]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libzha.so")
SOURCES = ["zha_api.cu", "zha_tree.cu", "zha_route.cu", "zha_attn.cu", "zha_attn_tc.cu", "zha_prefill_tc.cu", "zha_noalloc.cu"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "zha.h")]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(out: str = LIB, verbose: bool = False, force: bool = False) -> str:
    if not force and not needs_build(out):
        return out
    cmd = [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-Xptxas", "-v" if verbose else "-O3", "-o", out + ".tmp"] + sources()
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
