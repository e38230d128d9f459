"""Build libgqa_attn.so (sm_100a only) in-tree with nvcc.

    python -m gqa_flash_attention_attn_b200.build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgqa_attn.so")
SOURCES = ["abi.cu", "prefill_sm100.cu", "decode_sm100.cu", "merge.cu", "decode_noalloc.cu"]
HEADERS = ["ptx.cuh", "kernels.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "attn.h"))
    return files


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(verbose: bool = False, force: bool = False) -> str:
    """Compile each source to an object in _build/ (in parallel), then link
    the shared library."""
    if not force and not stale():
        return LIB
    obj_dir = os.path.join(ROOT, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    flags = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
             "-I", os.path.join(ROOT, "include")]
    if verbose:
        flags += ["-Xptxas", "-v"]
    objs = [os.path.join(obj_dir, os.path.splitext(s)[0] + ".o") for s in SOURCES]
    with ThreadPoolExecutor(max_workers=max(1, min(len(SOURCES), os.cpu_count() or 1))) as ex:
        jobs = [ex.submit(subprocess.run, flags + ["-c", os.path.join(CSRC, s), "-o", o], check=True)
                for s, o in zip(SOURCES, objs)]
        for j in jobs:
            j.result()
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", LIB, *objs], check=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
