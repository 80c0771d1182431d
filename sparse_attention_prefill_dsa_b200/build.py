"""Builds libdsa.so (the C-ABI library) in-tree with nvcc for sm_100a, and its
checking variant libdsa_check.so (the same sources with -DDSA_CHECK=1: every
dynamically indexed buffer access is bounds-checked and a bad index is
reported in the workspace status instead of being made).

Usage: python -m sparse_attention_prefill_dsa_b200.build [--verbose] [--check]
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(PKG, "libdsa.so")
BUILD = os.path.join(PKG, "_build")
VARIANTS = {  # name -> (library, object folder, extra nvcc flags)
    "release": (OUT, BUILD, []),
    "check": (os.path.join(PKG, "libdsa_check.so"), os.path.join(PKG, "_build_check"),
              ["-DDSA_CHECK=1"]),
}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps() -> list[str]:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    return files + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]


def build(force: bool = False, verbose: bool = False, variant: str = "release") -> str:
    out, build_dir, vflags = VARIANTS[variant]
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(p) for p in _deps())
        if os.path.getmtime(out) >= newest:
            return out
    nvcc = _nvcc()
    os.makedirs(build_dir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if verbose else []) + vflags

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
        return obj, r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        results = list(ex.map(compile_one, sources()))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    tmp = out + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *[o for o, _ in results]]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv,
                variant="check" if "--check" in sys.argv else "release"))
