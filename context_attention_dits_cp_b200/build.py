"""Builds libcpattn.so in-tree for sm_100a with nvcc.

    python -m context_attention_dits_cp_b200.build [--force]

Each .cu file under csrc/ is compiled to an object in _build/ (in parallel)
and the objects are linked into context_attention_dits_cp_b200/libcpattn.so;
the same sources compiled with -DCP_DEBUG (device-side bounds checks) give
libcpattn_debug.so.
The CUDA runtime is linked statically; the driver is reached through
cudaGetDriverEntryPoint, so nothing links against libcuda directly.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libcpattn.so")
DEBUG_LIB = os.path.join(PKG, "libcpattn_debug.so")   # CP_DEBUG: device-side bounds checks

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    return sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                        if f.endswith((".cuh", ".h"))] + [os.path.join(INCLUDE, "cpattn.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def _compile(src: str, extra, tag: str = "") -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + tag + ".o")
    cmd = [nvcc()] + ARCH + FLAGS + list(extra) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def _build_one(lib: str, extra, tag: str, verbose: bool) -> str:
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, tag), sources()))
    tmp = lib + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    if verbose:
        print(f"built {lib}")
    return lib


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = True) -> str:
    """Builds libcpattn.so and, with debug=True, the bounds-checking
    libcpattn_debug.so (same sources compiled with -DCP_DEBUG)."""
    if force or not up_to_date(LIB):
        _build_one(LIB, extra, "", verbose)
    if debug and (force or not up_to_date(DEBUG_LIB)):
        _build_one(DEBUG_LIB, list(extra) + ["-DCP_DEBUG"], ".debug", verbose)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    build(force=a.force or a.ptxas_verbose, verbose=True,
          extra=["-Xptxas", "-v"] if a.ptxas_verbose else ())
    sys.exit(0)
