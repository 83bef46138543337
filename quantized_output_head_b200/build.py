"""Build libarchead.so (the forward pass) and libarchead_build.so (the GPU
construction of a packed head) in-tree with nvcc for sm_100a.

    python quantized_output_head_b200/build.py [--force] [--verbose]

Objects go to quantized_output_head_b200/_build/, the shared libraries next to
this file.  The CUDA runtime is linked statically, so libarchead.so needs only
the driver at run time; libarchead_build.so also needs cuBLAS and cuSOLVER,
found through an rpath to the CUDA wheels PyTorch loads (the same copies it
uses) and then the toolkit's lib64.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libarchead.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")
SOURCES = ["pack.cu", "api.cu", "decode.cu", "prologue.cu", "static_ws.cu", "actprep.cu", "tcgemm.cu"]
BUILDER_SOURCES = ["builder.cu"]
BUILDER_LIB = os.path.join(PKG, "libarchead_build.so")
FORWARD_HEADERS = ["archead.h"]
BUILDER_HEADERS = ["archead.h", "archead_build.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-Xptxas", "-v",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libarchead.so")
    return exe


def _deps(sources, headers):
    if sources is SOURCES:   # the forward library: every kernel source and shared header
        files = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f not in BUILDER_SOURCES]
    else:
        files = [os.path.join(CSRC, f) for f in sources]
    files += [os.path.join(INCLUDE, h) for h in headers]
    return files


def _cuda_library_dirs():
    """Directories holding libcublas / libcusolver (and what they load): the
    nvidia wheels next to PyTorch first, then the toolkit."""
    import importlib.util
    dirs = []
    for mod in ("nvidia.cublas", "nvidia.cusolver", "nvidia.cusparse", "nvidia.nvjitlink"):
        try:
            spec = importlib.util.find_spec(mod)
        except ImportError:
            spec = None
        if spec is not None and spec.submodule_search_locations:
            d = os.path.join(list(spec.submodule_search_locations)[0], "lib")
            if os.path.isdir(d):
                dirs.append(d)
    dirs.append(os.path.join(os.path.dirname(os.path.dirname(nvcc())), "lib64"))
    return dirs


def _build_one(lib, sources, headers, link_extra, force, verbose):
    newest = max(os.path.getmtime(f) for f in _deps(sources, headers))
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest:
        return lib
    objs = []
    for src in sources:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or r.returncode != 0:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}")
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, *link_extra, "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
        raise RuntimeError(f"link of {os.path.basename(lib)} failed")
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Build both libraries (each only when a source is newer); returns the
    forward library's path."""
    os.makedirs(BUILD, exist_ok=True)
    _build_one(LIB, SOURCES, FORWARD_HEADERS, [], force, verbose)
    dirs = _cuda_library_dirs()
    link = [f"-L{d}" for d in dirs] + ["-l:libcublas.so.12", "-l:libcusolver.so.11",
                                       "-Xlinker", "-rpath," + ":".join(dirs),
                                       "-Xlinker", "-rpath-link," + ":".join(dirs)]
    _build_one(BUILDER_LIB, BUILDER_SOURCES, BUILDER_HEADERS, link, force, verbose)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
