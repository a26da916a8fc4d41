"""Builds the CUDA library libnvfp4pw.so in-tree for sm_100a (B200) with nvcc,
and beside it libnvfp4pw_debug.so: the same sources with NVFP4_DEBUG defined
(the kernels check their tile and index arithmetic and report
NVFP4_ERR_BOUNDS instead of making an access that left its array).

Usage: python -m nvfp4_post_weight_b200.build [--verbose-ptxas]
Objects go to _build/ (and _build/debug/) at the repository root; the shared
libraries are written next to this file so that the Python binding finds
them."""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libnvfp4pw.so")
LIB_DEBUG = os.path.join(PKG, "libnvfp4pw_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src, verbose, debug=False):
    obj = os.path.join(BUILD, "debug" if debug else "", os.path.basename(src)[:-3] + ".o")
    deps = [src] + [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith(".cuh")]
    deps.append(os.path.join(INCLUDE, "nvfp4pw.h"))
    if os.path.exists(obj) and not verbose:
        if os.path.getmtime(obj) >= max(os.path.getmtime(d) for d in deps):
            return obj, ""
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DNVFP4_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def _link(lib, objs):
    newest = max(os.path.getmtime(o) for o in objs)
    if not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", lib, *objs, "-lcuda"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")


def build(verbose=False, debug=True):
    """Compiles and links the release library (and, with debug, the debug
    one); returns the release library's path."""
    os.makedirs(os.path.join(BUILD, "debug"), exist_ok=True)
    srcs = sources()
    jobs = [(src, False) for src in srcs] + ([(src, True) for src in srcs] if debug else [])
    with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
        results = list(ex.map(lambda j: _compile(j[0], verbose and not j[1], j[1]), jobs))
    rel = [o for (o, _), (_, d) in zip(results, jobs) if not d]
    dbg = [o for (o, _), (_, d) in zip(results, jobs) if d]
    if verbose:
        for (o, log), (_, d) in zip(results, jobs):
            if not d:
                sys.stdout.write(f"== {os.path.basename(o)}\n{log}")
    _link(LIB, rel)
    if debug:
        _link(LIB_DEBUG, dbg)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose-ptxas" in sys.argv))
