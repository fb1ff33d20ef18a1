"""Build libssd.so in-tree with nvcc for sm_100a.

    python mamba_ssd_chunked_03_b200/build.py [--force] [--verbose]

Each csrc/*.cu is compiled to an object under _build/ (rebuilt when it or a
header is newer than the object) and linked into
mamba_ssd_chunked_03_b200/libssd.so.  The CUDA runtime is linked statically so
the library does not depend on which libcudart the host process loaded.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libssd.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_time = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    build_py_time = os.path.getmtime(os.path.abspath(__file__))
    objs = []
    flags = NVCC_FLAGS + list(extra_flags or [])
    for src in srcs:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_time, build_py_time)):
            continue
        cmd = [nvcc(), *ARCH, *flags, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    newest = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < newest:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


PROBE_SRC = os.path.join(ROOT, "tests", "cuda", "tc_probe.cu")
PROBE_LIB = os.path.join(ROOT, "tests", "cuda", "libtcprobe.so")


def build_probe(force: bool = False, verbose: bool = False) -> str:
    """Test-only library probing the tcgen05 building blocks (tests/cuda)."""
    deps = [PROBE_SRC, os.path.join(CSRC, "sm100.cuh"), os.path.abspath(__file__)]
    if (not force and os.path.exists(PROBE_LIB)
            and os.path.getmtime(PROBE_LIB) >= max(os.path.getmtime(d) for d in deps)):
        return PROBE_LIB
    tmp = PROBE_LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-I", CSRC, "-shared", "-o", tmp, PROBE_SRC, "-cudart", "static"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, PROBE_LIB)
    return PROBE_LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))
    print(build_probe(force=args.force, verbose=args.verbose))
    sys.exit(0)
