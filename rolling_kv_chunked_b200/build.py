"""Build librkv.so (and the test-input generator libsynth.so) in-tree for sm_100a.

    python rolling_kv_chunked_b200/build.py [--force] [--ptxas-info]

nvcc cross-compiles without a GPU. The CUDA runtime is linked statically so
the library does not depend on which libcudart the host process loaded first.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]

LIB = os.path.join(HERE, "librkv.so")
SYNTH_LIB = os.path.join(ROOT, "synth", "libsynth.so")

CU_SOURCES = ["rkv_kernels.cu", "rkv_attention.cu", "rkv_noalloc.cu"]
CPP_SOURCES = ["rkv_host.cpp"]
HEADERS = ["ptx_sm100.cuh", "numeric.cuh", "rkv_internal.h"]


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"build step failed: {' '.join(cmd)}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    return res.stdout + res.stderr


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile every CUDA / C++ source and link the shared libraries; returns the librkv path."""
    if not os.path.exists(NVCC) and shutil.which("nvcc") is None:
        raise RuntimeError("nvcc not found; set CUDA_HOME")
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "rkv.h")]
    objs = []
    log = ""
    for src in CU_SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if force or ptxas_info or _stale(obj, [path] + headers):
            cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                   "-I", INCLUDE, "-c", path, "-o", obj]
            if ptxas_info:
                cmd.insert(1, "-Xptxas=-v")
            log += _run(cmd, verbose)
    for src in CPP_SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if force or _stale(obj, [path] + headers):
            cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-fvisibility=hidden", "-Wall",
                   "-I", os.path.join(CUDA_HOME, "include"), "-I", INCLUDE, "-c", path, "-o", obj]
            log += _run(cmd, verbose)
    if force or _stale(LIB, objs):
        log += _run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs], verbose)
    synth_src = os.path.join(ROOT, "synth", "synth.cu")
    if force or _stale(SYNTH_LIB, [synth_src]):
        log += _run([nvcc, *ARCH, "-O3", "-std=c++17", "-shared", "-cudart", "static", "-Xcompiler", "-fPIC",
                     "-o", SYNTH_LIB, synth_src], verbose)
    if ptxas_info:
        print(log)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print register / spill / smem usage")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    main()
