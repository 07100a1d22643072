"""Builds liblwc.so in-tree with nvcc for sm_100a (no GPU needed to build).

    python -m decode_dfloat11_b200.build [--force] [--ptxas-info]
"""
from __future__ import annotations

import argparse
import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "liblwc.so")

CUDA_SOURCES = ["lwc_df11.cu", "lwc_codebook.cu", "lwc_encode.cu", "lwc_gemm.cu"]
CXX_SOURCES = ["lwc_host.cpp"]
HEADERS = ["lwc_internal.h", "lwc_device.cuh", "lwc_df11_dev.cuh", "lwc_umma.cuh", "lwc_cb_dev.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: liblwc cannot be built")
    return path


def _inputs():
    files = [os.path.join(CSRC, f) for f in CUDA_SOURCES + CXX_SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "lwc.h"))
    files.append(os.path.abspath(__file__))
    return files


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False) -> str:
    """Compile every source of the library and link liblwc.so; returns its path."""
    if not force and not ptxas_info and not stale():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    common = ["-O3", "-std=c++17", "-I", INCLUDE, "-I", CSRC]
    jobs = []   # (source, object, command, tool), compiled in parallel
    for src in CUDA_SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, "-lineinfo", *common, "-Xcompiler", "-fPIC,-fvisibility=hidden",
               "--expt-relaxed-constexpr", "-c", os.path.join(CSRC, src), "-o", obj]
        if ptxas_info:
            cmd.insert(1, "-Xptxas=-v")
        jobs.append((src, obj, cmd, "nvcc"))
    for src in CXX_SOURCES:
        obj = os.path.join(BUILD, src.replace(".cpp", ".o"))
        cmd = ["g++", "-O2", "-fPIC", "-fvisibility=hidden", "-Wall", *common, "-c",
               os.path.join(CSRC, src), "-o", obj]
        jobs.append((src, obj, cmd, "g++"))
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(jobs)) as pool:
        results = list(pool.map(lambda j: subprocess.run(j[2], capture_output=True, text=True), jobs))
    log = []
    objs = []
    for (src, obj, _, tool), r in zip(jobs, results):
        log.append(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"{tool} failed on {src}:\n{r.stderr}")
        objs.append(obj)
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(os.path.join(BUILD, "build.log"), "w") as f:
        f.write("\n".join(log))
    if verbose or ptxas_info:
        print("\n".join(x for x in log if x.strip()))
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, ptxas_info=a.ptxas_info, verbose=True))


if __name__ == "__main__":
    sys.exit(main())
