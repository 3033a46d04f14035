"""Build the CUDA libraries in-tree with nvcc for sm_100a.

    python -m quantized_kv_cache_17_b200.build [--force]

Produces ``quantized_kv_cache_17_b200/libkvq.so`` (the product library) and
``kvq_inputs/libkvq_gen.so`` (the device twin of the seeded input generator).
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
LIB = os.path.join(PKG, "libkvq.so")
GEN_SRC = os.path.join(ROOT, "kvq_inputs", "csrc", "kvq_gen.cu")
GEN_LIB = os.path.join(ROOT, "kvq_inputs", "libkvq_gen.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
                 "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]
SOURCES = {
    "kvq_abi.cu": [],
    "kvq_append.cu": ["-fmad=false"],     # quantiser: no fused multiply-add anywhere in this unit
    "kvq_decode.cu": [],
    "kvq_noalloc.cu": [],
    "kvq_resident.cu": [],
}


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _headers():
    hs = [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    hs += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    return hs


def _compile(src: str, extra, verbose: bool) -> str:
    os.makedirs(BUILD, exist_ok=True)
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    if _stale(obj, [src, __file__] + _headers()):
        cmd = [nvcc(), "-c", src, "-o", obj] + COMMON + list(extra)
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stderr.strip() or r.stdout.strip()):
            print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if force and os.path.isdir(BUILD):
        for f in os.listdir(BUILD):
            os.remove(os.path.join(BUILD, f))
    srcs = [(os.path.join(CSRC, s), f) for s, f in SOURCES.items()]
    with cf.ThreadPoolExecutor(max_workers=len(srcs) + 1) as ex:
        futs = [ex.submit(_compile, s, f, verbose) for s, f in srcs]
        gen_fut = ex.submit(_compile, GEN_SRC, [], verbose)
        objs = [f.result() for f in futs]
        gen_obj = gen_fut.result()
    if force or _stale(LIB, objs):
        subprocess.run([nvcc()] + ARCH + ["-shared", "-o", LIB] + objs, check=True)
    if force or _stale(GEN_LIB, [gen_obj]):
        subprocess.run([nvcc()] + ARCH + ["-shared", "-o", GEN_LIB, gen_obj], check=True)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    sys.exit(0)
