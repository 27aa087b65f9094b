"""Builds libtempcache.so (the C-ABI library) for sm_100a with nvcc, in-tree.

Run `python kv_cache_attention_tempcache_b200/build.py` (add --ptxas for register
and spill reports) or call build(). Objects
go to kv_cache_attention_tempcache_b200/_build/, the library to
kv_cache_attention_tempcache_b200/_lib/libtempcache.so.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "_lib", "libtempcache.so")
SOURCES = ["tc_runtime.cu", "tc_commit.cu", "tc_attn_bf16.cu", "tc_attn_f32.cu", "tc_noalloc.cu", "tc_annca.cu", "tc_lvsa.cu"]
HEADERS = [os.path.join(CSRC, "tc_internal.h"), os.path.join(CSRC, "tc_device.cuh"),
           os.path.join(ROOT, "include", "tempcache.h")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(extra=()):
    return ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include"), *extra]


def _stale(obj, src):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src, *HEADERS])


def build(verbose: bool = False, ptxas_info: bool = False) -> str:
    nvcc = nvcc_path()
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    jobs = []
    for name in SOURCES:
        src = os.path.join(CSRC, name)
        obj = os.path.join(BUILD, name.replace(".cu", ".o"))
        if ptxas_info or _stale(obj, src):
            jobs.append([nvcc, *flags(extra), "-c", src, "-o", obj])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with ThreadPoolExecutor(max_workers=4) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose or ptxas_info or r.returncode:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode:
                raise RuntimeError(f"nvcc failed for {cmd[-3]}")
    objs = [os.path.join(BUILD, n.replace(".cu", ".o")) for n in SOURCES]
    if jobs or not os.path.exists(LIB):
        link = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", LIB, *objs]
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return LIB


if __name__ == "__main__":
    print(build(verbose=True, ptxas_info="--ptxas" in sys.argv))
