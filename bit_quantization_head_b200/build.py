"""Builds libkvtc.so in-tree for sm_100a (nvcc cross-compiles without a GPU).

python -m bit_quantization_head_b200.build [--verbose]
"""
from __future__ import annotations

import concurrent.futures as cf
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libkvtc.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "-I" + os.path.join(ROOT, "include")]

SOURCES = ["host_plan.cpp", "host_calibrate.cpp", "encode_append.cu", "encode_prefill.cu", "decode.cu", "decode_rope.cu", "decode_noalloc.cu"] + [f"decode_v{b}.cu" for b in range(2, 9)]


def _deps_hash(src):
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".h", ".cuh")):
            h.update(open(os.path.join(CSRC, name), "rb").read())
    h.update(open(os.path.join(ROOT, "include", "kvtc.h"), "rb").read())
    h.update(open(os.path.join(CSRC, src), "rb").read())
    h.update(" ".join(ARCH + FLAGS).encode())
    return h.hexdigest()[:16]


def _compile(src, verbose):
    obj = os.path.join(BUILD, src + "." + _deps_hash(src) + ".o")
    if os.path.exists(obj):
        return obj, ""
    cmd = [NVCC] + ARCH + FLAGS + ["-c", os.path.join(CSRC, src), "-o", obj + ".tmp"]
    if src.endswith(".cu") and verbose:
        cmd += ["-Xptxas", "-v"]
    if src.endswith(".cpp"):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-Wall", "-I" + os.path.join(ROOT, "include"),
               "-I/usr/local/cuda/include", "-c", os.path.join(CSRC, src), "-o", obj + ".tmp"]
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"compile failed: {src}\n{p.stdout}\n{p.stderr}")
    os.replace(obj + ".tmp", obj)
    return obj, p.stdout + p.stderr


def build(verbose=False):
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=max(2, os.cpu_count() or 2)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    objs = [r[0] for r in results]
    if verbose:
        for (o, log), s in zip(results, SOURCES):
            if log.strip():
                print(f"--- {s}\n{log}")
    tmp = LIB + ".tmp"
    cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-lpthread"]
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"link failed\n{p.stdout}\n{p.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv))
