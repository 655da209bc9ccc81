"""Build libhqq_b200.so in-tree with nvcc for sm_100a.

    python -m calibration_free_weight_hqq_b200.build [--force]

Each .cu file is compiled to an object in parallel, then linked into a shared library next
to this file. -fmad=false keeps every fp32/fp64 multiply and add separately rounded, as the
quantization definition requires (the kernels also use explicit _rn intrinsics).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libhqq_b200.so")
SOURCES = ["hqq_abi.cu", "hqq_quantize.cu", "hqq_quantize_stop.cu", "hqq_dequantize.cu",
           "hqq_noalloc.cu", "hqq_gemm.cu", "hqq_mx.cu"]
HEADERS = ["hqq_device.cuh", "hqq_kernels.h", "hqq_quantize_impl.cuh", "hqq_abi_internal.h"]
PUBLIC_HEADER = os.path.join(ROOT, "include", "hqq", "hqq.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-Xptxas", "-v",
    "-I" + os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    common = [os.path.join(CSRC, h) for h in HEADERS] + [PUBLIC_HEADER, __file__]
    procs, objs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD_DIR, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + common):
            log = open(o + ".log", "w")
            cmd = [nvcc(), *NVCC_FLAGS, "-c", s, "-o", o]
            procs.append((subprocess.Popen(cmd, stdout=log, stderr=subprocess.STDOUT), o, cmd))
    for p, o, cmd in procs:
        rc = p.wait()
        text = open(o + ".log").read()
        if rc != 0:
            raise RuntimeError("nvcc failed (%d): %s\n%s" % (rc, " ".join(cmd), text))
        if verbose:
            print(text)
    if force or procs or _stale(LIB, objs):
        tmp = LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                               *objs, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
