"""Measurements behind the roofline denominators of bench.py (bench-side, not the library).

    python bench_probes/probe.py sfu    # lg2/ex2 issue rate per SM per clock (solver bound)
    python bench_probes/probe.py hbm    # HBM read-only / write-only / copy bandwidth

The kernels are in hqq_probe.cu, built here into libhqq_probe.so (nvcc, sm_100a).
"""
from __future__ import annotations

import ctypes
import json
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "hqq_probe.cu")
LIB = os.path.join(HERE, "libhqq_probe.so")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp.%d" % os.getpid()
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        subprocess.check_call([nvcc, *FLAGS, SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def sfu():
    """Measured lg2/ex2 issue rate per SM per clock; clocks sampled meanwhile."""
    import torch
    sys.path.insert(0, ROOT)
    from bench import SM_MAX_MHZ, ClockSampler
    L = ctypes.CDLL(build())
    L.hqq_probe_sfu.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, ctypes.c_void_p]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    res = {"probe": "sfu", "sms": sms}
    with ClockSampler(0) as clk:
        for op, per, name in ((0, 1, "ex2"), (1, 1, "lg2"), (2, 2, "lg2+ex2")):
            blocks, threads, iters = sms * 8, 256, 4096
            out = torch.empty(blocks * threads, device="cuda")
            st = torch.cuda.current_stream()
            for _ in range(2):
                assert L.hqq_probe_sfu(op, out.data_ptr(), blocks, threads, iters,
                                       st.cuda_stream) == 0
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            L.hqq_probe_sfu(op, out.data_ptr(), blocks, threads, iters, st.cuda_stream)
            e1.record(st)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            ops = blocks * threads * iters * 8 * per
            res[name] = {"ms": round(ms, 3), "ops_per_s": ops / (ms * 1e-3)}
    c = clk.summary()
    res["clocks"] = c
    # The probe runs for milliseconds, shorter than the 200 ms clock sampling, so the rate
    # is normalised at the maximum SM clock (the clock held under the bench's sustained load).
    mhz = c.get("sm_max_mhz") or SM_MAX_MHZ
    res["normalised_at_mhz"] = mhz
    for name in ("ex2", "lg2", "lg2+ex2"):
        res[name]["per_clk_per_sm"] = round(res[name]["ops_per_s"] / sms / (mhz * 1e6), 2)
    return res


def hbm(gib: float = 1.0):
    """HBM bandwidth for read-only, write-only and copy traffic (16-byte accesses, grid of
    SMs x 8 blocks of 256 threads), on a buffer of `gib` GiB (far above L2)."""
    import torch
    L = ctypes.CDLL(build())
    L.hqq_probe_hbm.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    blocks, threads = sms * 8, 256
    nbytes = int(gib * (1 << 30)) // 16 * 16
    a = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    b = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    sink = torch.empty(blocks * threads, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()
    res = {"probe": "hbm", "bytes": nbytes}
    for op, name, moved in ((0, "write", nbytes), (1, "read", nbytes), (2, "copy", 2 * nbytes)):
        dst = sink if op == 1 else b
        for _ in range(3):
            assert L.hqq_probe_hbm(op, a.data_ptr(), dst.data_ptr(), nbytes, blocks, threads,
                                   st.cuda_stream) == 0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(10):
            L.hqq_probe_hbm(op, a.data_ptr(), dst.data_ptr(), nbytes, blocks, threads,
                            st.cuda_stream)
        e1.record(st)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 10
        res[name] = {"ms": round(ms, 4), "GB_per_s": round(moved / ms / 1e6, 1)}
    return res


if __name__ == "__main__":
    what = sys.argv[1] if len(sys.argv) > 1 else ""
    if what == "build":
        print(build(force=True))
    elif what in ("sfu", "hbm"):
        print(json.dumps(sfu() if what == "sfu" else hbm()), flush=True)
    else:
        raise SystemExit(__doc__)
