"""Benchmark: whole Llama-7B-shaped model HQQ quantization on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

A step is one pass of the whole hot path over the model: quantize all 224 linear weights
(32 blocks x q,k,v,o [4096,4096], gate,up [11008,4096], down [4096,11008]; 6,476,005,376 bf16
weights, 4-bit, group 64, axis 1, iters 20, p 0.7, beta0 10, kappa 1.01) and dequantize
them all back to bf16. Inputs are synthetic (seeded, LLM-like; see
calibration_free_weight_hqq_b200/synthetic.py), resident in HBM (13 GB, far above the 126 MB
L2, so no flush is needed between steps).

Printed on rank 0: one JSON line with the metric (Gweights/s, whole job), the per-kernel
roofline of the dominant kernel (the solver, bound by the MUFU rate), an end-to-end figure
through the public API with host buffers, the oracle timed on the host as the CPU baseline,
and the SM clocks sampled during the timed region.

--impl reference times the CPU oracle (the only reference this path has) on bounded samples
of the same workload and prints the same metric with "impl": "reference".

Multi-GPU (torchrun): weak scaling - every rank quantizes its own model replica (distinct
seeds); no collective on the data path; the barrier and the max-over-ranks time use NCCL.
--shard instead splits one model's matrices over the ranks (strong scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "HQQ quantize Gweights/s & % roofline (HBM|SFU), 7B-shaped bf16 4-bit g64"
UNIT = "Gweights/s"
MUFU_PER_CLK_PER_SM = 16          # lg2/ex2 issue rate of the B200 SFU (probed: 15.9 with
                                  # bench_probes/probe.py sfu)
N_SM = 148
SM_MAX_MHZ = 1965.0


def peaks():
    p = {"hbm_gbs": 6535.7, "sm_max_mhz": SM_MAX_MHZ, "source": "fallback"}
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        p.update({k: m[k] for k in ("hbm_gbs", "sm_max_mhz") if k in m})
        p["source"] = "measured"
    return p


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9 or not f[1].isdigit():
                    continue
                sm.append(int(f[1]))
                mx.append(int(f[2]))
                for n, v in zip(names, f[5:9]):
                    if v.lower() in ("active", "1"):
                        reasons.add(n)
        finally:
            os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- multi-rank helpers


def replica_seed_offset(rank: int) -> int:
    """Weak scaling: rank r quantizes its own model replica, seeded apart from the others."""
    return rank * 100003


def partition_by_weight(sizes, world: int):
    """Strong scaling (--shard): split matrix indices over ranks, largest first onto the
    least-loaded rank, so every matrix lands on exactly one rank and loads stay balanced."""
    loads = [0] * world
    parts = [[] for _ in range(world)]
    for i in sorted(range(len(sizes)), key=lambda i: -sizes[i]):
        r = min(range(world), key=lambda r: loads[r])
        parts[r].append(i)
        loads[r] += sizes[i]
    return [sorted(p) for p in parts]


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (every rank gets it)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def build_model(workload, device, seed_offset: int):
    from calibration_free_weight_hqq_b200 import synthetic
    Ws = []
    for m in workload.matrices:
        sigma = synthetic.layer_sigma(m.seed + seed_offset) if m.per_layer_sigma else 0.02
        Ws.append(synthetic.weight(m.rows, m.cols, seed=m.seed + seed_offset, dtype=m.dtype,
                                   outlier_rate=m.outlier_rate, sigma_layer=sigma, device=device))
    return Ws


def alloc_outputs(hqq, workload, device):
    outs, deqs = [], []
    for m in workload.matrices:
        ng = m.rows * m.cols // m.group_size
        outs.append((torch.empty(hqq.hqq_packed_bytes(m.rows, m.cols, m.nbits), dtype=torch.uint8,
                                 device=device),
                     torch.empty(ng, dtype=m.dtype, device=device),
                     torch.empty(ng, dtype=m.dtype, device=device)))
        deqs.append(torch.empty((m.rows, m.cols), dtype=m.dtype, device=device))
    return outs, deqs


def run_ours(args, rank, world, dev):
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import workloads
    wl = workloads.llama7b_model_4b()
    if args.shard and world > 1:
        part = partition_by_weight([m.numel for m in wl.matrices], world)[rank]
        wl = workloads.Workload(wl.name, wl.description, [wl.matrices[i] for i in part])
    mats = wl.matrices
    Ws = build_model(wl, dev, seed_offset=0 if args.shard else replica_seed_offset(rank))
    outs, deqs = alloc_outputs(hqq, wl, dev)
    stream = torch.cuda.current_stream()
    n_w = wl.weights
    pk = peaks()

    m0 = mats[0]
    params = hqq.make_params(m0.nbits, m0.group_size, m0.axis, m0.iters, m0.p, m0.beta0,
                             m0.kappa, w_dtype=m0.dtype)
    qbatch = hqq.matrix_batch(Ws, outs)   # built once: descriptors of all 224 matrices
    dbatch = hqq.matrix_batch(deqs, outs)
    shapes = [(m.rows, m.cols) for m in mats]

    def step(ev=None):
        if args.per_matrix:
            for i, (m, W, (p, s, z)) in enumerate(zip(mats, Ws, outs)):
                if ev is not None:
                    ev[i][0].record(stream)
                hqq.hqq_quantize(W, m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0,
                                 m.kappa, Wq_packed=p, scale=s, zero=z, stream=stream)
                if ev is not None:
                    ev[i][1].record(stream)
            for m, (p, s, z), D in zip(mats, outs, deqs):
                hqq.hqq_dequantize(p, s, z, m.rows, m.cols, m.nbits, m.group_size, m.axis,
                                   out=D, stream=stream)
            return
        # the whole model in one solver launch and one dequantize launch
        if ev is not None:
            ev[0][0].record(stream)
        hqq.hqq_quantize_batched(Ws, params, outs=outs, batch=qbatch, stream=stream)
        if ev is not None:
            ev[0][1].record(stream)
        hqq.hqq_dequantize_batched(outs, shapes, params, W_out=deqs, batch=dbatch, stream=stream)
        if ev is not None:
            ev[0][2].record(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    n_q = len(mats) if args.per_matrix else 1  # solver launches per step
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_q)]
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        barrier()
        t0.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t1.record(stream)
        barrier()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    q_ms = [e[0].elapsed_time(e[1]) for ev in evs for e in ev]
    dq_ms = None if args.per_matrix else [ev[0][1].elapsed_time(ev[0][2]) for ev in evs]
    ms_step = ms_total / args.steps
    # weak: every rank did a whole model; strong (--shard): the ranks shared one model
    total_weights = workloads.llama7b_model_4b().weights if args.shard else world * n_w
    value = total_weights / (ms_step * 1e-3) / 1e9

    # roofline of the dominant kernel (the solver): algorithmic MUFU work per launch over
    # its measured average launch duration
    launches = len(q_ms)
    avg_launch_ms = sum(q_ms) / launches
    mufu_per_weight = 2 * (mats[0].iters + 1)
    avg_weights = n_w / n_q
    achieved = mufu_per_weight * avg_weights / (avg_launch_ms * 1e-3) / 1e12
    peak = MUFU_PER_CLK_PER_SM * N_SM * pk["sm_max_mhz"] * 1e6 / 1e12
    traffic = _traffic_per_launch(avg_weights)
    clocks = clk.summary()
    quant_share = sum(q_ms) / args.steps / ms_step

    res = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "strong" if args.shard else "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded LLM-like bf16 weights: per-row sigma, 0.1% outliers)",
        "config": {"workload": wl.name, "matrices": len(mats), "weights": n_w,
                   "w_dtype": "bf16", "nbits": 4, "group_size": 64, "axis": 1, "iters": 20,
                   "p": 0.7, "beta0": 10.0, "kappa": 1.01,
                   "step": "quantize all 224 matrices + dequantize all 224 to bf16",
                   "launches_per_step": ("224 solver + 224 dequantize" if args.per_matrix
                                         else "1 batched solver + 1 batched dequantize"),
                   "l2": "inputs 13 GB > 126 MB L2, no flush",
                   "quantize_share_of_step": round(quant_share, 4),
                   "quantize_Gweights_per_s": round(n_w / (sum(q_ms) / args.steps * 1e-3) / 1e9, 3),
                   "dequantize": _dequant_figures(dq_ms, n_w, pk)},
        "roofline": {"bound": "alu", "kernel": "quantize_kernel (MUFU lg2+ex2)",
                     "achieved": round(achieved, 4), "peak": round(peak, 4), "unit": "Top/s (MUFU)",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic": f"{mufu_per_weight} MUFU/weight x {avg_weights:.0f} weights/launch",
                     "avg_launch_ms": round(avg_launch_ms, 4),
                     "hbm_frac": round(2.5625 * avg_weights / (avg_launch_ms * 1e-3) / 1e9
                                       / pk["hbm_gbs"], 4),
                     "peak_source": f"16 MUFU/clk/SM x 148 SM x {pk['sm_max_mhz']} MHz "
                                    f"(probed 15.9/clk/SM); hbm {pk['hbm_gbs']} GB/s {pk['source']}"},
        "clocks": clocks,
        "gpu_launches": 2 * n_q * args.steps,
    }
    if not args.per_matrix:
        res["fixed_point_stop"] = run_fixed_point(hqq, wl, Ws, outs, deqs, params, shapes,
                                                  stream, args)
    if rank == 0 and not args.no_e2e:
        res["e2e"] = run_e2e(hqq, wl, Ws, outs, params, dev, args)
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, Ws, args.cpu_seconds)
    if rank == 0 and not args.no_linear:
        del Ws, outs, deqs, qbatch, dbatch
        torch.cuda.empty_cache()
        if not args.no_configs:
            res["configs"] = configs_table(reps=max(3, min(args.steps, 10)))
        res["w4a16_linear"] = run_linear(hqq, dev, args)
        res["mxfp4_weightonly"] = run_mxfp4(hqq, dev, args)
    return res


def _dequant_figures(dq_ms, n_w, pk):
    """The batched dequantize launch of the step: average duration (CUDA events around it on
    the launch stream), algorithmic GB/s (2.5625 B per weight: read 0.5 B of codes and 4 B of
    bf16 scale/zero per 64 weights, write 2 B) and the fraction of the measured HBM copy
    bandwidth."""
    if not dq_ms:
        return None
    ms = sum(dq_ms) / len(dq_ms)
    gbs = 2.5625 * n_w / (ms * 1e-3) / 1e9
    return {"kernel": "dequant4_axis1_kernel (batched)", "avg_launch_ms": round(ms, 4),
            "GB_per_s": round(gbs, 1), "hbm_frac": round(gbs / pk["hbm_gbs"], 4),
            "algorithmic": "2.5625 B/weight"}


def solver_source_digest() -> str:
    """sha1 of the solver's sources, to tell whether a recorded capture is still current."""
    import hashlib
    h = hashlib.sha1()
    for f in ("hqq_quantize.cu", "hqq_quantize_impl.cuh", "hqq_device.cuh"):
        with open(os.path.join(HERE, "calibration_free_weight_hqq_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def run_fixed_point(hqq, wl, Ws, outs, deqs, params, shapes, stream, args):
    """The same step with HQQ_FLAG_STOP_AT_FIXED_POINT (bit-identical results; a warp stops
    once every remaining evaluation of its groups would repeat the last one). Reported beside
    the headline, not as it: the work done then depends on the data."""
    import ctypes
    fp = hqq.HQQParams.from_buffer_copy(params)
    fp.flags = hqq.HQQ_FLAG_STOP_AT_FIXED_POINT
    qb, db = hqq.matrix_batch(Ws, outs), hqq.matrix_batch(deqs, outs)

    def step():
        hqq.hqq_quantize_batched(Ws, fp, outs=outs, batch=qb, stream=stream)
        hqq.hqq_dequantize_batched(outs, shapes, fp, W_out=deqs, batch=db, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    return {"value": round(wl.weights / (ms * 1e-3) / 1e9, 3), "unit": UNIT,
            "ms_per_step": round(ms, 3), "flag": "HQQ_FLAG_STOP_AT_FIXED_POINT",
            "results": "bit-identical to the headline run (tests/test_gpu_fixed_point.py)"}


def _traffic_per_launch(avg_weights):
    """DRAM bytes (read + write) of one solver launch, from the committed ncu capture
    (bytes per weight measured on one [16384, 8192] bf16 launch, scaled to the average launch
    here). None if no capture is recorded or the solver changed since it was taken."""
    path = os.path.join(HERE, "profiles", "quantize_kernel_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    if t.get("solver_source_sha1") != solver_source_digest():
        return None
    return round(t["dram_bytes_per_weight"] * avg_weights)


def linear_source_digest() -> str:
    import hashlib
    h = hashlib.sha1()
    for f in ("hqq_gemm.cu", "hqq_device.cuh"):
        with open(os.path.join(HERE, "calibration_free_weight_hqq_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def capture_graph(fn):
    """fn's launches (on the current stream) captured in a CUDA graph, after one plain run."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
        side.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    return graph


def time_graph(graph, warmup: int, steps: int, flush) -> float:
    """Device time (ms) of one replay, L2 flushed (flush buffer written) before each: the mean
    of the per-replay CUDA-event times after dropping the fastest and slowest 10 %. Event times
    on B200 come in steps of 2.048 us, so a median of a short launch is quantized to that step;
    the trimmed mean of at least 20 replays resolves differences below it and still ignores
    outliers."""
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    per = []
    for _ in range(max(steps, 20)):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b))
    per.sort()
    cut = len(per) // 10
    kept = per[cut:len(per) - cut]
    return sum(kept) / len(kept)


def run_linear(hqq, dev, args, tokens: int = 4096):
    """The consumer of the packed format (row f2): the seven linear layers of one Llama-7B
    block (q, k, v, o [4096,4096]; gate, up [11008,4096]; down [4096,11008]) quantized to
    4-bit g64 axis 1, applied to a prefill batch of `tokens` bf16 tokens with hqq_linear
    (dequantization fused into the tcgen05 GEMM, bit-identical to hqq_dequantize). Beside it,
    in the same run: the unfused path (hqq_dequantize + torch.matmul on the bf16 result) and
    cuBLAS on an already dequantized bf16 weight. L2 is flushed (256 MB write) before every
    step; each launch is timed with CUDA events on the launching stream."""
    from calibration_free_weight_hqq_b200 import synthetic, workloads
    wl = workloads.llama7b_block_4b()
    stream = torch.cuda.current_stream()
    layers = []
    for m in wl.matrices:
        W = workloads.make_weight(m, dev)
        pk, sc, zr = hqq.hqq_quantize(W, 4, 64, 1)
        X = synthetic.activations(tokens, m.cols, seed=m.seed + 7, device=dev)
        Y = torch.empty(tokens, m.rows, dtype=torch.bfloat16, device=dev)
        Wd = hqq.hqq_dequantize(pk, sc, zr, m.rows, m.cols, 4, 64, 1)
        layers.append((m, X, pk, sc, zr, Y, Wd))
        del W
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    scratch = torch.empty(max(m.rows * m.cols for m, *_ in layers), dtype=torch.bfloat16,
                          device=dev)  # the unfused path's dequantized weight
    flops = sum(2.0 * tokens * m.rows * m.cols for m, *_ in layers)

    def timed(fn, steps):
        per = []
        for _ in range(args.warmup):
            for L in layers:
                fn(*L)
        torch.cuda.synchronize()
        for _ in range(steps):
            flush.fill_(1)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in layers]
            for (a, b), L in zip(evs, layers):
                a.record(stream)
                fn(*L)
                b.record(stream)
            torch.cuda.synchronize()
            per.append(sum(a.elapsed_time(b) for a, b in evs))
        return statistics.median(per)

    ms_fused = timed(lambda m, X, pk, sc, zr, Y, Wd: hqq.hqq_linear(X, pk, sc, zr, m.rows, Y=Y,
                                                                     stream=stream), args.steps)
    ms_unfused = timed(lambda m, X, pk, sc, zr, Y, Wd: torch.matmul(
        X, hqq.hqq_dequantize(pk, sc, zr, m.rows, m.cols, 4, 64, 1, stream=stream,
                              out=scratch[:m.rows * m.cols].view(m.rows, m.cols)).t(), out=Y),
        args.steps)
    ms_cublas = timed(lambda m, X, pk, sc, zr, Y, Wd: torch.matmul(X, Wd.t(), out=Y), args.steps)
    tf = flops / (ms_fused * 1e-3) / 1e12
    peak, source = None, "fallback"
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            peak = json.load(f).get("bf16_tflops")
        source = "measured"
    if peak is None:
        peak = 1590.0
    # DRAM traffic of one 4096^3 launch from the committed ncu capture (the launches here
    # have three shapes, so it is reported for that case, not scaled)
    profiled = None
    tpath = os.path.join(HERE, "profiles", "w4a16_gemm_kernel_traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            t = json.load(f)
        if t.get("source_sha1") == linear_source_digest():
            profiled = {"shape_MNK": [4096, 4096, 4096],
                        "dram_bytes": t.get("dram_bytes_per_launch_4096x4096x4096"),
                        "algorithmic_bytes": 2 * 4096 * 4096 * 2 + 4096 * 4096 // 2 + 4096 * 64 * 4}
    # decode-sized batch: the same layers at 16 tokens take the warp-MMA decode kernel;
    # weight-read bound (0.5 B of codes + 4/64 B of bf16 scale/zero per weight from HBM). A
    # launch takes microseconds, less than the binding's host time, so the seven launches of a
    # step are captured in a CUDA graph and the replay is timed (L2 flushed before each).
    dec_tokens = 16
    dec = []
    for m, X, pk, sc, zr, Y, Wd in layers:
        Xd = X[:dec_tokens].contiguous()
        Yd = torch.empty(dec_tokens, m.rows, dtype=torch.bfloat16, device=dev)
        dec.append((m, Xd, pk, sc, zr, Yd, Wd))

    # the weights were quantized and synchronised before: the decode launches may overlap the
    # previous layer's tail (HQQ_FLAG_OVERLAP_WEIGHTS, programmatic dependent launch)
    p_ovl = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, meta_dtype=torch.bfloat16,
                            overlap_weights=True)

    def dec_fused():
        for m, Xd, pk, sc, zr, Yd, Wd in dec:
            hqq.hqq_linear(Xd, pk, sc, zr, m.rows, p_ovl, Y=Yd)

    def dec_fused_plain():
        for m, Xd, pk, sc, zr, Yd, Wd in dec:
            hqq.hqq_linear(Xd, pk, sc, zr, m.rows, Y=Yd)

    def dec_cublas():
        for m, Xd, pk, sc, zr, Yd, Wd in dec:
            torch.matmul(Xd, Wd.t(), out=Yd)

    ms_dec = time_graph(capture_graph(dec_fused), args.warmup, args.steps, flush)
    ms_dec_plain = time_graph(capture_graph(dec_fused_plain), args.warmup, args.steps, flush)
    ms_dec_cublas = time_graph(capture_graph(dec_cublas), args.warmup, args.steps, flush)
    dec_fused()  # leave the fused result in Yd
    wbytes = sum(m.rows * m.cols * (0.5 + 4 / 64) for m, *_ in dec)
    hbm = peaks()["hbm_gbs"]
    dec_gbs = wbytes / (ms_dec * 1e-3) / 1e9
    return {
        "metric": "fused 4-bit linear TFLOP/s", "value": round(tf, 1), "unit": "TFLOP/s",
        "workload": f"Llama-7B block linear layers, {tokens} tokens, bf16 activations, "
                    "4-bit g64 axis-1 weights",
        "ms_per_step": round(ms_fused, 4), "launches_per_step": len(layers),
        "unfused_dequantize_plus_cublas_tflops": round(flops / (ms_unfused * 1e-3) / 1e12, 1),
        "cublas_bf16_weight_tflops": round(flops / (ms_cublas * 1e-3) / 1e12, 1),
        "roofline": {"bound": "tensor", "kernel": "w4a16_gemm_2sm_kernel (tcgen05 cta_group::2)",
                     "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tf / peak, 4), "traffic": None,
                     "traffic_profiled_case": profiled,
                     "algorithmic": "2*M*N*K flops per launch",
                     "peak_source": f"bf16 dense, {source} (burst: the kernel is timed alone)"},
        "l2": "flushed before every step",
        "decode_16_tokens": {
            "kernel": "w4a16_gemv_kernel (warp-level MMA on registers, split-K over a cluster "
                      "of up to 8 CTAs)",
            "timing": "CUDA graph of the 7 launches, L2 flushed before each replay",
            "ms_per_step": round(ms_dec, 4), "launches_per_step": len(dec),
            "overlap": "HQQ_FLAG_OVERLAP_WEIGHTS (programmatic dependent launch: a layer may "
                       "start, and load its weight codes, before the previous layer finishes)",
            "ms_per_step_without_overlap": round(ms_dec_plain, 4),
            "cublas_bf16_weight_ms_per_step": round(ms_dec_cublas, 4),
            "tflops": round(sum(2.0 * dec_tokens * m.rows * m.cols for m, *_ in dec)
                            / (ms_dec * 1e-3) / 1e12, 2),
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(dec_gbs / hbm, 4),
                         "algorithmic": "0.5625 B of packed codes + scale/zero per weight"}},
        "wait_timeouts": hqq.hqq_wait_timeouts(),
        "gpu_launches": 3 * len(layers) * args.steps,
    }


def run_mxfp4(hqq, dev, args):
    """Row f3, the MXFP4 weight-only encoding: one [28672, 8192] bf16 weight (the 70B-class
    MLP shape, 235M weights, 470 MB: above L2), encode and decode timed separately with CUDA
    events over `steps` launches after warm-up. Both are HBM-bound: 2.53125 algorithmic bytes
    per weight (read 2 B bf16; write 0.5 B codes + 1/32 B scale, or the reverse)."""
    from calibration_free_weight_hqq_b200 import synthetic
    rows, cols = 28672, 8192
    W = synthetic.weight(rows, cols, seed=3, dtype=torch.bfloat16, device=dev)
    codes, scales = hqq.hqq_mxfp4_quantize(W)
    D = torch.empty_like(W)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    ms_q = timed(lambda: hqq.hqq_mxfp4_quantize(W, codes=codes, scales=scales))
    ms_d = timed(lambda: hqq.hqq_mxfp4_dequantize(codes, scales, rows, cols, out=D))
    n = rows * cols
    bpw = 2.53125
    hbm = peaks()["hbm_gbs"]
    gbs_q, gbs_d = n * bpw / (ms_q * 1e-3) / 1e9, n * bpw / (ms_d * 1e-3) / 1e9
    return {"metric": "MXFP4 weight-only encode Gweights/s", "unit": "Gweights/s",
            "value": round(n / (ms_q * 1e-3) / 1e9, 1),
            "decode_Gweights_per_s": round(n / (ms_d * 1e-3) / 1e9, 1),
            "workload": "one [28672, 8192] bf16 weight, blocks of 32 along rows",
            "ms_encode": round(ms_q, 4), "ms_decode": round(ms_d, 4),
            "roofline": {"bound": "hbm", "kernel": "mxfp4_quantize_kernel",
                         "achieved": round(gbs_q, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs_q / hbm, 4), "traffic": None,
                         "algorithmic": "2.53125 B/weight x 234881024 weights",
                         "decode_achieved": round(gbs_d, 1),
                         "decode_frac": round(gbs_d / hbm, 4)},
            "gpu_launches": 2 * args.steps}


def run_e2e(hqq, wl, Ws, outs, params, dev, args):
    """Same metric through the public API with host buffers, on the batched calls the
    headline uses: every step copies each weight from pinned host memory, quantizes and
    dequantizes it, and reads the quantized model (packed codes, scale, zero) back into pinned
    host memory. The model goes through in chunks of one decoder block (7 matrices: one
    hqq_quantize_batched and one hqq_dequantize_batched call each), so that the host-to-device
    copy of block b+1, the kernels of block b and the device-to-host copy of block b-1 overlap
    on three streams; three staging slots on the device hold the blocks in flight."""
    mats = wl.matrices
    host_W = [torch.empty_like(W, device="cpu", pin_memory=True).copy_(W) for W in Ws]
    host_out = [tuple(torch.empty_like(t, device="cpu", pin_memory=True) for t in o)
                for o in outs]
    comp, h2d, d2h = (torch.cuda.Stream(dev) for _ in range(3))
    per_chunk = 7
    chunks = [list(range(i, min(i + per_chunk, len(mats)))) for i in range(0, len(mats), per_chunk)]
    n_slot = 3
    slot_elems = max(sum(mats[i].numel for i in c) for c in chunks)
    slot_in = [torch.empty(slot_elems, dtype=torch.bfloat16, device=dev) for _ in range(n_slot)]
    slot_deq = [torch.empty(slot_elems, dtype=torch.bfloat16, device=dev) for _ in range(n_slot)]
    views, qb, db = [], [], []
    for c_i, c in enumerate(chunks):
        s, off, wv, dv = c_i % n_slot, 0, [], []
        for i in c:
            m = mats[i]
            wv.append(slot_in[s][off:off + m.numel].view(m.rows, m.cols))
            dv.append(slot_deq[s][off:off + m.numel].view(m.rows, m.cols))
            off += m.numel
        views.append((wv, dv))
        qb.append(hqq.matrix_batch(wv, [outs[i] for i in c]))
        db.append(hqq.matrix_batch(dv, [outs[i] for i in c]))
    slot_free = [torch.cuda.Event() for _ in range(n_slot)]
    for e in slot_free:
        e.record(comp)
    h2d_bytes = sum(W.numel() * W.element_size() for W in host_W)
    d2h_bytes = sum(sum(t.numel() * t.element_size() for t in o) for o in host_out)
    launches = 0

    def step():
        nonlocal launches
        for c_i, c in enumerate(chunks):
            s = c_i % n_slot
            wv, dv = views[c_i]
            h2d.wait_event(slot_free[s])
            with torch.cuda.stream(h2d):
                for i, buf in zip(c, wv):
                    buf.copy_(host_W[i], non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(h2d)
            comp.wait_event(loaded)
            sub_outs = [outs[i] for i in c]
            hqq.hqq_quantize_batched(wv, params, outs=sub_outs, batch=qb[c_i], stream=comp)
            hqq.hqq_dequantize_batched(sub_outs, [tuple(v.shape) for v in dv], params,
                                       W_out=dv, batch=db[c_i], stream=comp)
            launches += 2
            slot_free[s].record(comp)
            done = torch.cuda.Event()
            done.record(comp)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                for i in c:
                    for src, dst in zip(outs[i], host_out[i]):
                        dst.copy_(src, non_blocking=True)
        d2h.synchronize()
        comp.synchronize()

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    launches = 0
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    sec = (time.perf_counter() - t) / args.steps
    return {"value": round(wl.weights / sec / 1e9, 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
            "ms_per_step": round(sec * 1e3, 2), "steps": args.steps,
            "gpu_launches": launches,
            "how": "per decoder block (7 matrices): pinned host W -> device (stream 1); "
                   "hqq_quantize_batched + hqq_dequantize_batched (stream 2); the quantized "
                   "model (packed codes, scale, zero; 3.64 GB) -> pinned host (stream 3). "
                   "The dequantized weights stay on the device (read back: none). Wall clock "
                   "with device synchronisation around the timed steps."}


def cpu_baseline(wl, Ws, seconds: float, impl_line=False):
    """The oracle, as it stands, on the host cores over a bounded sample of the workload:
    whole row blocks of the model's matrices in order until `seconds` of CPU time."""
    import oracle
    nt = oracle.default_threads()
    done_w, t_used, parts = 0, 0.0, []
    rows_per = 256
    i = 0
    while t_used < seconds and i < len(wl.matrices):
        m, W = wl.matrices[i], Ws[i]
        for r0 in range(0, m.rows, rows_per):
            Wh = W[r0:r0 + rows_per].float().cpu().numpy()
            t = time.perf_counter()
            oracle.quantize(Wh, m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0, m.kappa,
                            nthreads=nt)
            t_used += time.perf_counter() - t
            done_w += Wh.size
            if t_used >= seconds:
                break
        parts.append(m.name)
        i += 1
    return {"value": round(done_w / t_used / 1e9, 5), "unit": UNIT, "cores": nt, "kind": "oracle",
            "sample": f"{done_w} weights ({len(parts)} matrices, row blocks of {rows_per}) "
                      f"in {t_used:.1f} s of oracle time, {nt} threads"}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on bounded samples, timed per step."""
    from calibration_free_weight_hqq_b200 import workloads
    import oracle
    wl = workloads.llama7b_model_4b()
    nt = oracle.default_threads()
    m = wl.matrices[4]  # gate_proj [11008, 4096]
    from calibration_free_weight_hqq_b200 import synthetic
    W = synthetic.weight(m.rows, m.cols, seed=m.seed, dtype=m.dtype, outlier_rate=m.outlier_rate,
                         sigma_layer=synthetic.layer_sigma(m.seed)).float().numpy()
    rows = max(16, int(os.environ.get("HQQ_REF_ROWS", "512")))
    sample = W[:rows]
    for _ in range(args.warmup):
        oracle.quantize(sample, m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0, m.kappa,
                        nthreads=nt)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.quantize(sample, m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0, m.kappa,
                        nthreads=nt)
    sec = (time.perf_counter() - t) / args.steps
    value = sample.size / sec / 1e9
    desc = f"{rows} rows of {m.name} [{m.rows},{m.cols}] ({sample.size} weights) per step"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "sample": desc},
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": nt, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def single_linear(reps: int = 10, M: int = 4096):
    """One 4096 x 4096 hqq_linear launch with M tokens (bf16, 4-bit g64): the ncu profiling
    cases (M = 4096: the 2-SM kernel; M = 16: the decode kernel, launched with
    HQQ_FLAG_OVERLAP_WEIGHTS). `reps` launches are captured in one CUDA graph (a decode launch
    is shorter than the binding's host time) and the replay is timed; the weight (8.4 MB of
    codes) stays in L2 between launches."""
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import synthetic
    N = K = 4096
    W = synthetic.weight(N, K, seed=11, dtype=torch.bfloat16, device="cuda")
    pk, s, z = hqq.hqq_quantize(W, 4, 64, 1)
    X = synthetic.activations(M, K, seed=12, device="cuda")
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")

    p = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, overlap_weights=True)

    def launches():
        for _ in range(reps):
            hqq.hqq_linear(X, pk, s, z, N, p, Y=Y)

    graph = capture_graph(launches)
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    return {"single": "linear", "shape": [M, N, K], "ms": round(ms, 4),
            "TFLOP_per_s": round(2.0 * M * N * K / ms / 1e9, 1),
            "wait_timeouts": hqq.hqq_wait_timeouts()}


def configs_table(reps: int = 5):
    """Quantize and dequantize throughput of the four smaller workloads of the pages'
    configurations (the fifth, the whole model, is the headline), one line per configuration:
    solver Gweights/s and its MUFU fraction, dequantizer algorithmic GB/s and its HBM fraction.

    A workload whose matrices share one configuration without second-level meta (the Llama
    block at 4-bit and at 2-bit axis 0) is quantized and dequantized with the batched calls, one
    launch each, as a caller quantizing a block would; the others (one matrix; the 70B MLP with
    two bit widths and 8-bit meta, through hqq_quantize_ex) take a call per matrix, and the
    per-matrix figures are reported for every workload. Quantize: `reps` back-to-back calls
    timed with CUDA events after one warm-up (a launch takes milliseconds, so host gaps do not
    matter). Dequantize: one pass captured in a CUDA graph (so that microsecond launches run
    back to back), L2 flushed (256 MB write) before each of `reps` timed replays."""
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import workloads
    pk = peaks()
    mufu_peak = MUFU_PER_CLK_PER_SM * N_SM * pk["sm_max_mhz"] * 1e6
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def events_ms(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    def graph_ms(fn):
        fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        graph.replay()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1) / reps
        del graph
        return total

    out = []
    for wl in (workloads.single_fp16(), workloads.llama7b_block_4b(),
               workloads.llama7b_block_2b_axis0(), workloads.mlp70b_mixed()):
        Ws = [workloads.make_weight(m, "cuda") for m in wl.matrices]
        plist = [hqq.make_params(m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0, m.kappa,
                                 w_dtype=m.dtype, quant_scale=m.quant_meta,
                                 quant_zero=m.quant_meta, meta_group_size=m.meta_group_size)
                 for m in wl.matrices]
        dq_bytes = 0
        for m in wl.matrices:
            ng = m.numel // m.group_size
            meta_b = 2 * ng * (1 if m.quant_meta else 2)
            dq_bytes += hqq.hqq_packed_bytes(m.rows, m.cols, m.nbits) + meta_b + 2 * m.numel
        # per matrix: hqq_quantize_ex / hqq_dequantize_ex
        passes, q_ms_per = [], 0.0
        for m, W, params in zip(wl.matrices, Ws, plist):
            need = hqq.hqq_workspace_bytes(m.rows, m.cols, params)
            ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda") if need else None
            q = hqq.hqq_quantize_ex(W, params, workspace=ws)
            q_ms_per += events_ms(lambda: hqq.hqq_quantize_ex(W, params, out=q, workspace=ws))
            passes.append((q, m.rows, m.cols, params, m.dtype, torch.empty_like(W)))

        def dequantize_all():
            for q, rows, cols, params, dt, D in passes:
                hqq.hqq_dequantize_ex(q, rows, cols, params, out_dtype=dt, out=D)
        d_ms_per = graph_ms(dequantize_all)
        n = wl.weights
        nit = 2 * (wl.matrices[0].iters + 1)
        line = {"workload": wl.name, "weights": n}
        batched = len(wl.matrices) > 1 and not any(m.quant_meta for m in wl.matrices) and \
            all((m.nbits, m.group_size, m.axis, m.dtype) == (wl.matrices[0].nbits,
                wl.matrices[0].group_size, wl.matrices[0].axis, wl.matrices[0].dtype)
                for m in wl.matrices)
        if batched:
            p0 = plist[0]
            outs = hqq.hqq_quantize_batched(Ws, p0)
            qb = hqq.matrix_batch(Ws, outs)
            q_ms = events_ms(lambda: hqq.hqq_quantize_batched(Ws, p0, outs=outs, batch=qb))
            shapes = [tuple(W.shape) for W in Ws]
            Ds = [torch.empty_like(W) for W in Ws]
            db = hqq.matrix_batch(Ds, outs)
            d_ms = graph_ms(lambda: hqq.hqq_dequantize_batched(outs, shapes, p0, W_out=Ds,
                                                                batch=db))
            line["calls"] = "hqq_quantize_batched + hqq_dequantize_batched (one launch each)"
            del outs, Ds
        else:
            q_ms, d_ms = q_ms_per, d_ms_per
            line["calls"] = "hqq_quantize_ex + hqq_dequantize_ex per matrix"
        gbs = dq_bytes / (d_ms * 1e-3) / 1e9
        gbs_per = dq_bytes / (d_ms_per * 1e-3) / 1e9
        line.update({
            "quantize_ms": round(q_ms, 3), "quantize_Gweights_per_s": round(n / q_ms / 1e6, 2),
            "quantize_mufu_frac": round(nit * n / (q_ms * 1e-3) / mufu_peak, 4),
            "dequantize_ms": round(d_ms, 4), "dequantize_GB_per_s": round(gbs, 1),
            "dequantize_hbm_frac": round(gbs / pk["hbm_gbs"], 4),
            "per_matrix_quantize_mufu_frac": round(nit * n / (q_ms_per * 1e-3) / mufu_peak, 4),
            "per_matrix_dequantize_hbm_frac": round(gbs_per / pk["hbm_gbs"], 4),
            "dequantize_timing": "CUDA graph of one pass, L2 flushed before each replay"})
        out.append(line)
        del passes, Ws
        torch.cuda.empty_cache()
    return out


def run_mixed_model(args):
    """Per-layer mixed precision (row f1's per-matrix configurations): the whole Llama-7B-shaped
    model with block 0 at 8-bit g128, attention at 4-bit g64 and MLP at 2-bit g16
    (workloads.llama7b_model_mixed). A step is hqq_quantize_mixed over all 224 matrices (one
    batched solver launch per configuration) and hqq_dequantize_mixed back to bf16; CUDA events
    around each step on the launching stream; inputs 13 GB, above L2."""
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import workloads
    wl = workloads.llama7b_model_mixed()
    Ws = [workloads.make_weight(m, "cuda") for m in wl.matrices]
    cfgs = [hqq.make_params(m.nbits, m.group_size, m.axis, m.iters, m.p, m.beta0, m.kappa,
                            w_dtype=m.dtype) for m in wl.matrices]
    outs = hqq.hqq_quantize_mixed(Ws, cfgs)
    shapes = [tuple(W.shape) for W in Ws]
    D = hqq.hqq_dequantize_mixed(outs, shapes, cfgs)

    bq, bd = hqq.matrix_batch(Ws, outs), hqq.matrix_batch(D, outs)

    def step():
        hqq.hqq_quantize_mixed(Ws, cfgs, outs=outs, batch=bq)
        hqq.hqq_dequantize_mixed(outs, shapes, cfgs, W_out=D, batch=bd)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    per = []
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b))
    ms = statistics.median(per)
    groups = hqq.hqq_mixed_plan(cfgs)[1]
    counts = {}
    for m in wl.matrices:
        counts[f"{m.nbits}b_g{m.group_size}"] = counts.get(f"{m.nbits}b_g{m.group_size}", 0) + 1
    return {"metric": "HQQ quantize+dequantize Gweights/s, mixed per-layer configurations",
            "value": round(wl.weights / ms / 1e6, 3), "unit": "Gweights/s",
            "workload": wl.name, "weights": wl.weights, "matrices_per_config": counts,
            "ms_per_step": round(ms, 3), "launches_per_step": 2 * groups, "steps": args.steps}


# The single-matrix profiling cases: (rows, cols, dtype, nbits, group_size, axis). Each input
# is larger than the 126 MB L2 except the [4096, 1024] fp16 matrix of the single-layer workload.
SINGLE_CASES = {
    "quantize": (16384, 8192, "bf16", 4, 64, 1),
    "dequantize": (16384, 8192, "bf16", 4, 64, 1),
    "quantize_2b_g16_axis0": (16384, 8192, "bf16", 2, 16, 0),
    "quantize_1b_g32": (16384, 8192, "bf16", 1, 32, 1),
    "quantize_3b_g64": (16384, 8192, "bf16", 3, 64, 1),
    "quantize_fp16_4096x1024": (4096, 1024, "f16", 4, 64, 1),
    "dequantize_2b_g16_axis0": (16384, 8192, "bf16", 2, 16, 0),
}
# dequantize with 8-bit second-level scale/zero (runs of 128), the layouts of the 70B MLP
# workload's two matrices, on a [16384, 8192] bf16 weight
SINGLE_DEQ_META = {
    "dequantize_3b_g64_meta8": (16384, 8192, 3, 64),
    "dequantize_1b_g32_meta8": (16384, 8192, 1, 32),
}


def single_dequantize_block(reps: int = 10):
    """The batched dequantize launch of the bench step on one Llama-7B block (7 matrices,
    202M weights: 101 MB of codes and 6 MB of meta in, 405 MB of bf16 out): one launch, timed
    over `reps` launches after warm-up (the ncu case of the batched dequantizer)."""
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import workloads
    wl = workloads.llama7b_block_4b()
    Ws = [workloads.make_weight(m, "cuda") for m in wl.matrices]
    params = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16)
    outs = hqq.hqq_quantize_batched(Ws, params)
    shapes = [tuple(W.shape) for W in Ws]
    D = [torch.empty_like(W) for W in Ws]
    del Ws
    b = hqq.matrix_batch(D, outs)
    run = lambda: hqq.hqq_dequantize_batched(outs, shapes, params, W_out=D, batch=b)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    gbs = 2.5625 * wl.weights / (ms * 1e-3) / 1e9
    return {"single": "dequantize_block_batched", "weights": wl.weights, "ms": round(ms, 4),
            "GB_per_s_algorithmic": round(gbs, 1), "hbm_frac": round(gbs / peaks()["hbm_gbs"], 4)}


def single_dequantize_meta(kind: str, reps: int = 10):
    """One matrix of SINGLE_DEQ_META[kind], quantized with 8-bit scale and zero, dequantized to
    bf16 `reps` times after warm-up (hqq_dequantize_ex)."""
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import synthetic
    rows, cols, nbits, G = SINGLE_DEQ_META[kind]
    W = synthetic.weight(rows, cols, seed=5, dtype=torch.bfloat16, device="cuda")
    params = hqq.make_params(nbits, G, 1, w_dtype=torch.bfloat16, quant_scale=True,
                             quant_zero=True, meta_group_size=128)
    q = hqq.hqq_quantize_ex(W, params)
    D = torch.empty_like(W)
    for _ in range(2):
        hqq.hqq_dequantize_ex(q, rows, cols, params, out=D)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        hqq.hqq_dequantize_ex(q, rows, cols, params, out=D)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    n = rows * cols
    ng = n // G
    runs = -(-ng // 128)
    nbytes = hqq.hqq_packed_bytes(rows, cols, nbits) + 2 * ng + 2 * runs * 8 + 2 * n
    return {"single": kind, "shape": [rows, cols], "nbits": nbits, "group_size": G,
            "ms": round(ms, 4), "GB_per_s": round(nbytes / ms / 1e6, 1),
            "hbm_frac": round(nbytes / ms / 1e6 / peaks()["hbm_gbs"], 4)}


def single(kind: str, reps: int = 10):
    """One matrix of SINGLE_CASES[kind]: time `reps` solver or dequantize launches after
    warm-up (the cases the ncu captures in profiles/ use)."""
    import calibration_free_weight_hqq_b200 as hqq
    from calibration_free_weight_hqq_b200 import synthetic
    if kind in SINGLE_DEQ_META:
        return single_dequantize_meta(kind, reps)
    rows, cols, dt, nbits, G, axis = SINGLE_CASES[kind]
    dtype = torch.float16 if dt == "f16" else torch.bfloat16
    W = synthetic.weight(rows, cols, seed=5, dtype=dtype, device="cuda")
    pk, s, z = hqq.hqq_quantize(W, nbits, G, axis)
    D = torch.empty_like(W)
    run = (lambda: hqq.hqq_dequantize(pk, s, z, rows, cols, nbits, G, axis, out=D)) \
        if kind.startswith("dequantize") else \
        (lambda: hqq.hqq_quantize(W, nbits, G, axis, Wq_packed=pk, scale=s, zero=z))
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    n = rows * cols
    mufu = 2 * 21 * n / (ms * 1e-3) / (MUFU_PER_CLK_PER_SM * N_SM * SM_MAX_MHZ * 1e6)
    return {"single": kind, "shape": [rows, cols], "nbits": nbits, "group_size": G,
            "axis": axis, "ms": round(ms, 4), "Gweights_per_s": round(n / ms / 1e6, 2),
            "mufu_frac": round(mufu, 4) if not kind.startswith("dequantize") else None}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shard", action="store_true",
                    help="N>1: split one model's matrices over the ranks (strong scaling) "
                         "instead of one replica per rank (weak scaling, the default)")
    ap.add_argument("--per-matrix", action="store_true",
                    help="one launch per matrix instead of the batched whole-model calls")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-linear", action="store_true",
                    help="skip the fused 4-bit linear-layer measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--configs", action="store_true",
                    help="print only the four smaller configurations' lines and exit")
    ap.add_argument("--no-configs", action="store_true",
                    help="leave the four smaller configurations out of the JSON line")
    ap.add_argument("--mixed", action="store_true",
                    help="whole model with per-layer configurations (8/4/2 bits) and exit")
    ap.add_argument("--single", choices=sorted(SINGLE_CASES) + sorted(SINGLE_DEQ_META) +
                    ["dequantize_block_batched", "linear", "decode"],
                    help="time one matrix of a profiling case (SINGLE_CASES, SINGLE_DEQ_META), "
                         "one 4096^3 linear layer, or one 4096x4096 layer at 16 tokens, and exit")
    args = ap.parse_args()
    if args.configs:
        for line in configs_table():
            print(json.dumps(line), flush=True)
        return
    if args.mixed:
        print(json.dumps(run_mixed_model(args)), flush=True)
        return
    if args.single:
        if args.single in ("linear", "decode"):
            print(json.dumps(single_linear(M=4096 if args.single == "linear" else 16)), flush=True)
        elif args.single == "dequantize_block_batched":
            print(json.dumps(single_dequantize_block()), flush=True)
        else:
            print(json.dumps(single(args.single)), flush=True)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        res = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
