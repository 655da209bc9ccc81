"""GPU <-> oracle comparison helpers for the parity tests, the smoke check and the bench.

The CUDA path is called through the C ABI (via the binding); the oracle runs on the host on
the same input bits (groups gathered on the device with plain tensor indexing and copied).
Nothing the GPU produces is ever passed to the oracle: GPU codes are read with np_unpack (a
numpy decoder of the header's layout, pinned on the CPU against the hand-derived layout
vectors), and the near-tie rule recomputes the definition's codes at the GPU's zero in numpy.
Packing and dequantization are checked on inputs the test constructs itself
(exact_grid_weights, dequant_parity).

Tolerances (stated once, used everywhere):
  scale           relative error <= 1e-5 (in practice bit-identical: it depends only on min/max)
  zero            |dz| <= 1e-5 * max(|z|, 1). A group outside that is a *near tie* when the
                  lp errors of the two candidate zeros, recomputed independently in fp64,
                  agree within 2*(G+8)*2^-24 relative - the most two correct fp32
                  evaluations of sum|r|^p can differ by (G-1 roundings of the sum, one of the
                  term, the pow error), so either choice is a correct result; its codes must
                  then be exactly the definition's codes at the GPU's zero. Any other
                  mismatch is *diverged*; diverged groups must be <= 0.01 % of the groups.
  codes           <= 0.01 % of the codes of non-near-tie groups differ, and only by +-1
  reconstruction  mean |W - W'| within 1e-4 relative of the oracle's
  pack, dequant   bit-exact given the same codes, scale and zero: packing on weights whose
                  codes are known by construction (an exact grid), dequantization on codes,
                  scale and zero drawn by the test and packed by the oracle
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field

import numpy as np
import torch

import calibration_free_weight_hqq_b200 as hqq
import oracle

ZERO_RTOL = 1e-5
SCALE_RTOL = 1e-5
CODE_FRAC = 1e-4
GROUP_FRAC = 1e-4
RECON_RTOL = 1e-4


def n_threads() -> int:
    return oracle.default_threads()


def group_view(W: torch.Tensor, G: int, axis: int) -> torch.Tensor:
    """[n_groups, G] view/copy of W in group order (plain indexing, no arithmetic)."""
    rows, cols = W.shape
    if axis == 1:
        return W.reshape(rows * cols // G, G)
    return W.reshape(rows // G, G, cols).permute(0, 2, 1).reshape(rows // G * cols, G)


def sample_groups(n_groups: int, n_sel: int, seed: int, runs_of: int = 1) -> np.ndarray:
    """Seeded sample of group ids (sorted, unique) that always contains the first and the
    last groups (ragged tail). With runs_of > 1 whole runs of that many consecutive groups
    are taken (for the second-level quantization, which works on runs)."""
    if n_sel >= n_groups:
        return np.arange(n_groups, dtype=np.int64)
    rng = np.random.default_rng(seed)
    if runs_of > 1:
        n_runs = (n_groups + runs_of - 1) // runs_of
        k = max(2, n_sel // runs_of)
        runs = set(rng.choice(n_runs, min(k, n_runs), replace=False).tolist()) | {0, n_runs - 1}
        ids = np.concatenate([np.arange(r * runs_of, min((r + 1) * runs_of, n_groups))
                              for r in sorted(runs)])
        return ids.astype(np.int64)
    ids = set(rng.choice(n_groups, n_sel, replace=False).tolist())
    ids |= set(range(min(8, n_groups))) | set(range(max(0, n_groups - 200), n_groups))
    return np.array(sorted(ids), dtype=np.int64)


def np_unpack(packed, n: int, nbits: int) -> np.ndarray:
    """Codes 0..n-1 of a packed stream in the header's layout, decoded with numpy (test-side
    reader of GPU output; independent of the oracle): 8/4/2/1 bits LSB-first in bytes, 3 bits
    10 per little-endian 32-bit word."""
    pk = np.ascontiguousarray(np.asarray(packed, np.uint8).ravel())
    k = np.arange(n, dtype=np.int64)
    if nbits == 3:
        words = pk[:4 * ((n + 9) // 10)].view("<u4").astype(np.int64)
        return ((words[k // 10] >> (3 * (k % 10))) & 7).astype(np.uint8)
    per = 8 // nbits
    return ((pk[k // per].astype(np.int64) >> ((k % per) * nbits)) & ((1 << nbits) - 1)).astype(np.uint8)


def codes_at_zero_np(w, nbits: int, zero) -> np.ndarray:
    """The definition's final codes of one group at a given zero, recomputed in numpy fp32
    (clamp(rint(w*s + zero), 0, qmax) with s = qmax/(max-min), or 1 for a constant group)."""
    w = np.asarray(w, np.float32)
    qmax = np.float32(2 ** nbits - 1)
    mn, mx = w.min(), w.max()
    s = np.float32(qmax / (mx - mn)) if mx > mn else np.float32(1)
    return np.clip(np.rint((w * s).astype(np.float32) + np.float32(zero)), 0, qmax).astype(np.uint8)


def unpack_groups(packed: np.ndarray, ids: np.ndarray, G: int, nbits: int, n_codes: int):
    """GPU codes of the selected groups -> [n_sel, G] (numpy reader)."""
    if nbits == 3:
        return np_unpack(packed, n_codes, 3).reshape(-1, G)[ids]
    per = G * nbits // 8  # whole bytes per group for 8/4/2/1 bits and G >= 8
    pk = packed.reshape(-1, per)[ids]
    return np_unpack(pk.ravel(), ids.size * G, nbits).reshape(-1, G)


@dataclass
class Report:
    n_groups: int = 0
    n_codes: int = 0
    scale_exact: int = 0
    scale_max_rel: float = 0.0
    zero_exact: int = 0
    zero_near_tie: int = 0
    zero_diverged: int = 0
    code_diff: int = 0
    code_maxdiff: int = 0
    recon_gpu: float = 0.0
    recon_oracle: float = 0.0
    meta_code_diff: int = 0
    meta_code_maxdiff: int = 0
    notes: list = field(default_factory=list)

    def check(self):
        assert self.scale_max_rel <= SCALE_RTOL, self
        assert self.zero_diverged <= GROUP_FRAC * self.n_groups, self
        assert self.code_maxdiff <= 1, self
        assert self.code_diff <= CODE_FRAC * self.n_codes, self
        assert abs(self.recon_gpu - self.recon_oracle) <= RECON_RTOL * self.recon_oracle + 1e-30, self
        assert self.meta_code_maxdiff <= 1, self
        assert self.meta_code_diff <= CODE_FRAC * max(1, 2 * self.n_groups), self


def compare(W: torch.Tensor, nbits: int, G: int, axis: int, iters: int = 20, p: float = 0.7,
            beta0: float = 10.0, kappa: float = 1.01, n_sample: int | None = None, seed: int = 0,
            quant_meta: bool = False, meta_group: int = 128) -> Report:
    """Quantize W (CUDA) through the C ABI with fp32 meta, run the oracle on the same groups
    (all of them, or a seeded sample), and fill a Report."""
    rows, cols = W.shape
    ng = rows * cols // G
    params = hqq.make_params(nbits, G, axis, iters, p, beta0, kappa, w_dtype=W.dtype,
                             meta_dtype=torch.float32, quant_scale=quant_meta,
                             quant_zero=quant_meta, meta_group_size=meta_group)
    out = hqq.hqq_quantize_ex(W, params)
    deq = hqq.hqq_dequantize_ex(out, rows, cols, params, out_dtype=torch.float32)
    # unquantized meta of the same run, for the first-level comparison
    plain = hqq.make_params(nbits, G, axis, iters, p, beta0, kappa, w_dtype=W.dtype,
                            meta_dtype=torch.float32)
    out_plain = hqq.hqq_quantize_ex(W, plain) if quant_meta else out
    deq_plain = hqq.hqq_dequantize_ex(out_plain, rows, cols, plain, out_dtype=torch.float32) \
        if quant_meta else deq
    torch.cuda.synchronize()

    ids = sample_groups(ng, n_sample if n_sample else ng, seed,
                        runs_of=meta_group if quant_meta else 1)
    ids_t = torch.from_numpy(ids).to(W.device)
    Wg = group_view(W, G, axis)[ids_t].float().cpu().numpy()
    Dg = group_view(deq_plain, G, axis)[ids_t].cpu().numpy()

    r = Report(n_groups=ids.size, n_codes=ids.size * G)
    oc, os_, oz = oracle.quantize(Wg, nbits, G, 1, iters, p, beta0, kappa, nthreads=n_threads())
    packed = out_plain["Wq_packed"].cpu().numpy()
    gc = unpack_groups(packed, ids, G, nbits, rows * cols)
    gs = out_plain["scale"].reshape(-1)[ids_t].cpu().numpy()
    gz = out_plain["zero"].reshape(-1)[ids_t].cpu().numpy()

    rel_s = np.abs(gs.astype(np.float64) - os_) / np.maximum(np.abs(os_.astype(np.float64)), 1e-30)
    r.scale_max_rel = float(rel_s.max()) if rel_s.size else 0.0
    r.scale_exact = int(np.sum(gs.view(np.uint32) == os_.view(np.uint32)))
    dz = np.abs(gz.astype(np.float64) - oz) / np.maximum(np.abs(oz.astype(np.float64)), 1.0)
    r.zero_exact = int(np.sum(gz.view(np.uint32) == oz.view(np.uint32)))
    off = np.nonzero(dz > ZERO_RTOL)[0]
    tie_rtol = 2.0 * (G + 8) * 2.0 ** -24
    oc_cmp = oc.copy()
    diverged = np.zeros(ids.size, bool)
    for i in off:
        e_g = lp_error64(Wg[i], gz[i], gs[i], nbits, p)
        e_o = lp_error64(Wg[i], oz[i], os_[i], nbits, p)
        if abs(e_g - e_o) <= tie_rtol * max(e_o, 1e-300):
            r.zero_near_tie += 1
            assert np.array_equal(gc[i], codes_at_zero_np(Wg[i], nbits, gz[i])), i
            oc_cmp[i] = gc[i]  # the GPU's alternative is judged by its own (exact) codes
        else:
            diverged[i] = True
    r.zero_diverged = int(diverged.sum())
    cd = np.abs(gc.astype(np.int32) - oc_cmp.astype(np.int32))
    r.code_diff = int(np.count_nonzero(cd))
    r.code_maxdiff = int(cd.max()) if cd.size else 0

    # reconstruction error: GPU (its dequant) vs oracle (its own codes and meta)
    od = oracle.dequantize(oc, os_, oz, ids.size, G, G, 1)
    r.recon_oracle = float(np.mean(np.abs(Wg.astype(np.float64) - od)))
    r.recon_gpu = float(np.mean(np.abs(Wg.astype(np.float64) - Dg)))

    if quant_meta:
        _compare_meta(r, out, deq, ids, ids_t, os_, oz, G, axis, meta_group, nbits, gc,
                      rows, cols, diverged=dz > ZERO_RTOL)
    return r


def lp_error64(w, z, step, nbits, p):
    """sum_j |w_j - (Q_j - z)*step|^p in fp64, with the codes Q_j decided in fp32 exactly as
    the definition decides them (an independent recomputation, not the oracle's code)."""
    w = np.asarray(w, np.float32)
    qmax = np.float32(2 ** nbits - 1)
    mn, mx = w.min(), w.max()
    s = np.float32(qmax / (mx - mn)) if mx > mn else np.float32(1)
    q = np.clip(np.rint((w * s).astype(np.float32) + np.float32(z)), 0, qmax).astype(np.float64)
    res = w.astype(np.float64) - (q - np.float64(z)) * np.float64(step)
    return float(np.sum(np.abs(res) ** p))


def _compare_meta(r, out, deq, ids, ids_t, os_, oz, G, axis, meta_group, nbits, gc, rows, cols,
                  diverged):
    """Second level: runs of meta_group consecutive groups; the sample holds whole runs.
    A group whose first-level zero already diverged (counted above) is not counted again
    for its zero's 8-bit code."""
    qs_g = out["scale"].reshape(-1)[ids_t].cpu().numpy()
    qz_g = out["zero"].reshape(-1)[ids_t].cpu().numpy()
    smm = out["scale_mm"].cpu().numpy()
    zmm = out["zero_mm"].cpu().numpy()
    diffs = []
    maxd = 0
    run_ids = np.unique(ids // meta_group)
    pos = 0
    for run in run_ids:
        sel = ids[(ids >= run * meta_group) & (ids < (run + 1) * meta_group)]
        k = sel.size
        q_s, mm_s = oracle.quantize_meta(os_[pos:pos + k], meta_group)
        q_z, mm_z = oracle.quantize_meta(oz[pos:pos + k], meta_group)
        d1 = np.abs(q_s.astype(int) - qs_g[pos:pos + k].astype(int))
        d2 = np.abs(q_z.astype(int) - qz_g[pos:pos + k].astype(int))
        d2[diverged[pos:pos + k]] = 0
        diffs.append(np.count_nonzero(d1) + np.count_nonzero(d2))
        maxd = max(maxd, int(d1.max()), int(d2.max()))
        # the scale run parameters depend only on scale min/max: exact
        assert np.array_equal(mm_s[0].view(np.uint32), smm[run].view(np.uint32))
        pos += k
    r.meta_code_diff = int(sum(diffs))
    r.meta_code_maxdiff = maxd


# ------------------------------------------------------------------ independent constructions

TORCH_OF = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def exact_grid_weights(rows: int, cols: int, nbits: int, G: int, axis: int, seed: int,
                       dtype=torch.bfloat16):
    """Weights whose quantization is known by construction: every group is
    (q - z) * 2^-k with random codes q (each group holds 0 and qmax), an integer zero z in
    [0, qmax] and a power-of-two step 2^-k. Min/max RTN then reproduces step, zero and codes
    exactly, the residual is 0 at iteration 0 (the best), and every zero update returns z.
    Returns (W on the device, codes in stream order, step per group, zero per group)."""
    rng = np.random.default_rng(seed)
    qmax = 2 ** nbits - 1
    ng = rows * cols // G
    q = rng.integers(0, qmax + 1, size=(ng, G))
    q[:, 0], q[:, 1] = 0, qmax
    for g in range(ng):
        rng.shuffle(q[g])
    z = rng.integers(0, qmax + 1, size=ng)
    k = rng.integers(2, 12, size=ng)
    step = (2.0 ** -k).astype(np.float32)
    vals = ((q - z[:, None]) * step[:, None]).astype(np.float32)  # exact in bf16 (|q-z| < 256)
    if axis == 1:
        Wn = vals.reshape(rows, cols)
    else:
        Wn = vals.reshape(rows // G, cols, G).transpose(0, 2, 1).reshape(rows, cols)
    W = torch.from_numpy(np.ascontiguousarray(Wn)).to(dtype).cuda()
    assert np.array_equal(W.float().cpu().numpy(), Wn)  # the construction is exact in dtype
    return W, q.astype(np.uint8).ravel(), step, z.astype(np.float32)


def dequant_parity(rows: int, cols: int, nbits: int, G: int, axis: int, out_dtype: str,
                   meta_dtype: str = "f32", quant_meta: bool = False, meta_group: int = 128,
                   seed: int = 0) -> None:
    """hqq_dequantize_ex against the oracle's dequantize on codes, scale and zero drawn here
    (packed by the oracle; with quant_meta, 8-bit meta codes and run pairs drawn here and
    decoded by the oracle's dequantize_meta): bit-exact after one rounding to out_dtype."""
    rng = np.random.default_rng(seed)
    qmax = 2 ** nbits - 1
    ng = rows * cols // G
    codes = rng.integers(0, qmax + 1, size=rows * cols).astype(np.uint8)
    packed = torch.from_numpy(oracle.pack(codes, nbits)).cuda()
    params = hqq.make_params(nbits, G, axis, w_dtype=torch.bfloat16,
                             meta_dtype=TORCH_OF[meta_dtype], quant_scale=quant_meta,
                             quant_zero=quant_meta, meta_group_size=meta_group)
    if quant_meta:
        runs = (ng + meta_group - 1) // meta_group
        qs = rng.integers(0, 256, size=ng).astype(np.uint8)
        qz = rng.integers(0, 256, size=ng).astype(np.uint8)
        smm = np.stack([rng.random(runs) * 1e-4 + 1e-6, rng.random(runs) * 10], 1).astype(np.float32)
        zmm = np.stack([rng.random(runs) * 0.1 + 1e-3, rng.random(runs) * 20], 1).astype(np.float32)
        scale = oracle.dequantize_meta(qs, smm, meta_group)
        zero = oracle.dequantize_meta(qz, zmm, meta_group)
        out = {"Wq_packed": packed, "scale": torch.from_numpy(qs).cuda(),
               "zero": torch.from_numpy(qz).cuda(), "scale_mm": torch.from_numpy(smm).cuda(),
               "zero_mm": torch.from_numpy(zmm).cuda()}
    else:
        scale = oracle.round_to_dtype((rng.random(ng) * 0.02 + 1e-4).astype(np.float32), meta_dtype)
        zero = oracle.round_to_dtype((rng.random(ng) * qmax).astype(np.float32), meta_dtype)
        out = {"Wq_packed": packed, "scale": torch.from_numpy(scale).to(TORCH_OF[meta_dtype]).cuda(),
               "zero": torch.from_numpy(zero).to(TORCH_OF[meta_dtype]).cuda()}
    D = hqq.hqq_dequantize_ex(out, rows, cols, params, out_dtype=TORCH_OF[out_dtype])
    torch.cuda.synchronize()
    want = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, rows, cols, G, axis),
                                 out_dtype)
    got = D.float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), \
        np.flatnonzero(got != want)[:8]
