"""GPU <-> oracle comparison helpers for the parity tests, the smoke check and the bench.

The CUDA path is called through the C ABI (via the binding); the oracle runs on the host on
the same input bits (groups gathered on the device with plain tensor indexing and copied).
Nothing the GPU produces is ever passed to the oracle: GPU codes are read with np_unpack (a
numpy decoder of the header's layout, pinned on the CPU against the hand-derived layout
vectors); the near-tie rule asks the oracle for its own candidate zeros and its own codes at
them, and only compares the GPU's numbers against those. Packing and dequantization are
checked on inputs the test constructs itself (exact_grid_weights, dequant_parity).

Tolerances (stated once, used everywhere):
  scale           relative error <= 1e-5 (in practice bit-identical: it depends only on min/max)
  zero            |dz| <= 1e-5 * max(|z|, 1). A group outside that is a *near tie* only when
                  (a) the GPU's zero is bit-equal to one of the oracle's own candidate zeros
                  z_0 .. z_T of that group (the RTN zero and every updated zero), and
                  (b) that candidate's lp error and the oracle's best, both recomputed
                  independently in fp64, differ by no more than the sum of the error bounds
                  of the two sides' fp32 evaluations of sum|r|^p at the two candidates
                  (lp_eval_bound: the summation, the oracle's pow, and the GPU's MUFU
                  log2/exp2 at their documented accuracy), so either choice is a correct
                  result. The GPU's codes of a near-tie group are then compared with the
                  oracle's codes at that candidate (same +-1 budget as every other group).
                  Near ties are capped (near_tie_cap). Any other mismatch is *diverged*;
                  diverged groups must be <= 0.01 % of the groups.
  codes           <= 0.01 % of the codes differ, and only by +-1
  reconstruction  mean |W - W'| within 1e-4 relative of the oracle's
  second level    the 8-bit meta codes within the code budget; each run's (step2, zero2) pair
                  bit-exact whenever the run's first-level values agree bit for bit at its
                  minimum and maximum (the pair depends on nothing else)
  pack, dequant   bit-exact given the same codes, scale and zero: packing on weights whose
                  codes are known by construction (an exact grid), dequantization on codes,
                  scale and zero drawn by the test and packed by the oracle

Every comparison appends its counts to RECORDS; the test session prints them at the end.
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
# Near ties happen where two candidates' errors differ by less than the fp32 evaluation noise.
# For p < 1 the error is strictly concave between code changes and such coincidences are rare
# (<= 1.3e-4 of the groups on every workload measured); the cap is ten times that. For p = 1
# the L1 error is linear in z between code changes and flat wherever a group has as many
# positive as negative residuals, so candidates on a flat stretch tie exactly and only the
# summation order picks one (2.4 % of the groups measured); the cap is twice that.
NEAR_TIE_FRAC = 1e-3
NEAR_TIE_FRAC_P1 = 5e-2


def near_tie_cap(p: float) -> float:
    return NEAR_TIE_FRAC_P1 if p == 1.0 else NEAR_TIE_FRAC

RECORDS: list = []  # (label, Report) of every comparison in this process


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
    zero_off_not_candidate: int = 0   # diverged: the GPU's zero is none of the oracle's
    meta_runs_exact: int = 0          # second-level (step2, zero2) pairs checked bit for bit
    meta_runs_skipped: int = 0        # runs whose first-level min/max differ (not comparable)
    code_diff: int = 0
    code_maxdiff: int = 0
    recon_gpu: float = 0.0
    recon_oracle: float = 0.0
    meta_code_diff: int = 0
    meta_code_maxdiff: int = 0
    p: float = 0.7
    notes: list = field(default_factory=list)

    def summary(self) -> str:
        return (f"groups {self.n_groups}: zeros bit-exact {self.zero_exact}, near ties "
                f"{self.zero_near_tie}, diverged {self.zero_diverged}; codes off "
                f"{self.code_diff}/{self.n_codes} (max {self.code_maxdiff})")

    def check(self):
        assert self.scale_max_rel <= SCALE_RTOL, self
        assert self.zero_diverged <= GROUP_FRAC * self.n_groups, self
        assert self.zero_near_tie <= near_tie_cap(self.p) * self.n_groups, self
        assert self.meta_runs_skipped <= max(1, GROUP_FRAC * self.n_groups), self
        assert self.code_maxdiff <= 1, self
        assert self.code_diff <= CODE_FRAC * self.n_codes, self
        assert abs(self.recon_gpu - self.recon_oracle) <= RECON_RTOL * self.recon_oracle + 1e-30, self
        assert self.meta_code_maxdiff <= 1, self
        assert self.meta_code_diff <= CODE_FRAC * max(1, 2 * self.n_groups), self


def compare(W: torch.Tensor, nbits: int, G: int, axis: int, iters: int = 20, p: float = 0.7,
            beta0: float = 10.0, kappa: float = 1.01, n_sample: int | None = None, seed: int = 0,
            quant_meta: bool = False, meta_group: int = 128, label: str | None = None) -> Report:
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
    packed = out_plain["Wq_packed"].cpu().numpy()
    gc = unpack_groups(packed, ids, G, nbits, rows * cols)
    gs = out_plain["scale"].reshape(-1)[ids_t].cpu().numpy()
    gz = out_plain["zero"].reshape(-1)[ids_t].cpu().numpy()

    r, oc, os_, oz, oz_cmp, settled = judge(Wg, gc, gs, gz, nbits, iters, p, beta0, kappa)
    # reconstruction error: GPU (its dequant) vs oracle (its own codes and meta)
    od = oracle.dequantize(oc, os_, oz, ids.size, G, G, 1)
    r.recon_oracle = float(np.mean(np.abs(Wg.astype(np.float64) - od)))
    r.recon_gpu = float(np.mean(np.abs(Wg.astype(np.float64) - Dg)))

    if quant_meta:
        _compare_meta(r, out, ids, ids_t, gz, os_, oz_cmp, meta_group, settled)
    record(label, r)
    return r


def record(label: str | None, r: Report) -> None:
    """Keep the counts of one comparison for the end-of-session table."""
    if label is None:
        label = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    RECORDS.append((label, r))


def judge(Wg, gc, gs, gz, nbits: int, iters: int, p: float, beta0: float, kappa: float):
    """Compare the GPU's codes gc [n, G], scale gs and zero gz (fp32) of n groups with the
    oracle run on the same weights Wg [n, G] (fp32 values of the input).

    Returns (report, oracle codes, oracle scale, oracle zero, the oracle's zero each GPU zero
    is judged against - its best, or for a near tie the candidate the GPU returned - and the
    mask of groups whose zero is the oracle's or a near tie)."""
    n, G = Wg.shape
    r = Report(n_groups=n, n_codes=n * G, p=p)
    oc, os_, oz = oracle.quantize(Wg, nbits, G, 1, iters, p, beta0, kappa, nthreads=n_threads())
    rel_s = np.abs(gs.astype(np.float64) - os_) / np.maximum(np.abs(os_.astype(np.float64)), 1e-30)
    r.scale_max_rel = float(rel_s.max()) if rel_s.size else 0.0
    r.scale_exact = int(np.sum(gs.view(np.uint32) == os_.view(np.uint32)))
    dz = np.abs(gz.astype(np.float64) - oz) / np.maximum(np.abs(oz.astype(np.float64)), 1.0)
    r.zero_exact = int(np.sum(gz.view(np.uint32) == oz.view(np.uint32)))
    oc_cmp = oc.copy()
    oz_cmp = oz.copy()
    settled = dz <= ZERO_RTOL
    for i in np.nonzero(~settled)[0]:
        og = oracle.quantize_group(Wg[i], nbits, iters, p, beta0, kappa)
        cand = np.nonzero(og["z_trace"].view(np.uint32) == np.float32(gz[i]).view(np.uint32))[0]
        if cand.size == 0:
            r.zero_off_not_candidate += 1
            continue
        zk = og["z_trace"][cand[0]]
        e_k, b_k = lp_error64(Wg[i], zk, os_[i], nbits, p, with_bound=True)
        e_b, b_b = lp_error64(Wg[i], oz[i], os_[i], nbits, p, with_bound=True)
        if abs(e_k - e_b) <= b_k + b_b:
            r.zero_near_tie += 1
            settled[i] = True
            oc_cmp[i] = oracle.codes_at_zero(Wg[i], nbits, zk)  # the oracle's codes there
            oz_cmp[i] = zk
        elif len(r.notes) < 4:  # what a failure report needs to reproduce the case
            kb = np.nonzero(og["z_trace"].view(np.uint32) == np.float32(oz[i]).view(np.uint32))[0]
            r.notes.append(dict(k=int(cand[0]), b=int(kb[0]) if kb.size else -1, e64_k=e_k,
                                e64_b=e_b, bound=b_k + b_b,
                                e32_trace=og["e_trace"].tolist(), w=Wg[i].tolist()))
    r.zero_diverged = int(np.count_nonzero(~settled))
    cd = np.abs(gc.astype(np.int32) - oc_cmp.astype(np.int32))
    r.code_diff = int(np.count_nonzero(cd))
    r.code_maxdiff = int(cd.max()) if cd.size else 0
    return r, oc, os_, oz, oz_cmp, settled


def lp_error64(w, z, step, nbits, p, with_bound: bool = False):
    """sum_j |w_j - (Q_j - z)*step|^p in fp64, with the codes Q_j and the residuals r_j
    decided in fp32 exactly as the definition decides them (an independent recomputation, not
    the oracle's code). With `with_bound`, also lp_eval_bound of the same residuals."""
    w = np.asarray(w, np.float32)
    qmax = np.float32(2 ** nbits - 1)
    mn, mx = w.min(), w.max()
    s = np.float32(qmax / (mx - mn)) if mx > mn else np.float32(1)
    z32 = np.float32(z)
    q = np.clip(np.rint((w * s).astype(np.float32) + z32), 0, qmax).astype(np.float32)
    r = (w - ((q - z32).astype(np.float32) * np.float32(step)).astype(np.float32)).astype(np.float32)
    a = np.abs(r.astype(np.float64))
    e = float(np.sum(a ** p))
    if not with_bound:
        return e
    return e, lp_eval_bound(a, p)


U = 2.0 ** -24  # unit roundoff of fp32


def _ulp32(x):
    """Spacing of fp32 numbers at |x| (for |x| >= 2^-126)."""
    x = np.abs(np.asarray(x, np.float64))
    return 2.0 ** (np.floor(np.log2(np.maximum(x, 2.0 ** -126))) - 23)


def lp_eval_bound(a, p):
    """Bound on |e_fp32 - sum a_j^p| for either side's fp32 evaluation of the lp error of
    residual magnitudes a_j (fp64 array):
      - the fp32 summation of G non-negative terms: (G - 1) u of the sum (any order);
      - the oracle's term a * a^(p-1): the power rounded once, then a product: 2 u per term;
      - the GPU's term exp2(p * log2 a) on the MUFU approximations, at their documented
        accuracy: log2 within 2 ulp of its result (an absolute 2^-22 for a in [0.5, 2]),
        the product p * log2 a rounded (half an ulp), exp2 within 2 ulp - the first two are
        absolute errors d of the exponent, a relative error ln2 * d of the term.
    The larger of the two sides' term errors is taken, plus one u for the term's own
    fp32 rounding."""
    a = np.asarray(a, np.float64)
    a = a[a > 0]
    if a.size == 0:
        return 0.0
    t = a ** p
    L = np.log2(a)
    d_lg2 = np.where((a >= 0.5) & (a <= 2.0), 2.0 ** -22, 2.0 * _ulp32(L))
    d_exp = p * d_lg2 + 0.5 * _ulp32(p * L)
    rel_gpu = np.log(2.0) * d_exp + 2.0 * 2.0 * U
    rel = np.maximum(rel_gpu, 2.0 * U) + U
    return float(np.sum(t * rel) + (a.size - 1) * U * np.sum(t))


def _compare_meta(r, out, ids, ids_t, gz, os_, oz, meta_group, settled):
    """Second level: runs of meta_group consecutive groups; the sample holds whole runs.
    `oz` holds, per group, the oracle's zero the GPU's is judged against (for a near tie, the
    oracle's candidate that the GPU returned), and the oracle's second level runs on those.
    The 8-bit codes of scale and zero go into the code budget (a group whose first-level zero
    diverged is not counted again for its zero's code). A run's (step2, zero2) pair depends
    only on the minimum and maximum of its first-level values: it must be bit-exact whenever
    those agree bit for bit with the oracle's (always for the scale; for the zero unless a
    diverged group moved an extreme), and such runs are counted."""
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
        d2[~settled[pos:pos + k]] = 0
        diffs.append(np.count_nonzero(d1) + np.count_nonzero(d2))
        maxd = max(maxd, int(d1.max()), int(d2.max()))
        # the scale run pair depends only on the scale min/max, which are exact: bit-exact
        assert np.array_equal(mm_s[0].view(np.uint32), smm[run].view(np.uint32)), run
        r.meta_runs_exact += 1
        zg, zo = gz[pos:pos + k], oz[pos:pos + k]
        if zg.min() == zo.min() and zg.max() == zo.max():
            assert np.array_equal(mm_z[0].view(np.uint32), zmm[run].view(np.uint32)), run
            r.meta_runs_exact += 1
        else:
            r.meta_runs_skipped += 1
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
                   seed: int = 0, one_sided: str | None = None) -> None:
    """hqq_dequantize_ex against the oracle's dequantize on codes, scale and zero drawn here
    (packed by the oracle; with quant_meta, 8-bit meta codes and run pairs drawn here and
    decoded by the oracle's dequantize_meta): bit-exact after one rounding to out_dtype.
    one_sided = "scale" or "zero": only that side is second-level, the other is stored in
    meta_dtype."""
    rng = np.random.default_rng(seed)
    qmax = 2 ** nbits - 1
    ng = rows * cols // G
    codes = rng.integers(0, qmax + 1, size=rows * cols).astype(np.uint8)
    packed = torch.from_numpy(oracle.pack(codes, nbits)).cuda()
    if one_sided is not None:
        runs = (ng + meta_group - 1) // meta_group
        qs = rng.integers(0, 256, size=ng).astype(np.uint8)
        smm = np.stack([rng.random(runs) * 1e-4 + 1e-6, rng.random(runs) * 10], 1).astype(np.float32)
        plain_s = oracle.round_to_dtype((rng.random(ng) * 0.02 + 1e-4).astype(np.float32), meta_dtype)
        plain_z = oracle.round_to_dtype((rng.random(ng) * qmax).astype(np.float32), meta_dtype)
        params = hqq.make_params(nbits, G, axis, w_dtype=torch.bfloat16,
                                 meta_dtype=TORCH_OF[meta_dtype],
                                 quant_scale=one_sided == "scale", quant_zero=one_sided == "zero",
                                 meta_group_size=meta_group)
        q8 = torch.from_numpy(qs).cuda()
        mm = torch.from_numpy(smm).cuda()
        if one_sided == "scale":
            scale, zero = oracle.dequantize_meta(qs, smm, meta_group), plain_z
            out = {"Wq_packed": packed, "scale": q8, "scale_mm": mm, "zero_mm": None,
                   "zero": torch.from_numpy(plain_z).to(TORCH_OF[meta_dtype]).cuda()}
        else:
            scale, zero = plain_s, oracle.dequantize_meta(qs, smm, meta_group)
            out = {"Wq_packed": packed, "zero": q8, "zero_mm": mm, "scale_mm": None,
                   "scale": torch.from_numpy(plain_s).to(TORCH_OF[meta_dtype]).cuda()}
        D = hqq.hqq_dequantize_ex(out, rows, cols, params, out_dtype=TORCH_OF[out_dtype])
        torch.cuda.synchronize()
        want = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, rows, cols, G, axis),
                                     out_dtype)
        got = D.float().cpu().numpy()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), \
            np.flatnonzero(got != want)[:8]
        return
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
