"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a closed form, an invariant, a special case that
reduces to a textbook routine, a library routine, a hand-derived vector or brute force on
tiny inputs, chosen so that a plausible mistake (a dropped term, a wrong sign or index, a
transposed operand, a wrong error metric) fails at least one of them. No GPU needed.

Definition being pinned (the pages give no equations; see the oracle's header for the
readings R1-R10): min/max RTN init, iters+1 candidate zeros scored by the lp error
sum |r|^p, lp generalised soft-threshold of the residual, closed-form mean zero update,
beta *= kappa, earliest best candidate kept.
"""
from fractions import Fraction
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def rtn_fp32(w, nbits):
    """Textbook asymmetric min/max round-to-nearest quantizer, in numpy fp32."""
    w = np.asarray(w, F32)
    qmax = F32(2 ** nbits - 1)
    mn, mx = w.min(), w.max()
    if mx > mn:
        s, step = F32(qmax / (mx - mn)), F32((mx - mn) / qmax)
    else:
        s, step = F32(1), F32(1)
    z = F32(-mn * s)
    q = np.clip(np.rint((w * s).astype(F32) + z), 0, qmax).astype(np.uint8)
    return q, step, z, s


def lp_error64(w, z, nbits, p):
    """lp error of the candidate zero z, in fp64 from the fp32 codes (codes decided in fp32
    exactly as the definition does; the error itself summed in fp64)."""
    w = np.asarray(w, F32)
    _, step, _, s = rtn_fp32(w, nbits)
    qmax = F32(2 ** nbits - 1)
    q = np.clip(np.rint((w * s).astype(F32) + F32(z)), 0, qmax).astype(np.float64)
    r = w.astype(np.float64) - (q - np.float64(z)) * np.float64(step)
    return float(np.sum(np.abs(r) ** p))


def rand_groups(rng, n, G, outliers=True):
    sig = 0.02 * np.exp(0.3 * rng.standard_normal((n, 1)))
    w = rng.standard_normal((n, G)) * sig
    if outliers:
        m = rng.random((n, G)) < 0.02
        w = np.where(m, w * rng.uniform(5, 20, (n, G)) * np.sign(rng.random((n, G)) - 0.5), w)
    return w.astype(F32)


PARAMS = dict(p=0.7, beta0=10.0, kappa=1.01)


# ---------------------------------------------------------------- RTN / iteration 0


@pytest.mark.parametrize("nbits,G", [(8, 64), (4, 64), (3, 64), (2, 16), (1, 32), (4, 128)])
def test_iters0_equals_textbook_rtn(nbits, G):
    rng = np.random.default_rng(nbits * 1000 + G)
    W = rand_groups(rng, 200, G)
    codes, scale, zero = oracle.quantize(W, nbits, G, 1, 0, **PARAMS)
    for i in range(W.shape[0]):
        q, step, z, _ = rtn_fp32(W[i], nbits)
        assert np.array_equal(codes[i], q)
        assert scale[i] == step and zero[i] == z


def test_scale_does_not_depend_on_iterations():
    rng = np.random.default_rng(1)
    W = rand_groups(rng, 300, 64)
    _, s0, _ = oracle.quantize(W, 4, 64, 1, 0, **PARAMS)
    _, s20, _ = oracle.quantize(W, 4, 64, 1, 20, **PARAMS)
    assert np.array_equal(s0.view(np.uint32), s20.view(np.uint32))


def test_trace_starts_at_rtn_and_has_iters_plus_one_candidates():
    rng = np.random.default_rng(2)
    w = rand_groups(rng, 1, 64)[0]
    out = oracle.quantize_group(w, 4, 7, **PARAMS)
    assert out["z_trace"].shape == (8,)
    assert out["z_trace"][0] == rtn_fp32(w, 4)[2]


# ---------------------------------------------------------------- invariants


@pytest.mark.parametrize("nbits,G", [(8, 64), (4, 64), (3, 64), (2, 16), (1, 32), (1, 8)])
def test_codes_in_range(nbits, G):
    rng = np.random.default_rng(3 + nbits)
    W = rand_groups(rng, 500, G)
    codes, _, _ = oracle.quantize(W, nbits, G, 1, 20, **PARAMS)
    assert codes.max() <= 2 ** nbits - 1


@pytest.mark.parametrize("nbits,G", [(4, 64), (3, 64), (2, 16), (1, 32), (2, 8)])
def test_best_error_not_worse_than_rtn(nbits, G):
    """Best tracking: e(z_best) <= e(z_RTN), both recomputed independently in fp64."""
    rng = np.random.default_rng(10 + nbits)
    W = rand_groups(rng, 400, G)
    _, _, zero = oracle.quantize(W, nbits, G, 1, 20, **PARAMS)
    improved = 0
    for i in range(W.shape[0]):
        z_rtn = rtn_fp32(W[i], nbits)[2]
        e_best = lp_error64(W[i], zero[i], nbits, 0.7)
        e_rtn = lp_error64(W[i], z_rtn, nbits, 0.7)
        assert e_best <= e_rtn * (1 + 1e-5) + 1e-30
        improved += e_best < e_rtn * (1 - 1e-4)
    assert improved > 0.1 * W.shape[0]  # the solver does move the zero


@pytest.mark.parametrize("nbits,G,p", [(4, 64, 0.7), (2, 16, 0.7), (3, 32, 0.5), (4, 64, 1.0)])
def test_error_trace_is_lp_error_and_best_is_its_argmin(nbits, G, p):
    """e_k equals sum|r|^p of the k-th candidate (fp64 recomputation, pins the metric and
    the residual), and the returned zero is the first argmin over the candidates."""
    rng = np.random.default_rng(20 + nbits)
    W = rand_groups(rng, 60, G)
    for w in W:
        out = oracle.quantize_group(w, nbits, 20, p, 10.0, 1.01)
        e64 = np.array([lp_error64(w, z, nbits, p) for z in out["z_trace"]])
        # fp32 residuals carry a few ulps of max|w| of rounding; |a^p - b^p| <= |a - b|^p
        atol = G * (8 * np.finfo(F32).eps * float(np.abs(w).max())) ** p
        np.testing.assert_allclose(out["e_trace"], e64, rtol=2e-5, atol=atol)
        k = int(np.argmin(out["e_trace"]))
        assert out["zero"] == out["z_trace"][k]
        assert lp_error64(w, out["zero"], nbits, p) <= e64.min() * (1 + 2e-5) + 2 * atol


def test_eight_bit_reconstruction_bound():
    """8 bits: |w - W'| <= step/2 (up to fp32 rounding of the operands) for every element
    at iters=0 and for every unclamped element after solving."""
    rng = np.random.default_rng(30)
    G = 64
    W = rand_groups(rng, 300, G)
    eps = np.finfo(F32).eps
    for iters in (0, 20):
        codes, scale, zero = oracle.quantize(W, 8, G, 1, iters, **PARAMS)
        Wd = oracle.dequantize(codes, scale, zero, W.shape[0], G, G, 1)
        for i in range(W.shape[0]):
            _, step, _, s = rtn_fp32(W[i], 8)
            v = (W[i] * s).astype(F32) + zero[i]
            ok = (v > 0) & (v < 255) if iters else np.ones(G, bool)
            bound = step / 2 * (1 + 1e-5) + 8 * eps * np.abs(W[i]).max()
            assert np.all(np.abs(W[i] - Wd[i])[ok] <= bound)


def test_constant_group():
    """max == min: s = step = 1, zero = -min, every code 0, exact reconstruction."""
    w = np.full(64, 0.3, F32)
    out = oracle.quantize_group(w, 4, 20, **PARAMS)
    assert np.all(out["codes"] == 0) and out["scale"] == 1 and out["zero"] == F32(-0.3)
    Wd = oracle.dequantize(out["codes"], [out["scale"]], [out["zero"]], 1, 64, 64, 1)
    assert np.all(Wd == w)


@pytest.mark.parametrize("offset,zero", [(0.0, 0.0), (-1.0, 2.0)])
def test_exact_grid_group(offset, zero):
    """w_j = j/2 + offset, 4 bits, 16 values: s = 2, step = 1/2, codes 0..15, no residual,
    the zero never moves (closed form)."""
    w = (np.arange(16) * 0.5 + offset).astype(F32)
    out = oracle.quantize_group(w, 4, 20, **PARAMS)
    assert np.array_equal(out["codes"], np.arange(16))
    assert out["scale"] == 0.5 and out["zero"] == zero and out["best_err"] == 0


# ---------------------------------------------------------------- shrinkage


def test_power_is_correctly_rounded():
    """a^(p-1) as the solver uses it is the exact power rounded once to fp32: checked against
    a 40-digit decimal evaluation (the fp32 value must lie within half an ulp of it)."""
    import decimal
    ctx = decimal.Context(prec=40)
    rng = np.random.default_rng(17)
    a_vals = np.concatenate([rng.random(300) * 10, 10.0 ** rng.uniform(-7, 0, 300)])
    for p in (0.5, 0.7, 0.9, 1.0):
        pm1 = decimal.Decimal(float(np.float32(np.float32(p) - np.float32(1))))
        for a in a_vals.astype(np.float32):
            if not a > 0:
                continue
            t = oracle.pow_pm1(float(a), p)
            exact = ctx.power(decimal.Decimal(float(a)), pm1)
            half_ulp = decimal.Decimal(float(np.spacing(t))) / 2
            assert abs(decimal.Decimal(float(t)) - exact) <= half_ulp, (a, p, t)


def test_shrink_p1_is_textbook_soft_threshold():
    rng = np.random.default_rng(40)
    for r in rng.standard_normal(200).astype(F32):
        for beta in (0.5, 2.0, 10.0, 37.0):
            ib = F32(1) / F32(beta)
            expect = F32(np.sign(r)) * max(F32(abs(r) - ib), F32(0))
            assert oracle.shrink(float(r), beta, 1.0) == expect


@pytest.mark.parametrize("p", [0.3, 0.7, 0.9])
def test_shrink_closed_forms(p):
    """At |r| = 1 the generalised threshold is 1/beta for every p; 0 maps to 0; the operator
    is odd; it is zero exactly below |r| = beta^(-1/(2-p)) and positive above."""
    for beta in (2.0, 10.0, 100.0):
        assert oracle.shrink(1.0, beta, p) == F32(1) - F32(1) / F32(beta)
        assert oracle.shrink(-1.0, beta, p) == -(F32(1) - F32(1) / F32(beta))
        assert oracle.shrink(0.0, beta, p) == 0
        thr = beta ** (-1.0 / (2.0 - p))
        assert oracle.shrink(thr * 0.999, beta, p) == 0
        assert oracle.shrink(thr * 1.001, beta, p) > 0
        assert oracle.shrink(-thr * 1.001, beta, p) < 0


def test_huge_beta_keeps_the_zero_fixed():
    """beta -> inf: the shrinkage is the identity (We = r), so the update returns the same
    zero: z_{k+1} = z_k up to rounding. A dropped or sign-flipped s*sum(We) term fails."""
    rng = np.random.default_rng(50)
    for w in rand_groups(rng, 50, 64):
        out = oracle.quantize_group(w, 4, 20, 0.7, 1e30, 1.01)
        z0 = out["z_trace"][0]
        assert np.all(np.abs(out["z_trace"] - z0) <= 1e-4 * max(1.0, abs(float(z0))))


def test_tiny_beta_is_the_least_squares_zero_step():
    """beta -> 0: the shrinkage is zero, so each update is the least-squares zero for the
    current codes, argmin_z sum_j (Q_j - Ws_j - z)^2, checked with numpy's lstsq."""
    rng = np.random.default_rng(60)
    for nbits, G in ((4, 64), (2, 16)):
        for w in rand_groups(rng, 30, G):
            out = oracle.quantize_group(w, nbits, 6, 0.7, 1e-30, 1.01)
            _, _, _, s = rtn_fp32(w, nbits)
            Ws = (w * s).astype(F32)
            qmax = 2 ** nbits - 1
            for k in range(6):
                zk = out["z_trace"][k]
                Q = np.clip(np.rint(Ws + F32(zk)), 0, qmax).astype(np.float64)
                sol = np.linalg.lstsq(np.ones((G, 1)), Q - Ws.astype(np.float64), rcond=None)[0]
                assert abs(out["z_trace"][k + 1] - sol[0]) <= 2e-6 * max(1.0, abs(sol[0]))


# ---------------------------------------------------------------- brute force


def _brute(w, nbits, p, z_lo, z_hi, h=1e-4):
    zs = np.arange(z_lo, z_hi + h / 2, h)
    return min(lp_error64(w, z, nbits, p) for z in zs.astype(F32))


@pytest.mark.parametrize("seed", range(4))
def test_bruteforce_tiny_two_bit_groups(seed):
    """4-element 2-bit groups (random and adversarial): the solver's zero is never worse
    than RTN, and its gap to the brute-force optimum over a 1e-4 grid of z in
    [z_RTN - 2, z_RTN + 2] is reported."""
    rng = np.random.default_rng(70 + seed)
    groups = list(rng.standard_normal((12, 4)).astype(F32) * 0.02)
    groups += [np.array(g, F32) for g in ([0, 1 / 6, 0.5, 1], [0, 0.49, 0.51, 1],
                                          [-1, 0, 0, 5], [0.3, 0.3, 0.3, 0.31])]
    gaps = []
    for w in groups:
        out = oracle.quantize_group(w, 2, 20, **PARAMS)
        z_rtn = out["z_trace"][0]
        e_sol = lp_error64(w, out["zero"], 2, 0.7)
        e_rtn = lp_error64(w, z_rtn, 2, 0.7)
        assert e_sol <= e_rtn * (1 + 1e-6) + 1e-30
        e_opt = _brute(w, 2, 0.7, float(z_rtn) - 2, float(z_rtn) + 2)
        assert e_opt <= e_sol * (1 + 1e-6) + 1e-30 or e_sol - e_opt < 1e-6
        gaps.append((e_sol - e_opt) / max(e_rtn, 1e-30))
    print("relative gap to the grid optimum:", np.round(gaps, 4))


# ---------------------------------------------------------------- monotone sanity


def _mean_abs_err(W, nbits, G):
    codes, s, z = oracle.quantize(W, nbits, G, 1, 20, **PARAMS, nthreads=oracle.default_threads())
    Wd = oracle.dequantize(codes, s, z, W.shape[0], W.shape[1], G, 1)
    return float(np.mean(np.abs(W.astype(np.float64) - Wd)))


def test_more_bits_and_smaller_groups_lower_the_error():
    """More bits give lower error ("HQQ tutorial" (devpress.csdn.net) section 3.3, nbits)
    and smaller groups give lower error (same section, group_size)."""
    rng = np.random.default_rng(80)
    W = rand_groups(rng, 128, 1024).reshape(128, 1024)
    errs_bits = [_mean_abs_err(W, b, 64) for b in (1, 2, 3, 4, 8)]
    assert all(a > b for a, b in zip(errs_bits, errs_bits[1:])), errs_bits
    errs_g = [_mean_abs_err(W, 4, g) for g in (256, 128, 64, 32, 16)]
    assert all(a > b for a, b in zip(errs_g, errs_g[1:])), errs_g


# ---------------------------------------------------------------- layout, pack, dequant


def _golden_pack():
    rows = []
    with open(os.path.join(GOLDEN, "pack_layout.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            nb, codes, hexs = [x.strip() for x in line.split("|")]
            rows.append((int(nb), [int(c) for c in codes.split()],
                         bytes(int(h, 16) for h in hexs.split())))
    return rows


@pytest.mark.parametrize("nbits,codes,packed", _golden_pack())
def test_pack_matches_hand_derived_layout(nbits, codes, packed):
    out = oracle.pack(codes, nbits)
    assert bytes(out) == packed
    assert list(oracle.unpack(out, len(codes), nbits)) == codes


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
def test_pack_round_trip_and_size(nbits):
    rng = np.random.default_rng(90 + nbits)
    for n in (1, 7, 10, 64, 333, 1000):
        c = rng.integers(0, 2 ** nbits, n).astype(np.uint8)
        pk = oracle.pack(c, nbits)
        expect = 4 * math.ceil(n / 10) if nbits == 3 else math.ceil(n * nbits / 8)
        assert pk.size == expect
        assert np.array_equal(oracle.unpack(pk, n, nbits), c)


def test_dequantize_closed_form_axis1():
    out = oracle.dequantize([0, 1, 2, 3], [0.5], [2.0], 1, 4, 4, 1)
    assert np.array_equal(out, np.array([[-1.0, -0.5, 0.0, 0.5]], F32))


def test_dequantize_axis0_index_map():
    """axis=0, group 2 on a 4x2 matrix: group g = rb*cols + c holds W[2rb], W[2rb+1] of
    column c. Codes 10*g + j with scale 1, zero 0 land at hand-derived positions."""
    codes = [10 * g + j for g in range(4) for j in range(2)]
    out = oracle.dequantize(codes, [1.0] * 4, [0.0] * 4, 4, 2, 2, 0)
    expect = np.array([[0, 10], [1, 11], [20, 30], [21, 31]], F32)
    assert np.array_equal(out, expect)


def test_axis0_equals_axis1_of_transpose():
    """Grouping down columns of W is grouping along rows of W^T (with the group order
    permuted): pins the strided gather against the contiguous one."""
    rng = np.random.default_rng(100)
    rows, cols, G = 64, 48, 16
    W = rand_groups(rng, rows, cols)
    c0, s0, z0 = oracle.quantize(W, 2, G, 0, 20, **PARAMS)
    c1, s1, z1 = oracle.quantize(np.ascontiguousarray(W.T), 2, G, 1, 20, **PARAMS)
    for rb in range(rows // G):
        for c in range(cols):
            g0, g1 = rb * cols + c, c * (rows // G) + rb
            assert np.array_equal(c0[g0], c1[g1]) and s0[g0] == s1[g1] and z0[g0] == z1[g1]


# ---------------------------------------------------------------- second level


def test_meta_quantize_closed_form():
    """Run 0..127: min 0, max 127, zero2 = 0, q_k = round(255 k / 127) (never a tie), and
    step2 = 127/255 in fp32."""
    m = np.arange(128, dtype=F32)
    q, mm = oracle.quantize_meta(m, 128)
    expect = [round(Fraction(255 * k, 127)) for k in range(128)]
    assert list(q) == expect
    assert mm[0, 0] == F32(F32(127) / F32(255)) and mm[0, 1] == 0


def test_meta_round_trip_bound_and_partial_run():
    rng = np.random.default_rng(110)
    m = (rng.standard_normal(300) * 0.01 + 0.02).astype(F32)
    q, mm = oracle.quantize_meta(m, 128)
    assert mm.shape == (3, 2)
    back = oracle.dequantize_meta(q, mm, 128)
    for i in range(3):
        sl = slice(128 * i, min(128 * (i + 1), 300))
        assert np.all(np.abs(back[sl] - m[sl]) <= mm[i, 0] / 2 * (1 + 1e-5) + 1e-9)


# ---------------------------------------------------------------- determinism


def test_deterministic_and_thread_count_invariant():
    """Quantization is deterministic ("HQQ calibration-free guide" (lnwmold.com) 6.4)."""
    rng = np.random.default_rng(120)
    W = rand_groups(rng, 64, 512)
    a = oracle.quantize(W, 4, 64, 1, 20, **PARAMS, nthreads=1)
    b = oracle.quantize(W, 4, 64, 1, 20, **PARAMS, nthreads=4)
    for x, y in zip(a, b):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))


# ---------------------------------------------------------------- the quantized linear layer

def test_round_to_bf16_ties_and_library():
    # hand-derived: bf16 keeps 8 significant bits, so its spacing at 1 is 2^-7
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -20,
                  2.0 ** -130], F32)
    want = np.array([1.0, 1 + 2.0 ** -6, -1.0, 1 + 2.0 ** -7, 2.0 ** -130], F32)
    assert np.array_equal(oracle.round_to_dtype(x, "bf16"), want)
    # library routine: torch's fp32 -> bf16 conversion rounds to nearest even as well
    import torch
    r = (np.random.default_rng(5).standard_normal(200_000) * 37.0).astype(F32)
    lib = torch.from_numpy(r).to(torch.bfloat16).float().numpy()
    assert np.array_equal(oracle.round_to_dtype(r, "bf16"), lib)
    assert np.array_equal(oracle.round_to_dtype(r, "f16"), r.astype(np.float16).astype(F32))


def _random_layer(N, K, seed, meta_scale=0.01):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, size=N * K, dtype=np.uint8)
    ng = N * K // 64
    scale = oracle.round_to_dtype((rng.random(ng) * meta_scale + 1e-4).astype(F32), "bf16")
    zero = oracle.round_to_dtype((rng.random(ng) * 15).astype(F32), "bf16")
    return codes, scale, zero


def test_linear_closed_form_constant_group():
    # one group per row, every code c_n, scale s_n, zero z_n, X = all ones:
    # Y[m, n] = 64·bf16((c_n - z_n)·s_n) exactly (64 equal terms, power-of-two multiple)
    N, K = 8, 64
    c = np.arange(N, dtype=np.uint8) * 2
    codes = np.repeat(c, K)
    scale = np.array([0.5, 0.25, 1.0, 2.0, 0.125, 0.75, 1.5, 3.0], F32)
    zero = np.array([0.0, 1.0, 3.0, 7.5, 15.0, 2.25, 0.5, 8.0], F32)
    X = np.ones((3, K), F32)
    Y = oracle.linear(X, codes, scale, zero, N, K, "bf16")
    want = 64.0 * ((c.astype(np.float64) - zero) * scale)  # every (c - z)·s is exact in bf16
    assert np.array_equal(Y, np.broadcast_to(want, (3, N)))
    bias = np.array([1, -2, 3, -4, 5, -6, 7, -8], F32)
    assert np.array_equal(oracle.linear(X, codes, scale, zero, N, K, "bf16", bias) - Y,
                          np.broadcast_to(bias.astype(np.float64), (3, N)))


def test_linear_one_hot_rows_give_transposed_weight():
    # X = identity: Y[k, n] = W'[n, k]. Fails on a transposed operand or a wrong group index.
    N, K = 24, 192
    codes, scale, zero = _random_layer(N, K, 3)
    Y = oracle.linear(np.eye(K, dtype=F32), codes, scale, zero, N, K, "bf16")
    Wd = np.empty((N, K), np.float64)
    for n in range(N):  # element by element from the definition
        for k in range(K):
            g = n * (K // 64) + k // 64
            v = F32(F32(F32(codes[n * K + k]) - zero[g]) * scale[g])
            Wd[n, k] = oracle.round_to_dtype(np.array([v], F32), "bf16")[0]
    assert np.array_equal(Y, Wd.T)


def test_linear_matches_brute_force_sum():
    N, K, M = 16, 128, 5
    codes, scale, zero = _random_layer(N, K, 4)
    rng = np.random.default_rng(6)
    X = oracle.round_to_dtype(rng.standard_normal((M, K)).astype(F32), "bf16")
    Y = oracle.linear(X, codes, scale, zero, N, K, "bf16")
    Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, N, K, 64, 1), "bf16")
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(X[m, k])) * Fraction(float(Wd[n, k])) for k in range(K))
            assert abs(Fraction(Y[m, n]) - exact) <= Fraction(1, 2 ** 40) * (1 + abs(exact))


# ---------------------------------------------------------------- MXFP4 (row f3)

def _e2m1_from_fields(code):
    """E2M1 from its bit fields (sign | 2 exponent bits | 1 mantissa bit, bias 1): exponent
    field 0 is subnormal (value = M/2), otherwise 2^(E-1) * (1 + M/2)."""
    s = -1.0 if code & 8 else 1.0
    E, M = (code >> 1) & 3, code & 1
    return s * (M * 0.5 if E == 0 else 2.0 ** (E - 1) * (1 + M / 2))


def test_e2m1_decode_matches_bit_fields():
    for c in range(16):
        assert oracle.e2m1_decode(c) == _e2m1_from_fields(c), c
    # the largest normal is 1.5 * 2^2 = 6, the exponent the MX scale rule subtracts
    assert max(_e2m1_from_fields(c) for c in range(16)) == 6.0


def test_e2m1_encode_is_nearest_ties_to_even_with_saturation():
    grid = np.array([_e2m1_from_fields(c) for c in range(8)])
    mids = (grid[1:] + grid[:-1]) / 2
    xs = np.concatenate([grid, mids, mids + 1e-3, mids - 1e-3, [6.5, 7.9, 8.0, 1e6],
                         np.linspace(0, 7, 701)])
    for x in xs:
        for sgn in (1.0, -1.0):
            v = np.float32(sgn * x)
            code = oracle.e2m1_encode(v)
            a = min(abs(float(v)), 6.0)  # saturation: anything above 6 becomes 6
            d = np.abs(grid - a)
            cands = np.flatnonzero(d == d.min())
            want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
            assert code & 7 == want, (v, code)
            assert (code >> 3) == (1 if np.signbit(v) else 0)


def test_mx_exponent_closed_form():
    rng = np.random.default_rng(14)
    for _ in range(300):
        v = (rng.standard_normal(32) * 10.0 ** rng.uniform(-6, 6)).astype(F32)
        amax = float(np.max(np.abs(v)))
        want = int(np.floor(np.log2(amax))) - 2
        assert oracle.mx_exponent(v) == max(-127, min(127, want))
    assert oracle.mx_exponent([4.0]) == 0 and oracle.mx_exponent([3.999]) == -1
    assert oracle.mx_exponent([-8.0, 1.0]) == 1
    assert oracle.mx_exponent(np.zeros(32, F32)) == -127


def test_mxfp4_exact_blocks_round_trip_and_packing():
    rng = np.random.default_rng(15)
    rows, cols = 6, 96
    W = np.zeros((rows, cols), F32)
    for b in range(rows * cols // 32):
        e = int(rng.integers(-20, 20))
        vals = np.array([_e2m1_from_fields(int(c)) for c in rng.integers(0, 16, 32)])
        vals[0] = 6.0 if b % 2 else -4.0  # the block maximum fixes the exponent at e
        W.reshape(-1)[b * 32:(b + 1) * 32] = (vals * 2.0 ** e).astype(F32)
    codes, scales = oracle.mxfp4_quantize(W)
    back = oracle.mxfp4_dequantize(codes, scales, rows, cols)
    nz = W != 0
    assert np.array_equal(back[nz], W[nz]) and np.all(back[~nz] == 0)
    # two codes per byte, element 2j in the low nibble: the 4-bit integer packing
    flat = np.array([oracle.e2m1_encode(np.float32(x) / np.float32(2.0 ** (int(s) - 127)))
                     for x, s in zip(W.reshape(-1), np.repeat(scales, 32))], np.uint8)
    assert np.array_equal(codes, oracle.pack(flat, 4))


def test_mxfp4_error_bound_and_extremes():
    rng = np.random.default_rng(16)
    W = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)))).astype(F32)
    codes, scales = oracle.mxfp4_quantize(W)
    back = oracle.mxfp4_dequantize(codes, scales, 64, 256)
    X = 2.0 ** (np.repeat(scales.astype(np.int64) - 127, 32).reshape(64, 256))
    x = np.abs(W) / X  # scaled magnitudes lie in [0, 8)
    assert x.max() < 8
    half_gap = np.where(x <= 2, 0.25, np.where(x <= 4, 0.5, 1.0))
    bound = np.where(x <= 6, half_gap, x - 6) * X
    assert np.all(np.abs(W - back) <= bound * (1 + 1e-6))
    # every block's largest magnitude lands on 4 or 6 (scaled max in [4, 8))
    top = np.abs(back).reshape(-1, 32).max(1) / X.reshape(-1, 32)[:, 0]
    assert np.all((top == 4) | (top == 6))
