"""CPU checks of the test-side helpers that read GPU output (no GPU needed): the numpy
decoder of the packed layout against the hand-derived layout vectors, and the exact-grid
construction's claims."""
import os

import numpy as np
import pytest
import torch

from parity import np_unpack

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pack_layout.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        nb, codes, hexs = [x.strip() for x in line.split("|")]
        rows.append((int(nb), [int(c) for c in codes.split()],
                     bytes(int(h, 16) for h in hexs.split())))
    return rows


@pytest.mark.parametrize("nbits,codes,packed", _golden())
def test_np_unpack_reads_the_hand_derived_layout(nbits, codes, packed):
    got = np_unpack(np.frombuffer(packed, np.uint8), len(codes), nbits)
    assert got.tolist() == codes


# ------------------------------------------------------------------ the parity judge itself
# The judge is exercised on the CPU with the oracle's own results standing in for the GPU's,
# then with one deliberate change each, to show that each kind of mismatch is classified.

import oracle
import parity
from parity import judge

ARGS = (4, 20, 0.7, 10.0, 1.01)  # nbits, iters, p, beta0, kappa


def _groups(n=3000, seed=5):
    from calibration_free_weight_hqq_b200 import synthetic
    W = synthetic.weight(n * 64 // 1024, 1024, seed=seed, dtype=torch.bfloat16)
    return W.float().numpy().reshape(-1, 64)



def test_judge_accepts_the_oracles_own_result():
    Wg = _groups()
    oc, os_, oz = oracle.quantize(Wg, 4, 64, 1, 20, 0.7, 10.0, 1.01, nthreads=4)
    r, *_ = judge(Wg, oc, os_, oz, *ARGS)
    assert r.zero_exact == r.n_groups and r.zero_near_tie == 0 and r.zero_diverged == 0
    assert r.code_diff == 0
    r.check()


def _tie_and_non_tie(Wg):
    """One group with a candidate zero (not the best) whose fp64 error ties the best's, and
    one group with a candidate zero that clearly loses."""
    tie = lose = None
    for i in range(Wg.shape[0]):
        og = oracle.quantize_group(Wg[i], *ARGS)
        e_b, b_b = parity.lp_error64(Wg[i], og["zero"], og["scale"], 4, 0.7, with_bound=True)
        for zk in og["z_trace"]:
            if abs(zk - og["zero"]) <= 1e-5 * max(abs(og["zero"]), 1):
                continue
            e_k, b_k = parity.lp_error64(Wg[i], zk, og["scale"], 4, 0.7, with_bound=True)
            if tie is None and abs(e_k - e_b) <= b_k + b_b:
                tie = (i, zk)
            if lose is None and e_k > e_b * 1.01:
                lose = (i, zk)
        if tie and lose:
            return tie, lose
    pytest.skip("no tying candidate in this sample")


def test_judge_classifies_near_ties_and_divergence():
    Wg = _groups()
    oc, os_, oz = oracle.quantize(Wg, 4, 64, 1, 20, 0.7, 10.0, 1.01, nthreads=4)
    (it, zt), (il, zl) = _tie_and_non_tie(Wg)
    # a tying candidate with the oracle's codes at that candidate: a near tie, codes exact
    gz, gc = oz.copy(), oc.copy()
    gz[it] = zt
    gc[it] = oracle.codes_at_zero(Wg[it], 4, zt)
    r, *_ = judge(Wg, gc, os_, gz, *ARGS)
    assert r.zero_near_tie == 1 and r.zero_diverged == 0 and r.code_diff == 0
    # the same zero with the best zero's codes kept: the codes are judged at the candidate
    gc2 = oc.copy()
    r2, *_ = judge(Wg, gc2, os_, gz, *ARGS)
    assert r2.zero_near_tie == 1
    assert r2.code_diff == np.count_nonzero(oracle.codes_at_zero(Wg[it], 4, zt) != oc[it])
    # a losing candidate: diverged, although it is one of the oracle's zeros
    gz3 = oz.copy()
    gz3[il] = zl
    r3, *_ = judge(Wg, oc, os_, gz3, *ARGS)
    assert r3.zero_near_tie == 0 and r3.zero_diverged == 1 and r3.zero_off_not_candidate == 0
    # a zero that is none of the candidates (the best moved by 1e-3): diverged
    gz4 = oz.copy()
    gz4[it] = np.float32(oz[it] + 1e-3 * max(abs(oz[it]), 1))
    r4, *_ = judge(Wg, oc, os_, gz4, *ARGS)
    assert r4.zero_diverged == 1 and r4.zero_off_not_candidate == 1


def test_judge_rejects_codes_off_by_two_and_too_many_near_ties():
    Wg = _groups()
    oc, os_, oz = oracle.quantize(Wg, 4, 64, 1, 20, 0.7, 10.0, 1.01, nthreads=4)
    gc = oc.copy()
    gc[7, 3] = (int(gc[7, 3]) + 2) % 16
    r, *_ = judge(Wg, gc, os_, oz, *ARGS)
    assert r.code_maxdiff == 2
    with pytest.raises(AssertionError):
        r.check()
    r.zero_near_tie = int(parity.NEAR_TIE_FRAC * r.n_groups) + 1
    gc[7, 3] = oc[7, 3]
    r.code_maxdiff = 0
    with pytest.raises(AssertionError):
        r.check()


def test_lp_eval_bound_covers_fp32_evaluations():
    """The bound covers what it claims for the oracle's side: an fp32 evaluation of
    sum a^p (powf per term, sequential fp32 sum) stays within it of the fp64 value, on
    residual magnitudes from 1e-6 to 1 (the range where the log2 error grows)."""
    rng = np.random.default_rng(3)
    for G in (8, 64, 256):
        for scale in (1e-6, 1e-3, 0.3):
            a = (rng.random(G) * scale).astype(np.float32).astype(np.float64)
            e64 = float(np.sum(a ** 0.7))
            acc = np.float32(0)
            for x in a.astype(np.float32):
                acc = np.float32(acc + np.float32(x * np.float32(np.power(x, np.float32(-0.3)))))
            assert abs(float(acc) - e64) <= parity.lp_eval_bound(a, 0.7)
    # it grows with |log2 a|: tiny residuals get a wider relative allowance
    small = parity.lp_eval_bound(np.full(64, 1e-5), 0.7) / (64 * 1e-5 ** 0.7)
    large = parity.lp_eval_bound(np.full(64, 0.6), 0.7) / (64 * 0.6 ** 0.7)
    assert small > large
