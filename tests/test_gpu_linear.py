"""GPU parity of hqq_linear (the tensor-core consumer of the packed 4-bit format) against the
oracle's fp64 definition.

Inputs: random codes, scale and zero drawn here and packed by the oracle's packer (none of
them come from the CUDA path), activations drawn from a seeded generator.

Bars:
  * one-hot activations (X = identity) make every output a single product with 1, exact in
    any accumulation: Y must equal the dequantized weight transposed, bit for bit;
  * random activations: |Y - Y64| <= u·|Y64| + (1 + u)·K·2^-23·sum_k |X[m,k]·W'[n,k]|,
    where u is the unit roundoff of the output type (2^-8 bf16, 2^-11 fp16) and the second
    term bounds an fp32 accumulation of K exact products in any order, with truncation
    (2^-23) instead of rounding (2^-24) allowed inside the tensor core.
"""
import numpy as np
import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
import oracle

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}
UNIT = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}


def make_layer(N, K, seed, meta_dtype="bf16"):
    """Random 4-bit g64 axis-1 layer [N, K]: codes, scale ~ U(1e-4, 0.01), zero ~ U(0, 15)."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, size=N * K, dtype=np.uint8)
    ng = N * K // 64
    scale = oracle.round_to_dtype((rng.random(ng) * 0.01 + 1e-4).astype(np.float32), meta_dtype)
    zero = oracle.round_to_dtype((rng.random(ng) * 15).astype(np.float32), meta_dtype)
    packed = oracle.pack(codes, 4)
    dev = dict(
        packed=torch.from_numpy(packed).cuda(),
        scale=torch.from_numpy(scale).to(TORCH[meta_dtype]).cuda(),
        zero=torch.from_numpy(zero).to(TORCH[meta_dtype]).cuda(),
    )
    return codes, scale, zero, dev


def make_x(M, K, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(M, K, generator=g).to(TORCH[dtype])


def run_linear(Xc, dev, N, dtype, meta_dtype, bias=None):
    params = hqq.make_params(4, 64, 1, w_dtype=TORCH[dtype], meta_dtype=TORCH[meta_dtype])
    Y = hqq.hqq_linear(Xc.cuda(), dev["packed"], dev["scale"], dev["zero"], N, params,
                       bias=None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64)


def check_against_oracle(Y, X, codes, scale, zero, N, K, dtype, bias=None, rows=None):
    Xf = X.float().numpy()
    if rows is not None:
        Xf, Y = Xf[rows], Y[rows]
    b = None if bias is None else bias.float().numpy()
    Y64 = oracle.linear(Xf, codes, scale, zero, N, K, dtype, b)
    Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, N, K, 64, 1), dtype)
    S = np.abs(Xf.astype(np.float64)) @ np.abs(Wd.astype(np.float64)).T
    u = UNIT[dtype]
    acc = K * 2.0 ** -23 * S
    tol = u * np.abs(Y64) + (1 + u) * acc + 1e-30
    err = np.abs(Y - Y64)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"max err/tol = {worst}"
    # the fp32 accumulation is far better than its bound: most outputs round like the
    # exact value does
    same = np.mean(Y == oracle.round_to_dtype(Y64.astype(np.float32), dtype))
    return worst, same


def assert_no_timeouts():
    assert hqq.hqq_wait_timeouts() == 0


def test_linear_one_hot_is_bit_exact_transposed_weight():
    # N = 2·256 + 8 (ragged last tile), K = 640 (10 k-blocks: the 3-stage ring wraps 3 times),
    # M = K = 640 (ragged last M tile of 128 rows)
    N, K = 520, 640  # M = 640 > 128: the 2-SM kernel
    codes, scale, zero, dev = make_layer(N, K, 11)
    X = torch.eye(K, dtype=torch.bfloat16)
    Y = run_linear(X, dev, N, "bf16", "bf16")
    Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, N, K, 64, 1), "bf16")
    assert np.array_equal(Y, Wd.T.astype(np.float64))
    assert_no_timeouts()


@pytest.mark.parametrize("M,N,K,dtype,meta,with_bias", [
    (300, 264, 128, "bf16", "bf16", False),
    (512, 1024, 4096, "bf16", "bf16", True),
    (257, 512, 1024, "f16", "f16", True),
    (128, 256, 64, "bf16", "f32", False),
    (1, 8, 64, "bf16", "bf16", True),
    (777, 1032, 704, "f16", "bf16", False),
    (300, 256, 320, "bf16", "bf16", True),    # K/64 odd: one value per copy
    (260, 512, 192, "f16", "f32", False),     # K/64 odd, fp32 meta
    (129, 136, 64, "bf16", "bf16", True),     # 2-SM kernel: one k-block, ragged M and N
])
def test_linear_random_matches_oracle(M, N, K, dtype, meta, with_bias):
    codes, scale, zero, dev = make_layer(N, K, 100 + M + N + K, meta)
    X = make_x(M, K, 7 + M, dtype)
    bias = make_x(1, N, 9, dtype)[0] if with_bias else None
    Y = run_linear(X, dev, N, dtype, meta, bias)
    worst, same = check_against_oracle(Y, X, codes, scale, zero, N, K, dtype, bias)
    assert same > 0.9, same
    assert_no_timeouts()


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_linear_llama_block_shapes_sampled_rows(N, K):
    # the Llama-7B block shapes at 4096 tokens, as timed; the oracle checks 48 sampled rows
    # (every column, so every N tile and every k-block of those rows)
    M = 4096
    codes, scale, zero, dev = make_layer(N, K, N + K)
    X = make_x(M, K, 21, "bf16")
    Y = run_linear(X, dev, N, "bf16", "bf16")
    rows = np.sort(np.random.default_rng(N * K).choice(M, 48, replace=False))
    worst, same = check_against_oracle(Y, X, codes, scale, zero, N, K, "bf16", rows=rows)
    assert same > 0.9, same
    assert np.isfinite(Y).all()
    assert_no_timeouts()


def test_linear_empty_and_zero_k():
    params = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16)
    e = torch.empty(0, dtype=torch.uint8, device="cuda")
    eb = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    # M = 0: nothing to do
    Y = hqq.hqq_linear(torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"), e, eb, eb, 16,
                       params)
    assert Y.shape == (0, 16)
    # K = 0: the sum is empty, Y = bias (or 0)
    bias = make_x(1, 24, 3, "bf16")[0].cuda()
    Y = hqq.hqq_linear(torch.empty(5, 0, dtype=torch.bfloat16, device="cuda"), e, eb, eb, 24,
                       params, bias=bias, Y=torch.full((5, 24), 7.0, dtype=torch.bfloat16,
                                                       device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(Y, bias.expand(5, 24))
    Y = hqq.hqq_linear(torch.empty(5, 0, dtype=torch.bfloat16, device="cuda"), e, eb, eb, 24,
                       params)
    torch.cuda.synchronize()
    assert torch.equal(Y, torch.zeros(5, 24, dtype=torch.bfloat16, device="cuda"))


def test_linear_consumes_the_quantizer_output():
    # hand-over consistency (not oracle parity): the format the GPU quantizer writes is the
    # format the linear layer reads - hqq_linear on the quantizer's output agrees with the GPU
    # dequantizer's weight multiplied in fp64, within the same accumulation bound
    from calibration_free_weight_hqq_b200 import synthetic
    N, K, M = 384, 1024, 200
    W = synthetic.weight(N, K, seed=77, dtype=torch.bfloat16, device="cuda")
    packed, scale, zero = hqq.hqq_quantize(W, 4, 64, 1)
    X = make_x(M, K, 78, "bf16")
    Y = hqq.hqq_linear(X.cuda(), packed, scale, zero, N)
    Wd = hqq.hqq_dequantize(packed, scale, zero, N, K)
    torch.cuda.synchronize()
    Xf = X.float().numpy().astype(np.float64)
    Wf = Wd.float().cpu().numpy().astype(np.float64)
    ref = Xf @ Wf.T
    tol = UNIT["bf16"] * np.abs(ref) + (1 + UNIT["bf16"]) * K * 2.0 ** -23 * (np.abs(Xf) @ np.abs(Wf).T)
    assert np.all(np.abs(Y.float().cpu().numpy() - ref) <= tol)
    assert_no_timeouts()


def test_linear_meta_views_with_odd_offsets():
    # scale/zero as views starting one element into a buffer: only 2-byte aligned, so the
    # kernel must not copy them in 4-byte pairs
    N, K, M = 264, 512, 130
    codes, scale, zero, dev = make_layer(N, K, 5)
    buf_s = torch.empty(scale.size + 1, dtype=torch.bfloat16, device="cuda")
    buf_z = torch.empty(zero.size + 1, dtype=torch.bfloat16, device="cuda")
    buf_s[1:] = dev["scale"]
    buf_z[1:] = dev["zero"]
    dev = dict(packed=dev["packed"], scale=buf_s[1:], zero=buf_z[1:])
    assert dev["scale"].data_ptr() % 4 == 2
    X = make_x(M, K, 6, "bf16")
    Y = run_linear(X, dev, N, "bf16", "bf16")
    check_against_oracle(Y, X, codes, scale, zero, N, K, "bf16")
    assert_no_timeouts()


def test_linear_skinny_one_hot_spans_every_k_slice():
    # 16 < M <= 128 takes the split-K kernel (4 CTAs per W' tile, each a slice of K): one-hot rows
    # picking k = 5m + 3 reach every slice; each output is one product with 1, so Y must be
    # the dequantized weight's columns exactly (partial sums of the other slices are +0)
    N, K, M = 264, 1024, 100
    codes, scale, zero, dev = make_layer(N, K, 31)
    ks = 5 * np.arange(M) + 3
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[torch.arange(M), torch.from_numpy(ks)] = 1.0
    Y = run_linear(X, dev, N, "bf16", "bf16")
    Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, N, K, 64, 1), "bf16")
    assert np.array_equal(Y, Wd[:, ks].T.astype(np.float64))
    assert_no_timeouts()


@pytest.mark.parametrize("M", [1, 7, 16, 64, 128])
@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_linear_skinny_llama_shapes(M, N, K):
    codes, scale, zero, dev = make_layer(N, K, N + K + M)
    X = make_x(M, K, 40 + M, "bf16")
    bias = make_x(1, N, 41, "bf16")[0]
    Y = run_linear(X, dev, N, "bf16", "bf16", bias)
    worst, same = check_against_oracle(Y, X, codes, scale, zero, N, K, "bf16", bias)
    assert same > 0.9, same
    assert_no_timeouts()


def test_linear_skinny_is_deterministic():
    N, K, M = 1024, 2048, 33
    codes, scale, zero, dev = make_layer(N, K, 8)
    X = make_x(M, K, 9, "f16")
    dev16 = make_layer(N, K, 8, "f16")[3]
    a = run_linear(X, dev16, N, "f16", "f16")
    b = run_linear(X, dev16, N, "f16", "f16")
    assert np.array_equal(a, b)


def test_linear_decode_one_hot_spans_every_k_slice():
    # M <= 16 takes the warp-MMA decode kernel: K = 2112 is 16.5 k-blocks of 128, split over a
    # cluster of 8 CTAs (3 k-blocks each, the last slices partial or empty, the last k-block
    # half). One-hot rows picking k = 131m + 7 reach every non-empty slice and every position
    # of the in-block permutation; each output is one product with 1: Y must be the
    # dequantized weight's columns exactly
    N, K, M = 264, 2112, 16
    codes, scale, zero, dev = make_layer(N, K, 32)
    ks = 131 * np.arange(M) + 7
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[torch.arange(M), torch.from_numpy(ks)] = 1.0
    Y = run_linear(X, dev, N, "bf16", "bf16")
    Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, N, K, 64, 1), "bf16")
    assert np.array_equal(Y, Wd[:, ks].T.astype(np.float64))
    # every k of one k-block through the permutation: token m picks k = 128 + m, 144 + m, ..
    for base in (128, 2048):
        ks = base + np.arange(16) * (4 if base == 128 else 1)
        X = torch.zeros(M, K, dtype=torch.bfloat16)
        X[torch.arange(M), torch.from_numpy(ks)] = 1.0
        Y = run_linear(X, dev, N, "bf16", "bf16")
        assert np.array_equal(Y, Wd[:, ks].T.astype(np.float64))


@pytest.mark.parametrize("M,N,K,dtype,meta,with_bias", [
    (1, 8, 64, "bf16", "bf16", False),        # one CTA, one half k-block
    (5, 136, 576, "f16", "f32", True),        # 2 slices, ragged row tile, half k-block
    (16, 264, 2112, "bf16", "f16", True),     # 8 slices, two of them empty
    (9, 1024, 4096, "f16", "f16", False),
    (3, 256, 32768, "bf16", "bf16", True),    # the largest K the decode kernel takes
    (2, 128, 32832, "bf16", "bf16", False),   # one k-block more: the split-K kernel
])
def test_linear_decode_matches_oracle(M, N, K, dtype, meta, with_bias):
    codes, scale, zero, dev = make_layer(N, K, 500 + M + N + K, meta)
    X = make_x(M, K, 60 + M, dtype)
    bias = make_x(1, N, 61, dtype)[0] if with_bias else None
    Y = run_linear(X, dev, N, dtype, meta, bias)
    worst, same = check_against_oracle(Y, X, codes, scale, zero, N, K, dtype, bias)
    assert same > 0.9, same
    assert_no_timeouts()


def test_linear_decode_is_deterministic():
    N, K, M = 1024, 4096, 11
    dev16 = make_layer(N, K, 12, "f16")[3]
    X = make_x(M, K, 13, "f16")
    a = run_linear(X, dev16, N, "f16", "f16")
    b = run_linear(X, dev16, N, "f16", "f16")
    assert np.array_equal(a, b)


def test_linear_decode_overlap_flag_keeps_every_dependency():
    """HQQ_FLAG_OVERLAP_WEIGHTS lets a decode launch start while the previous kernel on the
    stream finishes; it must still read X only after that kernel is done. A chain of decode
    layers where layer i+1 reads layer i's output, launched back to back on one stream with
    nothing in between, must give bit for bit what the same chain gives without the flag (a
    layer that read its X early would see the stale buffer, which holds other values), and
    one-hot rows through flagged launches must still return the dequantized weight."""
    N = K = 1024
    M = 16
    layers = [make_layer(N, K, 900 + i)[3] for i in range(6)]
    X0 = make_x(M, K, 77, "bf16").cuda()

    def chain(flag):
        p = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, meta_dtype=torch.bfloat16,
                            overlap_weights=flag)
        bufs = [torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        x = X0
        for i, dev in enumerate(layers):
            y = bufs[i % 2]
            hqq.hqq_linear(x, dev["packed"], dev["scale"], dev["zero"], N, p, Y=y)
            x = y
        torch.cuda.synchronize()
        return x.float().cpu().numpy()

    plain, overlapped = chain(False), chain(True)
    assert np.isfinite(plain).all()
    assert np.array_equal(plain, overlapped)
    # one-hot through a flagged launch right after another flagged launch
    codes, scale, zero, dev = make_layer(264, 2112, 32)
    ks = 131 * np.arange(M) + 7
    X = torch.zeros(M, 2112, dtype=torch.bfloat16)
    X[torch.arange(M), torch.from_numpy(ks)] = 1.0
    p = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, meta_dtype=torch.bfloat16,
                        overlap_weights=True)
    Xc = X.cuda()
    Y1 = hqq.hqq_linear(Xc, dev["packed"], dev["scale"], dev["zero"], 264, p)
    Y2 = hqq.hqq_linear(Xc, dev["packed"], dev["scale"], dev["zero"], 264, p)
    torch.cuda.synchronize()
    Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, 264, 2112, 64, 1), "bf16")
    for Y in (Y1, Y2):
        assert np.array_equal(Y.float().cpu().numpy(), Wd[:, ks].T)
    assert_no_timeouts()


def test_linear_decode_wide_layer_one_hot():
    """A layer wide enough that its 128-row tiles outnumber the clusters that fit on the GPU
    (11008 rows) runs the decode kernel with 64-row tiles, each cluster looping over several;
    one-hot rows make every output one dequantized weight: exact for every row tile."""
    N, K, M = 11008, 2112, 16
    codes, scale, zero, dev = make_layer(N, K, 4242)
    ks = 131 * np.arange(M) + 7
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[torch.arange(M), torch.from_numpy(ks)] = 1.0
    for flag in (False, True):
        p = hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16, meta_dtype=torch.bfloat16,
                            overlap_weights=flag)
        Y = hqq.hqq_linear(X.cuda(), dev["packed"], dev["scale"], dev["zero"], N, p)
        torch.cuda.synchronize()
        Wd = oracle.round_to_dtype(oracle.dequantize(codes, scale, zero, N, K, 64, 1), "bf16")
        assert np.array_equal(Y.float().cpu().numpy(), Wd[:, ks].T)
    assert_no_timeouts()
