"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs, element by element, within the tolerances stated in tests/parity.py.

Covers the five shipped workloads (full matrices where the oracle finishes in seconds,
seeded group samples that always include the ragged tail otherwise), every nbits, group
size, axis and dtype on small ragged shapes, and the edge cases: empty input, constant
groups, an active shrinkage, iters = 0, canary bytes past the outputs, stored meta dtypes,
determinism and a matrix with more than 2^32 elements."""
import copy

import numpy as np
import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
from calibration_free_weight_hqq_b200 import synthetic, workloads
import oracle
from parity import (compare, dequant_parity, exact_grid_weights, group_view, judge, np_unpack,
                    record, sample_groups, unpack_groups)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def W_of(m):
    return workloads.make_weight(m, device=DEV)


# ------------------------------------------------------------------ shipped workloads


def test_single_fp16_full():
    """[4096,1024] fp16, 4-bit g64 axis 1: every group compared."""
    m = workloads.single_fp16().matrices[0]
    r = compare(W_of(m), 4, 64, 1)
    print(r)
    r.check()


@pytest.mark.parametrize("i", range(7))
def test_llama7b_block_4b(i):
    m = workloads.llama7b_block_4b().matrices[i]
    r = compare(W_of(m), m.nbits, m.group_size, m.axis, n_sample=40000, seed=i)
    print(m.name, r)
    r.check()


@pytest.mark.parametrize("i", range(7))
def test_llama7b_block_2b_axis0(i):
    m = workloads.llama7b_block_2b_axis0().matrices[i]
    r = compare(W_of(m), m.nbits, m.group_size, m.axis, n_sample=100000, seed=i)
    print(m.name, r)
    r.check()


@pytest.mark.parametrize("i", range(2))
def test_mlp70b_mixed_with_meta(i):
    m = workloads.mlp70b_mixed().matrices[i]
    r = compare(W_of(m), m.nbits, m.group_size, m.axis, n_sample=60000, seed=i,
                quant_meta=True, meta_group=m.meta_group_size)
    print(m.name, r)
    r.check()


def test_llama7b_model_sampled():
    """Whole 7B-shaped model: all 224 matrices quantized on the GPU; a seeded sample of
    1/64 of every matrix's groups (plus its first and last groups) compared with the oracle
    (about 1.6 million groups in all)."""
    wl = workloads.llama7b_model_4b()
    total = None
    for i, m in enumerate(wl.matrices):
        ng = m.numel // m.group_size
        r = compare(W_of(m), m.nbits, m.group_size, m.axis, n_sample=-(-ng // 64), seed=i,
                    label=f"llama7b_model[{m.name}]")
        r.check()
        total = copy.copy(r) if total is None else _acc(total, r)
    assert total.n_groups >= wl.weights // 64 // 64
    print(total.summary())


def _acc(a, b):
    for f in ("n_groups", "n_codes", "scale_exact", "zero_exact", "zero_near_tie",
              "zero_diverged", "code_diff"):
        setattr(a, f, getattr(a, f) + getattr(b, f))
    a.code_maxdiff = max(a.code_maxdiff, b.code_maxdiff)
    return a


# ------------------------------------------------------------------ coverage grid


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("G", [8, 16, 32, 64, 128, 256])
@pytest.mark.parametrize("axis", [0, 1])
def test_grid_ragged(nbits, G, axis):
    """Ragged shapes: >= 10^4 groups (so that the 0.01 % rate admits one event), group
    count not a multiple of the 160-group block."""
    shape = (837, 12 * G) if axis == 1 else (11 * G, 1000)
    W = synthetic.weight(*shape, seed=1000 + nbits * 10 + G + axis, dtype=torch.bfloat16,
                         outlier_rate=0.01, device=DEV)
    compare(W, nbits, G, axis).check()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("axis", [0, 1])
def test_input_dtypes(dtype, axis):
    W = synthetic.weight(1024, 1024, seed=7, dtype=dtype, outlier_rate=0.002, device=DEV)
    compare(W, 4, 64, axis).check()


@pytest.mark.parametrize("p,beta0,kappa,iters", [(1.0, 10.0, 1.01, 20), (0.5, 3.0, 1.05, 20),
                                                 (0.7, 10.0, 1.01, 0), (0.7, 10.0, 1.01, 1),
                                                 (0.7, 10.0, 1.01, 57)])
def test_solver_constants(p, beta0, kappa, iters):
    W = synthetic.weight(1024, 1024, seed=11, dtype=torch.bfloat16, device=DEV)
    r = compare(W, 4, 64, 1, iters=iters, p=p, beta0=beta0, kappa=kappa)
    r.check()
    if iters == 0:  # pure RTN: everything bit-exact
        assert r.zero_exact == r.n_groups and r.code_diff == 0


def test_active_shrinkage():
    """Weights with sigma ~ 1 at 2 bits and beta0 = 1: residuals exceed the shrinkage
    cut-off, so the exact per-element path runs on most groups and iterations."""
    W = synthetic.weight(512, 1024, seed=12, dtype=torch.float32, sigma_layer=1.0, device=DEV)
    r = compare(W, 2, 16, 1, beta0=1.0, kappa=1.1)
    print(r)
    r.check()
    W = synthetic.weight(512, 1024, seed=13, dtype=torch.bfloat16, outlier_rate=0.02,
                         device=DEV)
    r = compare(W, 1, 32, 1)
    print(r)
    r.check()


def test_constant_groups():
    W = synthetic.weight(1024, 1024, seed=14, dtype=torch.bfloat16, device=DEV)
    W[5] = 0.25
    W[9, :64] = -1.0
    W[17] = 0
    r = compare(W, 4, 64, 1)
    r.check()
    pk, s, z = hqq.hqq_quantize(W, 4, 64, 1)
    assert torch.all(s[5] == 1) and torch.all(z[5] == -0.25) and torch.all(z[17] == 0)
    assert s[9, 0] == 1 and z[9, 0] == 1.0
    codes = np_unpack(pk.cpu().numpy(), W.numel(), 4).reshape(1024, 1024)
    assert np.all(codes[5] == 0) and np.all(codes[17] == 0) and np.all(codes[9, :64] == 0)


# ------------------------------------------------------------------ edge cases


def test_empty_inputs_write_nothing():
    W = torch.empty(0, 1024, dtype=torch.bfloat16, device=DEV)
    pk = torch.full((16,), 0xAB, dtype=torch.uint8, device=DEV)
    s = torch.full((4,), 7.0, dtype=torch.bfloat16, device=DEV)
    hqq.hqq_quantize(W, Wq_packed=pk, scale=s, zero=s)
    torch.cuda.synchronize()
    assert torch.all(pk == 0xAB) and torch.all(s == 7.0)


@pytest.mark.parametrize("nbits,G", [(3, 64), (4, 64), (2, 16), (1, 32), (8, 8)])
def test_no_write_past_outputs(nbits, G):
    rows, cols = 3, G * 5
    W = synthetic.weight(rows, cols, seed=15, dtype=torch.bfloat16, device=DEV)
    nb = hqq.hqq_packed_bytes(rows, cols, nbits)
    buf = torch.full((nb + 64,), 0xCD, dtype=torch.uint8, device=DEV)
    ng = rows * cols // G
    sbuf = torch.full((ng + 8,), 3.0, dtype=torch.bfloat16, device=DEV)
    zbuf = torch.full((ng + 8,), 3.0, dtype=torch.bfloat16, device=DEV)
    hqq.hqq_quantize(W, nbits, G, 1, Wq_packed=buf[:nb], scale=sbuf[:ng], zero=zbuf[:ng])
    torch.cuda.synchronize()
    assert torch.all(buf[nb:] == 0xCD)
    assert torch.all(sbuf[ng:] == 3.0) and torch.all(zbuf[ng:] == 3.0)
    if nbits == 3:  # 15 groups * 64 codes = 960 codes = 96 words exactly; bits 30-31 zero
        words = buf[:nb].view(torch.int32).cpu().numpy().view(np.uint32)
        assert np.all(words >> 30 == 0)


def test_three_bit_tail_word_is_zero_padded():
    W = synthetic.weight(3, 64, seed=16, dtype=torch.bfloat16, device=DEV)  # 192 codes
    pk, s, z = hqq.hqq_quantize(W, 3, 64, 1)
    words = pk.view(torch.int32).cpu().numpy().view(np.uint32)
    assert words.size == 20
    assert words[-1] >> 6 == 0  # only codes 190, 191 live in the last word


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_stored_meta_dtype_is_rounded_once(dtype):
    """Flat ABI: scale/zero stored in W's dtype = the fp32 values rounded to nearest even."""
    W = synthetic.weight(256, 1024, seed=17, dtype=dtype, device=DEV)
    pk, s, z = hqq.hqq_quantize(W, 4, 64, 1)
    params = hqq.make_params(4, 64, 1, w_dtype=dtype, meta_dtype=torch.float32)
    ref = hqq.hqq_quantize_ex(W, params)
    assert torch.equal(ref["Wq_packed"], pk)
    assert torch.equal(ref["scale"].to(dtype), s) and torch.equal(ref["zero"].to(dtype), z)
    # and the stored-dtype values against the oracle's fp32 results rounded the same way
    Wg = W.float().reshape(-1, 64).cpu().numpy()
    _, os_, oz = oracle.quantize(Wg, 4, 64, 1, 20, 0.7, 10.0, 1.01, nthreads=8)
    o_s = torch.from_numpy(os_).to(dtype)
    assert torch.equal(o_s, s.reshape(-1).cpu())
    o_z = torch.from_numpy(oz).to(dtype)
    assert (o_z != z.reshape(-1).cpu()).sum().item() <= 1e-4 * oz.size


@pytest.mark.parametrize("nbits,G,axis", [(8, 8, 1), (4, 64, 1), (4, 128, 0), (3, 64, 1),
                                          (3, 32, 0), (2, 16, 1), (2, 16, 0), (1, 32, 1),
                                          (1, 256, 0), (4, 256, 1)])
def test_packing_bit_exact_on_exact_grids(nbits, G, axis):
    # codes, step and zero known by construction (not from either implementation): the GPU
    # quantizer must reproduce them and pack them exactly as the oracle's packer does
    rows, cols = (4 * G, 320) if axis == 0 else (96, 5 * G)
    W, q, step, z = exact_grid_weights(rows, cols, nbits, G, axis, seed=nbits * 1000 + G)
    params = hqq.make_params(nbits, G, axis, w_dtype=torch.bfloat16, meta_dtype=torch.float32)
    out = hqq.hqq_quantize_ex(W, params)
    torch.cuda.synchronize()
    assert np.array_equal(out["Wq_packed"].cpu().numpy(), oracle.pack(q, nbits))
    assert np.array_equal(out["scale"].reshape(-1).cpu().numpy(), step)
    assert np.array_equal(out["zero"].reshape(-1).cpu().numpy(), z)


@pytest.mark.parametrize("nbits,G,axis", [(8, 32, 1), (4, 64, 1), (4, 64, 0), (3, 64, 1),
                                          (3, 16, 0), (2, 16, 1), (1, 32, 1), (1, 8, 0),
                                          (2, 16, 0), (2, 32, 0), (4, 16, 0), (8, 8, 0),
                                          (1, 64, 0)])
@pytest.mark.parametrize("out_dtype", ["f16", "bf16", "f32"])
def test_dequantize_bit_exact(nbits, G, axis, out_dtype):
    # axis 0 with 200 columns: the last 256-column unit of the column kernel is partial
    rows, cols = (3 * G + G, 200) if axis == 0 else (37, 12 * G)
    for meta in ("f32", "bf16", "f16"):
        dequant_parity(rows, cols, nbits, G, axis, out_dtype, meta_dtype=meta,
                       seed=nbits * 97 + G + axis)


@pytest.mark.parametrize("nbits,G,axis", [(4, 64, 1), (3, 64, 1), (2, 16, 0), (1, 32, 1)])
def test_dequantize_bit_exact_second_level(nbits, G, axis):
    rows, cols = (8 * G, 192) if axis == 0 else (64, 40 * G)
    for mg in (128, 100):
        dequant_parity(rows, cols, nbits, G, axis, "bf16", quant_meta=True, meta_group=mg,
                       seed=nbits + mg)


@pytest.mark.parametrize("side", ["scale", "zero"])
@pytest.mark.parametrize("nbits,G", [(3, 64), (1, 32), (4, 64)])
def test_dequantize_bit_exact_one_sided_second_level(nbits, G, side):
    # only one of scale / zero as 8-bit codes (runs of 128), the other stored in bf16
    dequant_parity(64, 40 * G, nbits, G, 1, "bf16", meta_dtype="bf16", meta_group=128,
                   seed=nbits * 7 + G, one_sided=side)


@pytest.mark.parametrize("rows,cols", [(16384, 8192), (4096, 11008)])
def test_dequantize_bit_exact_bench_layout(rows, cols):
    # 4-bit, group 64, axis 1, bf16 meta and output: the layout of the bench step (its
    # dedicated kernel), on full-size matrices
    dequant_parity(rows, cols, 4, 64, 1, "bf16", meta_dtype="bf16", seed=rows)


def test_quantize_meta_standalone():
    m = (torch.randn(1000, device=DEV) * 0.01 + 0.03).float()
    q, mm = hqq.hqq_quantize_meta(m, 128)
    oq, omm = oracle.quantize_meta(m.cpu().numpy(), 128)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(mm.cpu().numpy().view(np.uint32), omm.view(np.uint32))
    back = hqq.hqq_dequantize_meta(q, mm, 128)
    ob = oracle.dequantize_meta(oq, omm, 128)
    assert np.array_equal(back.cpu().numpy().view(np.uint32), ob.view(np.uint32))


def test_deterministic():
    W = synthetic.weight(1024, 4096, seed=19, dtype=torch.bfloat16, device=DEV)
    a = hqq.hqq_quantize(W, 4, 64, 1)
    b = hqq.hqq_quantize(W, 4, 64, 1)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_more_than_2_pow_32_elements():
    """[65536, 65600] bf16 (4.3e9 weights, 8.6 GB): 64-bit indexing end to end; groups at the
    start, across the 2^32-element boundary and at the end of the matrix are compared with
    the oracle under the same tolerances as every other workload."""
    rows, cols, G = 65536, 65600, 64
    W = torch.empty(rows, cols, dtype=torch.bfloat16, device=DEV)
    step = 2048
    for r0 in range(0, rows, step):
        W[r0:r0 + step] = synthetic.weight(step, cols, seed=20 + r0, dtype=torch.bfloat16,
                                           device=DEV)
    params = hqq.make_params(4, G, 1, w_dtype=torch.bfloat16, meta_dtype=torch.float32)
    out = hqq.hqq_quantize_ex(W, params)
    torch.cuda.synchronize()
    ng = rows * cols // G
    edge = 2 ** 32 // G  # first group past 2^32 elements
    ids = np.concatenate([np.arange(0, 4000), np.arange(edge - 6000, edge + 6000),
                          np.arange(ng - 10000, ng)]).astype(np.int64)
    ids_t = torch.from_numpy(ids).to(DEV)
    Wg = W.reshape(ng, G)[ids_t].float().cpu().numpy()
    per = G * 4 // 8
    pkg = out["Wq_packed"].reshape(ng, per)[ids_t].cpu().numpy()
    gc = np_unpack(pkg.ravel(), ids.size * G, 4).reshape(-1, G)
    gs = out["scale"].reshape(-1)[ids_t].cpu().numpy()
    gz = out["zero"].reshape(-1)[ids_t].cpu().numpy()
    r, *_ = judge(Wg, gc, gs, gz, 4, 20, 0.7, 10.0, 1.01)
    record("more_than_2_pow_32_elements", r)
    print(r.summary())
    r.check()
    del W, out
    torch.cuda.empty_cache()


def test_dequantize_axis0_column_kernel_large_and_ragged():
    # the config-3 layout (2-bit, group 16, axis 0) at a Llama shape, and a width that is not a
    # multiple of 8 (the element-wise kernel)
    dequant_parity(11008, 4096, 2, 16, 0, "bf16", meta_dtype="bf16", seed=3)
    dequant_parity(64, 4100, 2, 16, 0, "bf16", meta_dtype="bf16", seed=4)
