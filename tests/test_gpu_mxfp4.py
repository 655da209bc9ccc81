"""GPU parity of the MXFP4 weight-only encoding against the oracle: codes, scales and the
decoded values must be bit-identical (the encoding is a deterministic rounding; both sides
scale by an exact power of two and round once to the E2M1 grid, the kernel with the hardware
conversion, the oracle with a nearest-value search written from the definition)."""
import numpy as np
import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
import oracle
from calibration_free_weight_hqq_b200 import synthetic

pytestmark = pytest.mark.gpu


def run(W):
    codes, scales = hqq.hqq_mxfp4_quantize(W.cuda())
    torch.cuda.synchronize()
    return codes.cpu().numpy().ravel(), scales.cpu().numpy().ravel()


def check(W, rows_sample=None):
    rows, cols = W.shape
    codes, scales = run(W)
    Wf = W.float().numpy()
    if rows_sample is not None:
        sub = Wf[rows_sample]
        oc, osc = oracle.mxfp4_quantize(sub)
        codes = codes.reshape(rows, cols // 2)[rows_sample].ravel()
        scales = scales.reshape(rows, cols // 32)[rows_sample].ravel()
    else:
        oc, osc = oracle.mxfp4_quantize(Wf)
    assert np.array_equal(scales, osc)
    assert np.array_equal(codes, oc), np.flatnonzero(codes != oc)[:10]
    return oc, osc


@pytest.mark.parametrize("rows,cols,dtype", [
    (257, 4096, torch.bfloat16),
    (3, 96, torch.bfloat16),      # 288 elements: the last warp is partial
    (1, 32, torch.float16),
    (129, 1024, torch.float16),
    (65, 512, torch.float32),
])
def test_mxfp4_random_matches_oracle(rows, cols, dtype):
    W = synthetic.weight(rows, cols, seed=rows + cols, dtype=dtype)
    oc, osc = check(W)
    dev_c = torch.from_numpy(oc).cuda()
    dev_s = torch.from_numpy(osc).cuda()
    want = oracle.mxfp4_dequantize(oc, osc, rows, cols)
    for od, name in ((torch.bfloat16, "bf16"), (torch.float16, "f16"), (torch.float32, "f32")):
        out = hqq.hqq_mxfp4_dequantize(dev_c, dev_s, rows, cols, od)
        torch.cuda.synchronize()
        assert np.array_equal(out.float().cpu().numpy(), oracle.round_to_dtype(want, name)), name


def test_mxfp4_ties_saturation_zeros_and_extremes():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    blocks = []
    for e in (-20, -3, 0, 5, 60):
        s = 2.0 ** e
        b = [6.0 * s] + [t * s for t in ties] + [-t * s for t in ties] + \
            [g * s for g in grid] + [7.5 * s, -7.9 * s, -0.0, 0.1 * s, -0.1 * s, 3.2 * s,
                                      4.9 * s, 5.1 * s, 0.0]
        blocks.append(b[:32])
    blocks.append([0.0] * 32)                              # all-zero block: e = -127
    blocks.append([-0.0] * 31 + [0.0])                     # negative zeros
    blocks.append([2.0 ** -133 * k for k in range(32)])   # bf16 subnormals: e clamps to -127
    blocks.append([2.0 ** 120 * (k - 16) / 4 for k in range(32)])  # huge values
    W = torch.tensor(np.array(blocks, np.float32)).to(torch.bfloat16)
    check(W)
    check(torch.tensor(np.array(blocks[:5], np.float32)))  # the same in fp32 input


def test_mxfp4_70b_mlp_shape_sampled_and_round_trip():
    rows, cols = 28672, 8192
    W = synthetic.weight(rows, cols, seed=3, dtype=torch.bfloat16, device="cuda")
    codes, scales = hqq.hqq_mxfp4_quantize(W)
    back = hqq.hqq_mxfp4_dequantize(codes, scales, rows, cols)
    torch.cuda.synchronize()
    rs = np.sort(np.random.default_rng(4).choice(rows, 64, replace=False))
    Wf = W[torch.from_numpy(rs).cuda()].float().cpu().numpy()
    oc, osc = oracle.mxfp4_quantize(Wf)
    assert np.array_equal(codes[torch.from_numpy(rs).cuda()].cpu().numpy().ravel(), oc)
    assert np.array_equal(scales[torch.from_numpy(rs).cuda()].cpu().numpy().ravel(), osc)
    want = oracle.round_to_dtype(oracle.mxfp4_dequantize(oc, osc, 64, cols), "bf16")
    assert np.array_equal(back[torch.from_numpy(rs).cuda()].float().cpu().numpy(), want)


def test_mxfp4_empty():
    W = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    c, s = hqq.hqq_mxfp4_quantize(W)
    assert c.numel() == 0 and s.numel() == 0
