"""Batched (whole-model) quantize/dequantize: each matrix of a batch must come out bit for
bit as the single-matrix calls produce it, whatever the batch composition (mixed shapes,
ragged tails, empty members, more matrices than one launch takes)."""
import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
from calibration_free_weight_hqq_b200 import synthetic

pytestmark = pytest.mark.gpu


def _check_batch(shapes, nbits, G, axis, dtype=torch.bfloat16, seed=0):
    Ws = [synthetic.weight(r, c, seed=seed + i, dtype=dtype, outlier_rate=0.01, device="cuda")
          for i, (r, c) in enumerate(shapes)]
    params = hqq.make_params(nbits, G, axis, w_dtype=dtype)
    outs = hqq.hqq_quantize_batched(Ws, params)
    D = hqq.hqq_dequantize_batched(outs, shapes, params, out_dtype=torch.float32)
    for W, (pk, s, z), d, (r, c) in zip(Ws, outs, D, shapes):
        pk1, s1, z1 = hqq.hqq_quantize(W, nbits, G, axis)
        assert torch.equal(pk, pk1) and torch.equal(s, s1) and torch.equal(z, z1)
        d1 = hqq.hqq_dequantize(pk1, s1, z1, r, c, nbits, G, axis, out_dtype=torch.float32)
        assert torch.equal(d, d1)


@pytest.mark.parametrize("nbits,G,axis", [(4, 64, 1), (3, 64, 1), (2, 16, 0), (1, 32, 1),
                                          (8, 128, 1), (4, 256, 0)])
def test_batched_equals_single(nbits, G, axis):
    if axis == 1:
        shapes = [(37, 4 * G), (512, 8 * G), (0, 4 * G), (3, G), (1000, 2 * G)]
    else:
        shapes = [(4 * G, 37), (8 * G, 512), (0, 40), (G, 3), (2 * G, 1000)]
    _check_batch(shapes, nbits, G, axis)


def test_batch_larger_than_one_launch():
    shapes = [(8, 64 * (1 + i % 3)) for i in range(300)]  # 300 > 256 matrices per launch
    _check_batch(shapes, 4, 64, 1, seed=100)


def test_batched_model_block_fp16():
    shapes = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    _check_batch(shapes, 4, 64, 1, dtype=torch.float16, seed=200)
