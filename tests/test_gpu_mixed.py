"""Per-layer mixed precision in one call (hqq_quantize_mixed / hqq_dequantize_mixed): each
matrix must come out bit for bit as the single-matrix calls produce it with its own
configuration, whatever the mix; and one matrix of each configuration is checked against the
oracle directly. The configurations follow the pages' recipes: 8-bit group 128 for the first
block and the output head, 4-bit group 64 elsewhere ("HQQ tutorial" §4.2, layer_configs); 4-bit
attention and 2-bit MLP weights ("hqq-quantization skill summary", dynamic_config)."""
import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
from calibration_free_weight_hqq_b200 import synthetic
from parity import compare

pytestmark = pytest.mark.gpu


def _model(dtype, meta_dtype=None):
    c8 = hqq.make_params(8, 128, 1, w_dtype=dtype, meta_dtype=meta_dtype)
    c4 = hqq.make_params(4, 64, 1, w_dtype=dtype, meta_dtype=meta_dtype)
    c2 = hqq.make_params(2, 16, 1, w_dtype=dtype, meta_dtype=meta_dtype)
    c3a0 = hqq.make_params(3, 64, 0, w_dtype=dtype, meta_dtype=meta_dtype)
    # (shape, config): first block 8-bit, attention 4-bit, MLP 2-bit, a 3-bit axis-0 layer,
    # an empty member and the output head 8-bit; configurations interleaved
    layers = [((256, 512), c8), ((384, 256), c8), ((256, 256), c4), ((520, 256), c2),
              ((256, 768), c2), ((256, 256), c4), ((192, 320), c3a0), ((0, 256), c4),
              ((37, 640), c4), ((512, 256), c8)]
    Ws = [synthetic.weight(r, c, seed=300 + i, dtype=dtype, outlier_rate=0.01, device="cuda")
          for i, ((r, c), _) in enumerate(layers)]
    return Ws, [p for _, p in layers]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_mixed_equals_single_per_matrix(dtype):
    Ws, cfgs = _model(dtype)
    assert hqq.hqq_mixed_plan(cfgs)[1] == 4
    outs = hqq.hqq_quantize_mixed(Ws, cfgs)
    shapes = [tuple(W.shape) for W in Ws]
    D = hqq.hqq_dequantize_mixed(outs, shapes, cfgs, out_dtype=torch.float32)
    for W, p, (pk, s, z), d, (r, c) in zip(Ws, cfgs, outs, D, shapes):
        one = hqq.hqq_quantize_ex(W, p)
        assert torch.equal(pk, one["Wq_packed"])
        assert torch.equal(s.reshape(-1), one["scale"].reshape(-1))
        assert torch.equal(z.reshape(-1), one["zero"].reshape(-1))
        d1 = hqq.hqq_dequantize_ex(one, r, c, p, out_dtype=torch.float32)
        assert torch.equal(d, d1)


def test_mixed_matches_oracle_per_configuration():
    # fp32 meta (the oracle's precision): the mixed call's outputs equal the single-matrix
    # call's, which compare() checks against the oracle group by group
    Ws, cfgs = _model(torch.bfloat16, meta_dtype=torch.float32)
    outs = hqq.hqq_quantize_mixed(Ws, cfgs)
    seen = set()
    for i, (W, p, (pk, s, z)) in enumerate(zip(Ws, cfgs, outs)):
        key = (p.nbits, p.group_size, p.axis)
        if key in seen or W.numel() == 0:
            continue
        seen.add(key)
        one = hqq.hqq_quantize_ex(W, p)
        assert torch.equal(pk, one["Wq_packed"]) and torch.equal(s.reshape(-1), one["scale"].reshape(-1))
        r = compare(W, p.nbits, p.group_size, p.axis, n_sample=4000, seed=i)
        r.check()
    assert len(seen) == 4
