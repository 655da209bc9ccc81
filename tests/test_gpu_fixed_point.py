"""HQQ_FLAG_STOP_AT_FIXED_POINT changes no result bit: a warp stops iterating only when
every remaining evaluation of its groups would repeat the last one exactly."""
import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
from calibration_free_weight_hqq_b200 import synthetic

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbits,G,axis,dtype,p,beta0,kappa,iters", [
    (4, 64, 1, torch.bfloat16, 0.7, 10.0, 1.01, 20),
    (3, 64, 1, torch.bfloat16, 0.7, 10.0, 1.01, 20),
    (2, 16, 0, torch.bfloat16, 0.7, 10.0, 1.01, 20),
    (1, 32, 1, torch.float16, 0.7, 10.0, 1.01, 20),
    (8, 128, 1, torch.float32, 0.5, 3.0, 1.05, 57),
    (4, 64, 1, torch.bfloat16, 1.0, 10.0, 1.01, 20),
    (2, 16, 1, torch.float32, 0.7, 1.0, 1.1, 20),   # active shrinkage (sigma ~ 1)
])
def test_fixed_point_stop_is_bit_exact(nbits, G, axis, dtype, p, beta0, kappa, iters):
    sigma = 1.0 if beta0 == 1.0 else 0.02
    W = synthetic.weight(1024, 2048, seed=nbits * 7 + G, dtype=dtype, outlier_rate=0.01,
                         sigma_layer=sigma, device="cuda")
    outs = []
    for stop in (False, True):
        prm = hqq.make_params(nbits, G, axis, iters, p, beta0, kappa, w_dtype=dtype,
                              meta_dtype=torch.float32, stop_at_fixed_point=stop)
        outs.append(hqq.hqq_quantize_ex(W, prm))
    torch.cuda.synchronize()
    for k in ("Wq_packed", "scale", "zero"):
        assert torch.equal(outs[0][k].view(torch.uint8), outs[1][k].view(torch.uint8)), k


def test_fixed_point_stop_batched_model_block():
    shapes = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    Ws = [synthetic.weight(r, c, seed=300 + i, dtype=torch.bfloat16, device="cuda")
          for i, (r, c) in enumerate(shapes)]
    ref = hqq.hqq_quantize_batched(Ws, hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16))
    got = hqq.hqq_quantize_batched(Ws, hqq.make_params(4, 64, 1, w_dtype=torch.bfloat16,
                                                       stop_at_fixed_point=True))
    for a, b in zip(ref, got):
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
