"""hqq_quantize_ex_noalloc: the second-level quantize path without a caller workspace.

It is meant for callers that cannot allocate device memory themselves (a plugin handed only
a stream and tensors, code under a foreign allocator or fixed pool, a serving process that
forbids allocation after start-up); its scratch is a fixed array inside the library. These
tests call it through the C ABI and check that its outputs equal those of hqq_quantize_ex
with a caller-allocated workspace, on two calls in a row (the array keeps the previous
call's contents, which must not leak into the next result), and that a call needing more
scratch than the array holds is refused before anything runs.

This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import calibration_free_weight_hqq_b200 as hqq
from calibration_free_weight_hqq_b200 import synthetic

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 32 << 20
HQQ_ERR_WORKSPACE = 6


def _outputs(W, params):
    rows, cols = W.shape
    ng = rows * cols // params.group_size
    runs = (ng + params.meta_group_size - 1) // params.meta_group_size
    dev = W.device
    return {
        "Wq_packed": torch.full((hqq.hqq_packed_bytes(rows, cols, params.nbits),), 0x5A,
                                dtype=torch.uint8, device=dev),
        "scale": torch.full((ng,), 0x5A, dtype=torch.uint8, device=dev),
        "zero": torch.full((ng,), 0x5A, dtype=torch.uint8, device=dev),
        "scale_mm": torch.full((runs, 2), -7.0, dtype=torch.float32, device=dev),
        "zero_mm": torch.full((runs, 2), -7.0, dtype=torch.float32, device=dev),
    }


def _noalloc(W, params, out):
    rows, cols = W.shape
    return hqq.lib().hqq_quantize_ex_noalloc(
        W.data_ptr(), rows, cols, ctypes.byref(params), out["Wq_packed"].data_ptr(),
        out["scale"].data_ptr(), out["zero"].data_ptr(), out["scale_mm"].data_ptr(),
        out["zero_mm"].data_ptr(), torch.cuda.current_stream().cuda_stream)


def _with_workspace(W, params, out):
    rows, cols = W.shape
    need = hqq.hqq_workspace_bytes(rows, cols, params)
    ws = torch.empty(need, dtype=torch.uint8, device=W.device)
    return hqq.lib().hqq_quantize_ex(
        W.data_ptr(), rows, cols, ctypes.byref(params), out["Wq_packed"].data_ptr(),
        out["scale"].data_ptr(), out["zero"].data_ptr(), out["scale_mm"].data_ptr(),
        out["zero_mm"].data_ptr(), ws.data_ptr(), need, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_path_on_two_calls_in_a_row():
    cases = [
        # (rows, cols, nbits, group, seed): the second call is smaller than the first, so
        # stale scratch from the first call lies beyond what the second one writes
        (4096, 2048, 3, 64, 31),
        (1024, 1024, 4, 64, 32),
    ]
    for rows, cols, nbits, G, seed in cases:
        W = synthetic.weight(rows, cols, seed=seed, dtype=torch.bfloat16, device="cuda")
        params = hqq.make_params(nbits, G, 1, w_dtype=torch.bfloat16, quant_scale=True,
                                 quant_zero=True, meta_group_size=128)
        assert hqq.hqq_workspace_bytes(rows, cols, params) <= NOALLOC_SCRATCH_BYTES
        ref, got = _outputs(W, params), _outputs(W, params)
        assert _with_workspace(W, params, ref) == 0
        assert _noalloc(W, params, got) == 0
        torch.cuda.synchronize()
        # identical arithmetic on identical inputs: every output must match bit for bit
        for k in ref:
            assert torch.equal(ref[k].view(torch.uint8), got[k].view(torch.uint8)), k


def test_noalloc_refuses_sizes_beyond_its_scratch():
    params = hqq.make_params(1, 32, 1, w_dtype=torch.bfloat16, quant_scale=True,
                             quant_zero=True)
    rows, cols = 28672, 8192  # 7,340,032 groups of 32: 59 MB of scratch needed
    assert hqq.hqq_workspace_bytes(rows, cols, params) > NOALLOC_SCRATCH_BYTES
    W = torch.empty((1, 1), dtype=torch.bfloat16, device="cuda")  # never read: refused first
    pk = torch.full((16,), 0x33, dtype=torch.uint8, device="cuda")
    st = hqq.lib().hqq_quantize_ex_noalloc(W.data_ptr(), rows, cols, ctypes.byref(params),
                                           pk.data_ptr(), pk.data_ptr(), pk.data_ptr(),
                                           pk.data_ptr(), pk.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == HQQ_ERR_WORKSPACE
    assert torch.all(pk == 0x33)
