"""Seeded synthetic LLM-like weight matrices (inputs only; no quantization arithmetic).

Both the CUDA path and the CPU oracle take their inputs from here, so that both see the
same bits: a matrix is generated once (on the GPU for large sizes) and copied to the host
for the oracle.

Recipe (stands in for the Llama-7B / 70B-class weights the pages quantize, e.g. the
Llama-2-7B example of the "HQQ tutorial" (devpress.csdn.net) §3.2 and the Llama-7B row of
the benchmark table of the "Dropbox HQQ analysis" (ainews.cool); no real weights are used):
  - per row r: sigma_r = sigma_layer * exp(0.3 * N(0,1));
  - W[r, c] = sigma_r * N(0,1);
  - outliers: with probability `outlier_rate` an entry is multiplied by U(5, 20) with a
    random sign (the pages stress that LLM weights carry a few large outliers, "HQQ
    tutorial" §2);
  - the fp32 draw is rounded once to the storage dtype (bf16 or fp16).
sigma_layer is 0.02, or, for the whole-model workload, 0.02 * exp(0.3 * N(0,1)) drawn per
matrix from the matrix's own generator.
"""
from __future__ import annotations

import torch


def layer_sigma(seed: int, device="cpu") -> float:
    """Per-matrix sigma_layer = 0.02 * exp(0.3 * N(0,1)), from its own seeded stream."""
    g = torch.Generator(device=device)
    g.manual_seed(seed ^ 0x5EED)
    n = torch.randn(1, generator=g, device=device)
    return float(0.02 * torch.exp(0.3 * n).item())


def weight(rows: int, cols: int, *, seed: int, dtype=torch.bfloat16, outlier_rate: float = 0.001,
           sigma_layer: float = 0.02, device="cpu") -> torch.Tensor:
    """A [rows, cols] synthetic weight matrix of `dtype` on `device` (see module doc)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    sig = sigma_layer * torch.exp(0.3 * torch.randn(rows, 1, generator=g, device=device))
    W = torch.randn(rows, cols, generator=g, device=device)
    W.mul_(sig)
    if outlier_rate > 0:
        u = torch.rand(rows, cols, generator=g, device=device)
        mask = u < outlier_rate
        del u
        mag = torch.rand(rows, cols, generator=g, device=device)
        mag.mul_(15.0).add_(5.0)
        sgn = torch.rand(rows, cols, generator=g, device=device) < 0.5
        mag = torch.where(sgn, -mag, mag)
        del sgn
        W = torch.where(mask, W * mag, W)
        del mag, mask
    return W.to(dtype)


def activations(rows: int, cols: int, *, seed: int, dtype=torch.bfloat16,
                device="cpu") -> torch.Tensor:
    """Seeded layer inputs for the quantized linear layer: X[m, k] ~ N(0, 1), rounded once
    to dtype (stands in for a prefill batch of `rows` tokens; normalised hidden states of a
    Llama block have unit scale)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).to(dtype)
