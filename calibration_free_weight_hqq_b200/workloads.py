"""The five shipped workloads (shapes and quantization settings; no arithmetic).

Shapes follow the Llama-7B-class models the pages quantize ("HQQ tutorial"
(devpress.csdn.net) §3.2 Llama-2-7B with nbits=4, group_size=64; "Dropbox HQQ analysis"
(ainews.cool) benchmark table, Llama-7B), the single Linear(1024, 4096) fp16 layer of the
"HQQ calibration-free guide" (lnwmold.com) §3.2, its 2-bit/group 16 advice
("HQQ量化 skill page" (aitishiku.com), known pitfalls) and a 70B-class MLP shape.
Solver constants: iters=20, p=0.7, beta0=10, kappa=1.01 throughout.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple

import torch

ITERS, P, BETA0, KAPPA = 20, 0.7, 10.0, 1.01

BLOCK_SHAPES: List[Tuple[str, int, int]] = [
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
]


@dataclass
class Matrix:
    name: str
    rows: int
    cols: int
    seed: int
    dtype: torch.dtype
    nbits: int
    group_size: int
    axis: int
    outlier_rate: float = 0.001
    per_layer_sigma: bool = False
    quant_meta: bool = False      # quant_scale and quant_zero (8-bit, runs of 128)
    meta_group_size: int = 128
    iters: int = ITERS
    p: float = P
    beta0: float = BETA0
    kappa: float = KAPPA

    @property
    def numel(self) -> int:
        return self.rows * self.cols


@dataclass
class Workload:
    name: str
    description: str
    matrices: List[Matrix] = field(default_factory=list)

    @property
    def weights(self) -> int:
        return sum(m.numel for m in self.matrices)


def _base_seed(config: int) -> int:
    return 1234 + config * 100


def single_fp16() -> Workload:
    s = _base_seed(1)
    return Workload("single_4096x1024_fp16_4b_g64",
                    "one [4096,1024] fp16 weight, 4-bit, group 64, axis 1, fp16 scale/zero",
                    [Matrix("linear", 4096, 1024, s, torch.float16, 4, 64, 1)])


def llama7b_block_4b() -> Workload:
    s = _base_seed(2)
    return Workload("llama7b_block_bf16_4b_g64",
                    "one Llama-7B-shaped decoder block, bf16, 4-bit, group 64, axis 1",
                    [Matrix(n, r, c, s + i, torch.bfloat16, 4, 64, 1)
                     for i, (n, r, c) in enumerate(BLOCK_SHAPES)])


def llama7b_block_2b_axis0() -> Workload:
    s = _base_seed(3)
    return Workload("llama7b_block_bf16_2b_g16_axis0",
                    "one Llama-7B-shaped block, bf16, 2-bit, group 16, axis 0, 0.5% outliers",
                    [Matrix(n, r, c, s + i, torch.bfloat16, 2, 16, 0, outlier_rate=0.005)
                     for i, (n, r, c) in enumerate(BLOCK_SHAPES)])


def mlp70b_mixed() -> Workload:
    s = _base_seed(4)
    return Workload("mlp70b_28672x8192_3b_g64_1b_g32_meta8",
                    "[28672,8192] bf16: 3-bit g64 and 1-bit g32, axis 1, 8-bit scale/zero g128",
                    [Matrix("mlp_3b_g64", 28672, 8192, s, torch.bfloat16, 3, 64, 1,
                            quant_meta=True),
                     Matrix("mlp_1b_g32", 28672, 8192, s, torch.bfloat16, 1, 32, 1,
                            quant_meta=True)])


def llama7b_model_4b() -> Workload:
    s = _base_seed(5)
    mats = []
    for layer in range(32):
        for i, (n, r, c) in enumerate(BLOCK_SHAPES):
            idx = layer * len(BLOCK_SHAPES) + i
            mats.append(Matrix(f"layers.{layer}.{n}", r, c, s + idx, torch.bfloat16, 4, 64, 1,
                               per_layer_sigma=True))
    return Workload("llama7b_model_bf16_4b_g64",
                    "whole Llama-7B-shaped model: 32 blocks x 7 linear weights, bf16, 4-bit, "
                    "group 64, axis 1, per-matrix sigma", mats)


def llama7b_model_mixed() -> Workload:
    """The whole Llama-7B-shaped model with per-layer configurations after the pages' recipes:
    block 0 at 8 bits, group 128 ("HQQ tutorial" §4.2, layer_configs: the first block and the
    output head at 8 bits, the rest at 4 bits, group 64); in blocks 1-31 the attention
    projections at 4 bits, group 64, and the MLP at 2 bits, group 16 ("hqq-quantization skill
    summary", dynamic_config: attention 4-bit, MLP 2-bit; "HQQ量化 skill page": 2 bits want
    group 16). Same shapes and seeds as the uniform 4-bit model."""
    s = _base_seed(5)
    mats = []
    for layer in range(32):
        for i, (n, r, c) in enumerate(BLOCK_SHAPES):
            idx = layer * len(BLOCK_SHAPES) + i
            nbits, G = (8, 128) if layer == 0 else (4, 64) if i < 4 else (2, 16)
            mats.append(Matrix(f"layers.{layer}.{n}", r, c, s + idx, torch.bfloat16, nbits, G, 1,
                               per_layer_sigma=True))
    return Workload("llama7b_model_bf16_mixed_8b_4b_2b",
                    "whole Llama-7B-shaped model, bf16, axis 1: block 0 8-bit g128, attention "
                    "4-bit g64, MLP 2-bit g16 (blocks 1-31)", mats)


ALL = {1: single_fp16, 2: llama7b_block_4b, 3: llama7b_block_2b_axis0, 4: mlp70b_mixed,
       5: llama7b_model_4b}


def make_weight(m: Matrix, device="cpu") -> torch.Tensor:
    """Synthetic weight for one matrix of a workload (see ``synthetic``)."""
    from . import synthetic
    sigma = synthetic.layer_sigma(m.seed) if m.per_layer_sigma else 0.02
    return synthetic.weight(m.rows, m.cols, seed=m.seed, dtype=m.dtype,
                            outlier_rate=m.outlier_rate, sigma_layer=sigma, device=device)
