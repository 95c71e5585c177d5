"""Seeded synthetic inputs for the MatMul-free block forward.

This module is shared by the CPU oracle tests and the CUDA path's tests and
benchmark. It draws random numbers and nothing else: it holds none of the
method's arithmetic (no norm, no quantisation, no scan). Every tensor it
returns lives on the host unless a CUDA generator is asked for explicitly.

Shapes follow the 370M / 1.3B / 2.7B model family named in the project review
"MatMul-Free LM: using ternary weights and gated recurrence to take matrix
multiplication out of language models" (hysenlabs), section "Install and model
initialisation" (default hidden 2048, 24 layers; model zoo 370M / 1.3B / 2.7B).

Recipe (the same for every caller):
  * latent weights  W ~ N(0, 0.02^2), fp32, one independent stream per matrix,
    sub-seed = seed * 4096 + layer * 16 + proj;
  * activations     x ~ N(0, 1), optionally with each element multiplied by 20
    independently with probability 0.001 ("outliers"), then rounded to the
    run dtype (fp32 or bf16) by torch;
  * norm gains      1, biases 0, initial state h0 = 0 unless a test says otherwise.
"""
from __future__ import annotations

import dataclasses

import torch

# projection indices used in the sub-seed
PROJ_F, PROJ_C, PROJ_G, PROJ_O, PROJ_GATE, PROJ_UP, PROJ_DOWN = range(7)
PROJ_NAMES = ("f", "c", "g", "o", "gate", "up", "down")
ACT_SEED_OFFSET = 4095  # sub-seed slot used for the activations of a config


def sub_seed(seed: int, layer: int, proj: int) -> int:
    return seed * 4096 + layer * 16 + proj


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def latent_weight(seed: int, n: int, k: int, std: float = 0.02,
                  device: str = "cpu") -> torch.Tensor:
    """fp32 [n, k] latent weight drawn from N(0, std^2)."""
    g = _gen(seed, device)
    return torch.randn(n, k, generator=g, dtype=torch.float32, device=device) * std


def activations(seed: int, m: int, k: int, dtype: torch.dtype = torch.float32,
                outlier_p: float = 0.0, outlier_scale: float = 20.0,
                device: str = "cpu") -> torch.Tensor:
    """[m, k] activations ~ N(0,1) with optional sparse x20 outliers, in `dtype`."""
    g = _gen(seed, device)
    x = torch.randn(m, k, generator=g, dtype=torch.float32, device=device)
    if outlier_p > 0.0:
        u = torch.rand(m, k, generator=g, dtype=torch.float32, device=device)
        x = torch.where(u < outlier_p, x * outlier_scale, x)
    return x.to(dtype)


def preacts(seed: int, b: int, t: int, d: int, dtype: torch.dtype = torch.float32,
            scale: float = 1.0, device: str = "cpu") -> torch.Tensor:
    """[b, t, 3, d] gate pre-activations (f~, c~, g~) ~ N(0, scale^2) for scan-only tests."""
    g = _gen(seed, device)
    x = torch.randn(b, t, 3, d, generator=g, dtype=torch.float32, device=device) * scale
    return x.to(dtype)


def gains(seed: int, d: int, spread: float = 0.1, device: str = "cpu") -> torch.Tensor:
    """fp32 [d] norm gain ~ 1 + N(0, spread^2), for tests of a learned (non-unit) gain."""
    g = _gen(seed, device)
    return 1.0 + spread * torch.randn(d, generator=g, dtype=torch.float32, device=device)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic workload (no arithmetic, only sizes)."""
    name: str
    d: int            # hidden size
    inner: int        # GLU inner size
    layers: int
    batch: int
    seq: int          # prefill / prompt length
    decode_steps: int
    dtype: str        # "f32" or "bf16"
    seed: int


# The tiny block, the three model-shaped stacks and the GEMV sweep.
TINY_BLOCK = Workload("tiny_block_d256_i768_b2_t64_f32", 256, 768, 1, 2, 64, 0, "f32", 1000)
STACK_370M = Workload("stack370m_prefill_d1024_i2816_l24_b8_t2048_bf16", 1024, 2816, 24, 8, 2048, 0, "bf16", 1002)
STACK_1P3B = Workload("stack1p3b_d2048_i5632_l24_b4_t2048_dec256_bf16", 2048, 5632, 24, 4, 2048, 256, "bf16", 1003)
STACK_2P7B = Workload("stack2p7b_d2560_i6912_l32_prompt512_dec512_bf16", 2560, 6912, 32, 1, 512, 512, "bf16", 1004)
STACK_2P7B_BATCHES = (1, 8, 64)

GEMV_SWEEP_SEED = 1001
GEMV_SWEEP_SHAPES = ((2048, 2048), (2048, 5632), (5632, 2048))  # (K, N): K -> N
GEMV_SWEEP_TOKENS = (1, 4, 16)
GEMV_OUTLIER_P = 0.001
GEMV_OUTLIER_SCALE = 20.0
