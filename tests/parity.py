"""Helpers shared by the GPU parity tests: tolerances and input plumbing (no method arithmetic)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import synth

# Floating outputs: normwise max relative error 2e-3 (bf16 I/O, fp32 accumulate)
# for every stage fed the oracle's own inputs (teacher forcing).
TOL = 2e-3
# Composite paths (a whole block, a stack, decode loops) are not teacher-forced:
# one activation code that legitimately lands on the other side of a rounding tie
# in an inner stage moves a few outputs by ~1/|acc|, so they gate at 1e-2.
E2E_TOL = 1e-2
# Elements next to a rounding boundary of the storage type may land one or two
# units in the last place apart (fp32 vs fp64 evaluation before the rounding,
# or an upstream stored value that flipped); at most this fraction of them.
ULPS = 2
FLIP_FRACTION = 1e-3
# int8 activation codes: off by at most 1 on at most 0.01% of the elements.
CODE_FLIP_FRACTION = 1e-4

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    mant_bits = 7 if dtype == "bf16" else 23
    a = np.abs(np.asarray(ref, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - mant_bits)


def assert_close(gpu, ref, dtype: str, what: str = "", tol: float = TOL) -> float:
    """Compare a GPU tensor stored in `dtype` with the oracle's value rounded to `dtype`."""
    g = np.asarray(gpu, np.float64)
    r = O.store(np.asarray(ref, np.float64), dtype)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    err = np.abs(g - r)
    if r.size == 0:
        return 0.0
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    loose = tol * scale
    bound = loose + ULPS * ulp(r, dtype)
    bad = err > bound
    assert not np.any(bad), (f"{what}: {int(bad.sum())} elements beyond tolerance; worst err "
                             f"{float(err.max()):.3e} at ref scale {scale:.3e}")
    flips = int(np.count_nonzero(err > loose))
    assert flips <= max(1, int(FLIP_FRACTION * r.size)), f"{what}: {flips} rounding flips of {r.size}"
    return float(err.max() / scale) if scale > 0 else 0.0


def assert_codes_close(gpu_q, ref_q, what: str = "") -> int:
    d = np.abs(np.asarray(gpu_q, np.int64) - np.asarray(ref_q, np.int64))
    assert d.max(initial=0) <= 1, f"{what}: an activation code is off by {d.max()}"
    n = int(np.count_nonzero(d))
    assert n <= max(1, int(CODE_FLIP_FRACTION * d.size)), f"{what}: {n} code ties of {d.size}"
    return n


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64) if t.is_floating_point() else t.cpu().numpy()


def packed_to_np(packed: torch.Tensor) -> np.ndarray:
    return packed.cpu().numpy().view(np.uint32)


def make_layer(seed: int, n: int, k: int, device="cuda"):
    """(latent fp32 numpy, GPU TLinear, oracle TLinear built from the same latent)."""
    from ternary_weight_matmul_fusedbitlinear_b200 import quantize_weights
    W = synth.latent_weight(seed, n, k)
    lin = quantize_weights(W.to(device))
    return W.numpy(), lin, O.make_tlinear(W.numpy())


def make_block(seed: int, d: int, inner: int, layer: int = 0):
    """GPU Block + oracle Block from the same latents."""
    from ternary_weight_matmul_fusedbitlinear_b200 import Block, quantize_weights
    shapes = {"f": (d, d), "c": (d, d), "g": (d, d), "o": (d, d), "gate": (inner, d), "up": (inner, d),
              "down": (d, inner)}
    lins, lat = {}, {}
    for i, name in enumerate(synth.PROJ_NAMES):
        W = synth.latent_weight(synth.sub_seed(seed, layer, i), *shapes[name])
        lat[name] = W.numpy()
        lins[name] = quantize_weights(W.cuda())
    return Block(lins), O.make_block(lat)
