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
# A value within this relative distance of a midpoint between two neighbours of
# the storage type is a rounding tie for the kernels' fp32 arithmetic: fp32
# evaluation may land on the midpoint itself and round to even, the oracle's
# fp64 evaluation on either side, so both neighbours are correct results.
TIE_REL = 2.0 ** -21
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
    flips = (err > loose) & ~((err <= ulp(r, dtype)) & near_tie(ref, dtype))
    n = int(np.count_nonzero(flips))
    assert n <= max(1, int(FLIP_FRACTION * r.size)), f"{what}: {n} rounding flips of {r.size}"
    return float(err.max() / scale) if scale > 0 else 0.0


def near_tie(ref, dtype: str) -> np.ndarray:
    """Whether each unrounded reference value lies within TIE_REL of a rounding midpoint of `dtype`."""
    a = np.abs(np.asarray(ref, np.float64))
    u = ulp(a, dtype)
    mid = (np.floor(a / u) + 0.5) * u
    return np.abs(a - mid) <= TIE_REL * a


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


def normwise(gpu, ref) -> float:
    """max|gpu - ref| / max|ref| (the drift figure of composite paths)."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    return float(np.max(np.abs(g - r)) / scale) if scale > 0 else 0.0


def record_drift(name: str, data) -> None:
    """Write drift figures to $MMF_DRIFT_OUT/<name>.json when that directory is given."""
    import json
    import os
    out = os.environ.get("MMF_DRIFT_OUT")
    if out:
        os.makedirs(out, exist_ok=True)
        with open(os.path.join(out, f"{name}.json"), "w") as f:
            json.dump(data, f, indent=1)


def make_block(seed: int, d: int, inner: int, layer: int = 0, cache: bool = False, gnorm: bool = False):
    """GPU Block + oracle Block from the same latents (gnorm: with a seeded g_norm gain)."""
    from ternary_weight_matmul_fusedbitlinear_b200 import Block, quantize_weights
    shapes = {"f": (d, d), "c": (d, d), "g": (d, d), "o": (d, d), "gate": (inner, d), "up": (inner, d),
              "down": (d, inner)}
    lins, lat = {}, {}
    for i, name in enumerate(synth.PROJ_NAMES):
        W = synth.latent_weight(synth.sub_seed(seed, layer, i), *shapes[name])
        lat[name] = W.numpy()
        lins[name] = quantize_weights(W.cuda())
    gain = synth.gains(synth.sub_seed(seed, layer, 7), d) if gnorm else None
    return (Block(lins, None if gain is None else gain.cuda()),
            O.make_block(lat, cache=cache, gnorm=None if gain is None else gain.numpy()))


def scan_ref(pf, pc, pg, h0, oblk):
    """The oracle's scan with the block's output gate (sigmoid, or g_norm when the block has a gain)."""
    if oblk.gnorm is None:
        return O.mlgru_scan(pf, pc, pg, h0)
    return O.mlgru_scan_gnorm(pf, pc, pg, h0, oblk.gnorm)


def check_block_stages(x, h0, y, hT, dbg, oblk, dtype: str, what: str = "", seqs=None) -> dict:
    """Teacher-forced parity of one block call, stage by stage, at TOL.

    Every oracle stage is fed the GPU's own stored input to that stage (x, the
    stored pre-activations, o', y1, p), so a rounding tie in one stage cannot
    move the next; the codes must be within 1 LSB of the oracle's on <= 0.01%
    of elements, and each oracle contraction then uses the GPU's codes (a code
    at a tie moves every output of its contraction by a little). ``seqs`` restricts the check
    to some sequences of the batch (sequences are independent).
    Arrays: x [B,T,d] (GPU input, torch), h0 [B,d] fp64, y [B,T,d], hT [B,d],
    dbg the dict of block_forward_debug. Returns the per-stage max relative errors.
    """
    sel = slice(None) if seqs is None else seqs
    B, T, d = x.shape
    xn = O.store(to_np(x[sel]), dtype)
    Bs = xn.shape[0]
    pre = to_np(dbg["pre"][sel])
    og, y1, p = (to_np(dbg[k][sel]) for k in ("og", "y1", "p"))
    yg, hg = to_np(y[sel]), np.asarray(hT, np.float64)[sel]
    h0 = np.asarray(h0, np.float64)[sel]

    def rows(t, k):   # the selected sequences' rows of a [B*T, k] debug tensor, as numpy
        return to_np(t.reshape(B, T, k)[sel].reshape(Bs * T, k))

    errs = {}
    tag = f"{what}: " if what else ""
    # codes and scale of each quantised input: within 1 LSB on <= 0.01% of the
    # codes (rounding ties) and the same scale; the oracle's contractions below
    # then take the GPU's codes, so that a tie in one stage cannot move the
    # comparison of that stage's outputs
    lins = [(oblk.f, xn, 0), (oblk.o, og, 1), (oblk.gate, y1, 2), (oblk.down, p, 3)]
    qg = []
    for lin, inp, i in lins:
        _, parts = O.bitlinear(inp, lin, parts=True)
        q = rows(dbg["q"][i], lin.K)
        s = rows(dbg["s"][i].reshape(-1, 1), 1)[:, 0]
        assert_codes_close(q, parts["q"], f"{tag}codes of input {i}")
        np.testing.assert_allclose(s, parts["s"], rtol=1e-6, err_msg=f"{tag}scale of input {i}")
        qg.append(q)
    # 1. f|c|g on x
    for j, (lin, name) in enumerate(((oblk.f, "f~"), (oblk.c, "c~"), (oblk.g, "g~"))):
        errs[name] = assert_close(pre[:, :, j], _forced_bitlinear(xn, lin, qg[0], tag + "codes of x"), dtype,
                                  tag + name)
    # 2. gates and scan on the stored pre-activations
    o_ref, h_ref = scan_ref(pre[:, :, 0], pre[:, :, 1], pre[:, :, 2], h0, oblk)
    errs["o'"] = assert_close(og, o_ref, dtype, tag + "o'")
    errs["h_T"] = assert_close(hg, h_ref, "f32", tag + "h_T")
    # 3. o projection + residual on the stored o'
    errs["y1"] = assert_close(y1, xn + _forced_bitlinear(og, oblk.o, qg[1], tag + "codes of o'"), dtype, tag + "y1")
    # 4. gate|up and SiLU gate on the stored y1
    gate = _forced_bitlinear(y1, oblk.gate, qg[2], tag + "codes of y1")
    up = _forced_bitlinear(y1, oblk.up, qg[2], tag + "codes of y1")
    errs["p"] = assert_close(p, O.silu(gate) * up, dtype, tag + "p")
    # 5. down projection + residual on the stored p and y1
    errs["y"] = assert_close(yg, y1 + _forced_bitlinear(p, oblk.down, qg[3], tag + "codes of p"), dtype, tag + "y")
    return errs


def _forced_bitlinear(x, lin, q_gpu, what: str):
    """The oracle's BitLinear on its own input x, except that the int8 codes are the GPU's: they must be
    within 1 of the oracle's own codes on <= 0.01% of elements (rounding ties), and are then used as is."""
    x = np.asarray(x, np.float64)
    lead = x.shape[:-1]
    xhat = O.rmsnorm(x.reshape(-1, x.shape[-1]), lin.gain)
    q, s = O.absmax_quantize(xhat)
    assert_codes_close(q_gpu, q, what)
    y = O.rescale(O.ternary_accumulate(q_gpu, lin.weights()), lin.gamma, s, lin.bias)
    return y.reshape(*lead, lin.N)


def check_block_tie_forced(x, h0, y, hT, dbg, oblk, dtype: str, what: str = "", seqs=None) -> dict:
    """One block end to end at TOL with only the integer tie decisions taken from the GPU.

    The oracle runs the whole block from the GPU's input x and initial state
    with its own floating-point values throughout (pre-activations, scan, o',
    y1, p); at each of the four quantisations it takes the GPU's int8 codes,
    which must equal its own except at rounding ties (<= 0.01% of elements,
    off by one). The block's output and final state are then compared at TOL.
    """
    sel = slice(None) if seqs is None else seqs
    B, T, d = x.shape
    xn = O.store(to_np(x[sel]), dtype)
    Bs = xn.shape[0]
    h0 = np.asarray(h0, np.float64)[sel]

    def q_of(i, k):
        return dbg["q"][i].reshape(B, T, k)[sel].reshape(Bs * T, k).cpu().numpy()

    tag = f"{what}: " if what else ""
    q0 = q_of(0, d)
    pf = O.store(_forced_bitlinear(xn, oblk.f, q0, tag + "codes of x"), dtype)
    pc = O.store(_forced_bitlinear(xn, oblk.c, q0, tag + "codes of x"), dtype)
    pg = O.store(_forced_bitlinear(xn, oblk.g, q0, tag + "codes of x"), dtype)
    og, h_ref = scan_ref(pf, pc, pg, h0, oblk)
    og = O.store(og, dtype)
    y1 = O.store(xn + _forced_bitlinear(og, oblk.o, q_of(1, d), tag + "codes of o'"), dtype)
    q2 = q_of(2, d)
    u = _forced_bitlinear(y1, oblk.gate, q2, tag + "codes of y1")
    v = _forced_bitlinear(y1, oblk.up, q2, tag + "codes of y1")
    p = O.store(O.silu(u) * v, dtype)
    y_ref = y1 + _forced_bitlinear(p, oblk.down, q_of(3, oblk.inner), tag + "codes of p")
    return {"y": assert_close(to_np(y[sel]), y_ref, dtype, tag + "y (tie-forced block)"),
            "h_T": assert_close(np.asarray(hT, np.float64)[sel], h_ref, "f32", tag + "h_T (tie-forced block)")}
