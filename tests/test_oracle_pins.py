"""Pins for the CPU oracle: closed forms, hand-built cases, brute force, library routines.

Each test pins an oracle function to something other than itself, chosen so
that a plausible slip (dropped term, wrong sign or index, swapped operand)
fails at least one of them. CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.stats import norm as _norm

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_random_fp32():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 8)
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.to(torch.float64).numpy())
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 is exactly halfway between 1 and 1 + 2^-7 -> even (1.0)
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6 -> even (1 + 2^-6)
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130 * 1.5, 0.0])
    want = np.array([1.0, 1 + 2 ** -6, -1.0, 2 ** -130 * 1.5, 0.0])
    np.testing.assert_array_equal(O.round_bf16(x), want)
    t = torch.tensor(x[:3], dtype=torch.float32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_bf16(x[:3]), t)


# ----------------------------------------------------------------- ternarisation

def test_ternarize_worked_example():
    gd = _load("ternarize_worked.json")
    gamma, codes = O.ternarize(np.array(gd["W"]))
    assert gamma == np.float32(gd["gamma"])
    np.testing.assert_array_equal(codes, np.array(gd["codes"]))


@pytest.mark.parametrize("c", [0.02, -0.5, 3.0, 1e-3])
def test_ternarize_all_equal_gives_sign(c):
    W = np.full((7, 32), c, dtype=np.float32)
    gamma, codes = O.ternarize(W)
    assert gamma == np.float32(abs(c))
    assert np.all(codes == np.sign(c))


def test_ternarize_all_equal_below_eps_gives_zero():
    # |c| / (|c| + 1e-5) < 0.5 exactly when |c| < 1e-5: the epsilon wins
    W = np.full((3, 16), 1e-6, dtype=np.float32)
    _, codes = O.ternarize(W)
    assert np.all(codes == 0)


def test_ternarize_zero_matrix():
    gamma, codes = O.ternarize(np.zeros((4, 16), np.float32))
    assert gamma == 0 and np.all(codes == 0)


def test_ternarize_gaussian_zero_fraction_closed_form():
    # For W ~ N(0, s^2): mean|W| = s*sqrt(2/pi), and |W|/gamma < 1/2 has probability
    # 2*Phi(sqrt(2/pi)/2) - 1 ~= 0.3101; +/-1 split evenly.
    W = synth.latent_weight(7, 1024, 1024).numpy()
    _, codes = O.ternarize(W)
    p0 = 2 * _norm.cdf(0.5 * math.sqrt(2 / math.pi)) - 1
    assert abs(p0 - 0.3101) < 1e-4
    frac0 = np.mean(codes == 0)
    assert abs(frac0 - p0) < 3e-3
    assert abs(np.mean(codes == 1) - np.mean(codes == -1)) < 3e-3


def test_ternarize_negation_and_permutation():
    W = synth.latent_weight(8, 64, 128).numpy()
    g1, c1 = O.ternarize(W)
    g2, c2 = O.ternarize(-W)
    assert g1 == g2
    np.testing.assert_array_equal(c2, -c1)
    perm = np.random.default_rng(0).permutation(W.size)
    g3, c3 = O.ternarize(W.reshape(-1)[perm].reshape(W.shape))
    assert g3 == g1 or abs(float(g3) - float(g1)) <= 1e-7 * float(g1)
    np.testing.assert_array_equal(c3.reshape(-1), c1.reshape(-1)[perm])


def test_ternarize_gamma_is_mean_abs_library():
    W = synth.latent_weight(9, 100, 48).numpy()
    gamma, _ = O.ternarize(W)
    ref = math.fsum(abs(float(v)) for v in W.reshape(-1)) / W.size   # exactly rounded sum
    assert gamma == np.float32(ref)


# ----------------------------------------------------------------- packing

def test_pack_golden_words():
    gd = _load("packed_words.json")
    for case in gd["cases"]:
        codes = np.array([case["codes"]], dtype=np.int8)
        w = O.pack_codes(codes)
        assert w.shape == (1, 1)
        assert int(w[0, 0]) == int(case["word"], 16), case["why"]
        np.testing.assert_array_equal(O.unpack_codes(w, 16), codes)


def test_pack_roundtrip_exhaustive_one_word():
    # every one of the 3^16 code patterns of one uint32 round-trips; a left
    # inverse also proves that no two patterns share a packed word
    n = 3 ** 16
    chunk = 3 ** 12
    for start in range(0, n, chunk):
        idx = np.arange(start, start + chunk, dtype=np.int64)
        digits = np.empty((chunk, 16), dtype=np.int8)
        v = idx.copy()
        for k in range(16):
            digits[:, k] = v % 3 - 1
            v //= 3
        words = O.pack_codes(digits)
        np.testing.assert_array_equal(O.unpack_codes(words, 16), digits)


def test_pack_multiword_layout():
    rng = np.random.default_rng(3)
    codes = rng.integers(-1, 2, size=(5, 64)).astype(np.int8)
    words = O.pack_codes(codes)
    assert words.shape == (5, 4)
    # word j only depends on columns 16j..16j+15
    for j in range(4):
        np.testing.assert_array_equal(words[:, j], O.pack_codes(codes[:, 16 * j:16 * j + 16])[:, 0])


# ----------------------------------------------------------------- RMSNorm + absmax quantisation

def test_quant_constant_vector():
    for c in (0.3, -2.0, 1e-3):
        q, s = O.absmax_quantize(O.rmsnorm(np.full((1, 64), c, np.float32)))
        assert np.all(q == 127 * np.sign(c))


def test_quant_one_hot():
    x = np.zeros((1, 128), np.float32)
    x[0, 17] = -3.5
    xhat = O.rmsnorm(x)
    q, s = O.absmax_quantize(xhat)
    assert q[0, 17] == -127 and np.count_nonzero(q) == 1
    # x^ at the hot index = x / sqrt(x^2/K + eps) (~= -sqrt(K))
    want = -3.5 / math.sqrt(3.5 ** 2 / 128 + O.EPS_NORM)
    assert abs(xhat[0, 17] - want) < 1e-6 * abs(want)


@pytest.mark.parametrize("a,b", [(2.0, 0.75), (-4.0, 1.1), (0.5, -0.2)])
def test_quant_two_value_closed_form(a, b):
    # x^ is proportional to x, so q_b = round(127 * b / |a|) * sign... and q_a = 127*sign(a)
    x = np.zeros((1, 48), np.float32)
    x[0, 0], x[0, 1] = a, b
    xhat = O.rmsnorm(x)
    q, s = O.absmax_quantize(xhat)
    assert q[0, 0] == 127 * np.sign(a)
    assert q[0, 1] == round(127 * b / abs(a))
    assert np.count_nonzero(q) == 2
    # s = 127 / max|x^| with x^ = x / sqrt(mean(x^2) + eps)
    r = math.sqrt((a * a + b * b) / 48 + O.EPS_NORM)
    assert abs(float(s[0]) - 127 * r / abs(a)) <= 1e-6 * 127 * r / abs(a)


def test_quant_gain_closed_form():
    gain = np.array([1.0, 0.5, -1.0, 0.25, 2.0, -0.1, 0.0, 1.5] * 4, np.float32)
    q, _ = O.absmax_quantize(O.rmsnorm(np.ones((1, 32), np.float32), gain=gain))
    np.testing.assert_array_equal(q[0], np.rint(127 * gain / 2.0).astype(np.int8))


def test_quant_max_element_is_127_and_negation_symmetry():
    x = synth.activations(11, 64, 256, outlier_p=0.01).numpy()
    q, s = O.absmax_quantize(O.rmsnorm(x))
    am = np.argmax(np.abs(x), axis=1)
    np.testing.assert_array_equal(np.abs(q[np.arange(64), am]), 127)
    assert np.all(np.abs(q) <= 127)
    qn, sn = O.absmax_quantize(O.rmsnorm(-x))
    np.testing.assert_array_equal(qn, -q)
    np.testing.assert_array_equal(sn, s)


def test_quant_error_bound():
    # |q/s - x^| <= 1/(2s): the round-to-nearest bound
    x = synth.activations(12, 32, 512).numpy()
    xhat = O.rmsnorm(x)
    q, s = O.absmax_quantize(xhat)
    err = np.abs(q / s[:, None].astype(np.float64) - xhat.astype(np.float64))
    assert np.all(err <= 0.5 / s[:, None] * (1 + 1e-6))


def test_rmsnorm_textbook():
    x = synth.activations(13, 16, 300).numpy().astype(np.float64)
    ref = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + O.EPS_NORM)
    np.testing.assert_allclose(O.rmsnorm(x), ref, rtol=2e-7, atol=0)


def test_quant_zero_row_is_degenerate_zero():
    q, s = O.absmax_quantize(O.rmsnorm(np.zeros((2, 32), np.float32)))
    assert np.all(q == 0)
    assert np.all(s == np.float32(127) / np.float32(1e-5))


# ----------------------------------------------------------------- ternary accumulation

def test_accumulate_brute_force_all_ternary_rows():
    # every ternary row of length 4 against every integer input in {-2..2}^4
    rows = np.array(np.meshgrid(*[[-1, 0, 1]] * 4, indexing="ij")).reshape(4, -1).T.astype(np.int8)
    qs = np.array(np.meshgrid(*[range(-2, 3)] * 4, indexing="ij")).reshape(4, -1).T.astype(np.int8)
    acc = O.ternary_accumulate(qs, rows)
    ref = qs.astype(np.float64) @ rows.astype(np.float64).T
    np.testing.assert_array_equal(acc, ref.astype(np.int64))


def test_accumulate_extremes_and_library_matmul():
    rng = np.random.default_rng(5)
    K = 6912
    q = rng.integers(-127, 128, size=(3, K)).astype(np.int8)
    codes = rng.integers(-1, 2, size=(9, K)).astype(np.int8)
    q[0] = 127
    codes[0] = 1
    codes[1] = -1
    acc = O.ternary_accumulate(q, codes)
    ref = torch.tensor(q, dtype=torch.int64) @ torch.tensor(codes, dtype=torch.int64).T
    np.testing.assert_array_equal(acc, ref.numpy())
    assert acc[0, 0] == 127 * K and acc[0, 1] == -127 * K


def test_accumulate_exact_at_the_fp32_bound():
    # K = F32_EXACT_K: the extreme rows sum to +-128 * K = +-2^24 and must stay exact;
    # one past the bound switches to fp64 and stays exact too
    for K in (O.F32_EXACT_K, O.F32_EXACT_K + 16):
        q = np.full((2, K), 127, dtype=np.int8)
        q[1, ::2] = -128
        codes = np.ones((3, K), dtype=np.int8)
        codes[1] = -1
        codes[2, 1::2] = 0
        acc = O.ternary_accumulate(q, codes)
        ref = torch.tensor(q, dtype=torch.int64) @ torch.tensor(codes, dtype=torch.int64).T
        np.testing.assert_array_equal(acc, ref.numpy())
        assert O.ternary_weights_dense(codes).dtype == (np.float32 if K <= O.F32_EXACT_K else np.float64)


def test_accumulate_cached_dense_weights_same_result():
    lin = O.make_tlinear(synth.latent_weight(7, 40, 64).numpy(), cache=True)
    x = synth.activations(8, 5, 64).numpy()
    plain = O.TLinear(lin.codes, lin.gamma)
    np.testing.assert_array_equal(O.bitlinear(x, lin), O.bitlinear(x, plain))
    assert lin.weights().dtype == np.float32 and plain.weights().dtype == np.int8


def test_accumulate_via_packed_words():
    rng = np.random.default_rng(6)
    codes = rng.integers(-1, 2, size=(33, 96)).astype(np.int8)
    q = rng.integers(-127, 128, size=(5, 96)).astype(np.int8)
    back = O.unpack_codes(O.pack_codes(codes), 96)
    np.testing.assert_array_equal(O.ternary_accumulate(q, back), O.ternary_accumulate(q, codes))


# ----------------------------------------------------------------- BitLinear

def _lin(seed, n, k):
    return O.make_tlinear(synth.latent_weight(seed, n, k).numpy())


def test_bitlinear_identity_weights_closed_form():
    K = 64
    W = np.eye(K, dtype=np.float32) * 0.3
    lin = O.make_tlinear(W)
    np.testing.assert_array_equal(lin.codes, np.eye(K, dtype=np.int8))
    assert lin.gamma == np.float32(0.3 / K)
    x = synth.activations(21, 10, K).numpy()
    y, p = O.bitlinear(x, lin, parts=True)
    xhat = O.rmsnorm(x).astype(np.float64)
    s = p["s"].astype(np.float64)[:, None]
    np.testing.assert_allclose(y, float(lin.gamma) * p["q"] / s, rtol=1e-15)
    assert np.all(np.abs(y - float(lin.gamma) * xhat) <= float(lin.gamma) * 0.5 / s * (1 + 1e-6))


def test_bitlinear_sign_symmetries():
    lin = _lin(22, 40, 128)
    x = synth.activations(23, 7, 128).numpy()
    y = O.bitlinear(x, lin)
    np.testing.assert_array_equal(O.bitlinear(-x, lin), -y)
    neg = O.TLinear(-lin.codes, lin.gamma)
    np.testing.assert_array_equal(O.bitlinear(x, neg), -y)


def test_bitlinear_scale_invariance():
    lin = _lin(24, 64, 256)
    x = synth.activations(25, 9, 256).numpy()
    y = O.bitlinear(x, lin)
    y2 = O.bitlinear(x * 4.0, lin)      # power of two: x^ changes only through eps
    y3 = O.bitlinear(x * 3.7, lin)
    scale = np.max(np.abs(y))
    assert np.max(np.abs(y2 - y)) <= 1e-2 * scale
    assert np.max(np.abs(y3 - y)) <= 1e-2 * scale


def test_bitlinear_zero_input_gives_bias():
    lin = _lin(26, 8, 32)
    lin.bias = np.arange(8, dtype=np.float64)
    np.testing.assert_array_equal(O.bitlinear(np.zeros((3, 32)), lin), np.tile(np.arange(8.0), (3, 1)))


def test_bitlinear_approximates_dense_product():
    # dequantised result is close to x^ @ (gamma*codes)^T: the quantisation error bound
    lin = _lin(27, 50, 512)
    x = synth.activations(28, 6, 512).numpy()
    y, p = O.bitlinear(x, lin, parts=True)
    dense = p["xhat"].astype(np.float64) @ (float(lin.gamma) * lin.codes.astype(np.float64)).T
    bound = float(lin.gamma) * 0.5 / p["s"].astype(np.float64)[:, None] * np.sum(np.abs(lin.codes), axis=1)[None, :]
    assert np.all(np.abs(y - dense) <= bound * (1 + 1e-9))


# ----------------------------------------------------------------- MLGRU scan

def test_sigmoid_silu_identities():
    z = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(O.sigmoid(z) + O.sigmoid(-z), 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(O.silu(z) - O.silu(-z), z, rtol=0, atol=1e-13)
    assert O.sigmoid(0.0) == 0.5 and O.silu(0.0) == 0.0
    assert O.sigmoid(-1e4) == 0.0 and O.sigmoid(1e4) == 1.0


def _scan_inputs(seed, B=2, T=32, d=8):
    p = synth.preacts(seed, B, T, d).numpy().astype(np.float64)
    return p[:, :, 0], p[:, :, 1], p[:, :, 2]


def test_scan_forget_zero_gives_candidate():
    _, pc, pg = _scan_inputs(31)
    pf = np.full_like(pc, -1e4)
    h0 = np.ones(pc[:, 0].shape) * 5
    o, hT = O.mlgru_scan(pf, pc, pg, h0)
    np.testing.assert_allclose(o, O.sigmoid(pg) * O.silu(pc), rtol=1e-15)
    np.testing.assert_allclose(hT, O.silu(pc[:, -1]), rtol=1e-15)


def test_scan_forget_one_holds_state():
    _, pc, pg = _scan_inputs(32)
    pf = np.full_like(pc, 1e4)
    h0 = synth.activations(33, 2, 8).numpy().astype(np.float64)
    o, hT = O.mlgru_scan(pf, pc, pg, h0)
    np.testing.assert_array_equal(hT, h0)
    np.testing.assert_allclose(o, O.sigmoid(pg) * h0[:, None, :], rtol=1e-15)


def test_scan_unrolled_closed_form():
    pf, pc, pg = _scan_inputs(34, T=24)
    h0 = synth.activations(35, 2, 8).numpy().astype(np.float64)
    o, hT = O.mlgru_scan(pf, pc, pg, h0)
    f, c, g = O.sigmoid(pf), O.silu(pc), O.sigmoid(pg)
    T = pf.shape[1]
    for t in range(T):
        # h_t = (prod_{r<=t} f_r) h0 + sum_{s<=t} (prod_{s<r<=t} f_r) (1 - f_s) c_s
        h = np.prod(f[:, :t + 1], axis=1) * h0
        for s in range(t + 1):
            h = h + np.prod(f[:, s + 1:t + 1], axis=1) * (1 - f[:, s]) * c[:, s]
        np.testing.assert_allclose(o[:, t], g[:, t] * h, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(hT, h, rtol=1e-12)


def test_scan_convex_bound_and_chunking_and_batch_independence():
    pf, pc, pg = _scan_inputs(36, B=3, T=40, d=16)
    h0 = synth.activations(37, 3, 16).numpy().astype(np.float64)
    o, hT = O.mlgru_scan(pf, pc, pg, h0)
    c = O.silu(pc)
    # |h_t| <= max(|h0|, max_s |c_s|) because h_t is a convex combination
    h = o / O.sigmoid(pg)
    bound = np.maximum(np.abs(h0), np.max(np.abs(c), axis=1))
    assert np.all(np.abs(h) <= bound[:, None, :] * (1 + 1e-12))
    # split the sequence: scan(T) == scan(T1) then scan(T - T1) from its state
    o1, h1 = O.mlgru_scan(pf[:, :13], pc[:, :13], pg[:, :13], h0)
    o2, h2 = O.mlgru_scan(pf[:, 13:], pc[:, 13:], pg[:, 13:], h1)
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=1), o)
    np.testing.assert_array_equal(h2, hT)
    # batch rows do not interact
    ob, hb = O.mlgru_scan(pf[1:2], pc[1:2], pg[1:2], h0[1:2])
    np.testing.assert_array_equal(ob[0], o[1])


# ----------------------------------------------------------------- g_norm output gate

def test_gnorm_hand_worked_two_channels():
    # h = (3, 4): mean square 12.5, so h / rms = (3, 4) * sqrt(2) / 5; sigmoid(ln 3) = 3/4,
    # so swish(ln 3) = 0.75 ln 3 and swish(-ln 3) = -0.25 ln 3; gain (2, 5)
    ln3 = math.log(3.0)
    o = O.rmsnorm_swish_gate(np.array([3.0, 4.0]), np.array([ln3, -ln3]), w=np.array([2.0, 5.0]), eps=0.0)
    r2 = math.sqrt(2.0)
    np.testing.assert_allclose(o, [2 * 3 * r2 / 5 * 0.75 * ln3, 5 * 4 * r2 / 5 * (-0.25 * ln3)], rtol=1e-14)
    # eps adds to the mean square: sqrt(12.5 + 0.5) = sqrt(13)
    o = O.rmsnorm_swish_gate(np.array([3.0, 4.0]), np.array([ln3, ln3]), eps=0.5)
    np.testing.assert_allclose(o, np.array([3.0, 4.0]) / math.sqrt(13.0) * 0.75 * ln3, rtol=1e-14)
    # h constant across channels, eps = 0: the norm is the sign, o' = sign(a) swish(g~)
    g = np.array([-2.0, 0.5, 3.0])
    np.testing.assert_allclose(O.rmsnorm_swish_gate(np.full(3, -7.5), g, eps=0.0), -O.silu(g), rtol=1e-15)


def test_gnorm_zero_gate_scale_invariance_and_axis():
    pf, pc, pg = _scan_inputs(38, B=2, T=20, d=16)
    h0 = synth.activations(39, 2, 16).numpy().astype(np.float64)
    # g~ = 0: swish(0) = 0, so o' = 0 exactly whatever the state
    o, _ = O.mlgru_scan_gnorm(pf, pc, np.zeros_like(pg), h0)
    assert np.all(o == 0.0)
    # constant g~ = z and unit gain: every token's mean square is swish(z)^2 ms/(ms + eps),
    # ms the token's mean square of h (taken from the recurrence with a unit sigmoid gate
    # written as g~ = +inf); normalising over time instead of channels breaks it
    z, eps = 0.8, 1e-3
    o, _ = O.mlgru_scan_gnorm(pf, pc, np.full_like(pg, z), h0, eps=eps)
    h, _ = O.mlgru_scan(pf, pc, np.full_like(pg, 1e4), h0)
    ms = np.mean(h * h, axis=-1)
    np.testing.assert_allclose(np.mean(o * o, axis=-1), O.silu(z) ** 2 * ms / (ms + eps), rtol=1e-12)
    # with eps = 0 the output is invariant to a positive scale of the state and odd in it
    hh = synth.activations(40, 6, 16).numpy().astype(np.float64)
    a = O.rmsnorm_swish_gate(hh, pg[0, :6], eps=0.0)
    np.testing.assert_allclose(O.rmsnorm_swish_gate(hh * 37.0, pg[0, :6], eps=0.0), a, rtol=1e-13)
    np.testing.assert_allclose(O.rmsnorm_swish_gate(-hh, pg[0, :6], eps=0.0), -a, rtol=1e-13)


def test_gnorm_scan_forget_zero_and_unrolled():
    pf, pc, pg = _scan_inputs(56, B=2, T=12, d=8)
    w = 0.5 + synth.activations(57, 1, 8).numpy().astype(np.float64)[0] ** 2
    h0 = synth.activations(58, 2, 8).numpy().astype(np.float64)
    # forget gate 0: h_t = SiLU(c~_t)
    o, hT = O.mlgru_scan_gnorm(np.full_like(pc, -1e4), pc, pg, h0, w)
    c = O.silu(pc)
    ref = c / np.sqrt(np.mean(c * c, axis=-1, keepdims=True) + O.EPS_NORM) * w * O.silu(pg)
    np.testing.assert_allclose(o, ref, rtol=1e-13)
    np.testing.assert_allclose(hT, c[:, -1], rtol=1e-15)
    # general gates: the state is the unrolled sum, the same one the sigmoid gate multiplies
    o, hT = O.mlgru_scan_gnorm(pf, pc, pg, h0, w)
    og, _ = O.mlgru_scan(pf, pc, pg, h0)
    H = og / O.sigmoid(pg)
    np.testing.assert_allclose(O.rmsnorm_swish_gate(H, pg, w), o, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(H[:, -1], hT, rtol=1e-12)


# ----------------------------------------------------------------- GLU and block

def _block(seed, d, inner):
    lat = {}
    for i, name in enumerate(synth.PROJ_NAMES):
        n, k = {"f": (d, d), "c": (d, d), "g": (d, d), "o": (d, d),
                "gate": (inner, d), "up": (inner, d), "down": (d, inner)}[name]
        lat[name] = synth.latent_weight(synth.sub_seed(seed, 0, i), n, k).numpy()
    return O.make_block(lat)


def test_glu_identity_weights_closed_form():
    # gate = up = I: p = SiLU(gamma_g q/s) * (gamma_u q/s); swapping the SiLU branch changes it
    d = 32
    eye = O.make_tlinear(np.eye(d, dtype=np.float32) * d)            # gamma = 1
    eye2 = O.make_tlinear(-np.eye(d, dtype=np.float32) * 2 * d)      # up = -I, gamma = 2
    blk = _block(41, d, d)
    blk.gate, blk.up = eye, eye2
    x = synth.activations(42, 5, d).numpy()
    _, parts = O.glu(x, blk, "f32", parts=True)
    q, s = O.absmax_quantize(O.rmsnorm(x))
    u = float(eye.gamma) * q / s[:, None].astype(np.float64)
    v = -float(eye2.gamma) * q / s[:, None].astype(np.float64)
    np.testing.assert_allclose(parts["p"], O.round_f32(O.silu(u) * v), rtol=1e-7)
    swapped = O.silu(v) * u
    assert np.max(np.abs(swapped - parts["p"])) > 0.1 * np.max(np.abs(parts["p"]))


def _scaled_eye(d, alpha):
    # latent alpha*d*I: gamma = |alpha|, codes sign(alpha)*I, so the BitLinear is alpha * q/s
    lin = O.make_tlinear(np.eye(d, dtype=np.float32) * np.float32(alpha * d))
    np.testing.assert_array_equal(lin.codes, np.sign(alpha) * np.eye(d, dtype=np.int8))
    return lin


def _dq(lin, x):
    # identity-weight BitLinear: sign * gamma * q / s of RMSNorm(x) (pinned stage functions)
    x2 = np.asarray(x).reshape(-1, x.shape[-1])
    q, s = O.absmax_quantize(O.rmsnorm(x2))
    sign = float(lin.codes[0, 0])
    return (sign * float(lin.gamma) * q / s[:, None].astype(np.float64)).reshape(x.shape)


def _unrolled_scan(f, c, g, h0):
    # h_t = (prod_{r<=t} f_r) h0 + sum_{s<=t} (prod_{s<r<=t} f_r) (1 - f_s) c_s ; o'_t = g_t h_t
    T = f.shape[1]
    o = np.empty_like(f)
    for t in range(T):
        h = np.prod(f[:, :t + 1], axis=1) * h0
        for s_ in range(t + 1):
            h = h + np.prod(f[:, s_ + 1:t + 1], axis=1) * (1 - f[:, s_]) * c[:, s_]
        o[:, t] = g[:, t] * h
    return o, h


ALPHAS = {"f": 0.7, "c": -1.3, "g": 2.1, "o": 0.45, "gate": 1.6, "up": -0.8, "down": 0.35}


def _eye_block(d):
    return O.Block(**{name: _scaled_eye(d, a) for name, a in ALPHAS.items()})


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mlgru_identity_weights_closed_form(dtype):
    # f, c, g, o = alpha_* I with distinct alphas: the projections reduce to
    # alpha * q/s, the scan to its unrolled sum; any swap of the three gate
    # projections, SiLU/sigmoid mix-up, missing (1 - f) or o-projection of h
    # instead of o' changes the result. Storage points in the run dtype.
    d, B, T = 32, 2, 6
    blk = _eye_block(d)
    x = O.store(synth.activations(61, B * T, d).numpy().reshape(B, T, d), dtype)
    h0 = synth.activations(62, B, d).numpy().astype(np.float64)
    o, hT, parts = O.mlgru(x, blk, h0, dtype, parts=True)
    pf, pc, pg = (O.store(_dq(getattr(blk, n), x), dtype) for n in ("f", "c", "g"))
    np.testing.assert_array_equal(parts["pf"], pf)
    np.testing.assert_array_equal(parts["pc"], pc)
    np.testing.assert_array_equal(parts["pg"], pg)
    og, h = _unrolled_scan(O.sigmoid(pf), O.silu(pc), O.sigmoid(pg), h0)
    # o' is stored: agreement up to one storage ulp where the two sums round apart
    ulp = 2.0 ** -7 if dtype == "bf16" else 2.0 ** -23
    np.testing.assert_allclose(parts["o_gate"], O.store(og, dtype), rtol=ulp, atol=1e-12)
    np.testing.assert_allclose(hT, O.round_f32(h), rtol=2e-7)
    np.testing.assert_allclose(o, _dq(blk.o, parts["o_gate"]), rtol=1e-12)
    # f and g swapped would give a different o'
    og_swapped, _ = _unrolled_scan(O.sigmoid(pg), O.silu(pc), O.sigmoid(pf), h0)
    assert np.max(np.abs(og_swapped - og)) > 0.05 * np.max(np.abs(og))


def test_block_identity_weights_closed_form():
    # all seven projections alpha_* I: y1 = x + alpha_o q/s(o'), y = y1 + alpha_d q/s(p),
    # p = SiLU(alpha_gate q/s(y1)) * alpha_up q/s(y1): pins the residual wiring and which
    # tensor each mixer reads
    d, B, T = 32, 2, 5
    blk = _eye_block(d)
    x = O.round_f32(synth.activations(63, B * T, d).numpy().reshape(B, T, d))
    h0 = synth.activations(64, B, d).numpy().astype(np.float64)
    y, hT, parts = O.block_forward(x, blk, h0, "f32", parts=True)
    pf, pc, pg = (O.round_f32(_dq(getattr(blk, n), x)) for n in ("f", "c", "g"))
    og, h = _unrolled_scan(O.sigmoid(pf), O.silu(pc), O.sigmoid(pg), h0)
    og = O.round_f32(og)
    np.testing.assert_allclose(parts["o_gate"], og, rtol=2e-7, atol=1e-12)
    y1 = O.round_f32(x + _dq(blk.o, parts["o_gate"]))
    np.testing.assert_array_equal(parts["y1"], y1)
    u, v = _dq(blk.gate, y1), _dq(blk.up, y1)
    p = O.round_f32(O.silu(u) * v)
    np.testing.assert_array_equal(parts["p"], p)
    np.testing.assert_array_equal(y, O.round_f32(y1 + _dq(blk.down, p)))
    np.testing.assert_allclose(hT, O.round_f32(h), rtol=2e-7)
    # a block that skipped the first residual (GLU of x) would differ
    p_x = O.round_f32(O.silu(_dq(blk.gate, x)) * _dq(blk.up, x))
    assert np.max(np.abs(O.round_f32(x + _dq(blk.down, p_x)) - y)) > 1e-3


def test_block_gnorm_identity_weights_and_zero_gate():
    # identity weights with the g_norm gate: o' = RMSNorm(h) * w * SiLU(g~) with h the
    # unrolled state; the sigmoid gate would give a different o'
    d, B, T = 32, 2, 5
    blk = _eye_block(d)
    blk.gnorm = 0.25 + synth.activations(65, 1, d).numpy().astype(np.float64)[0] ** 2
    x = O.round_f32(synth.activations(66, B * T, d).numpy().reshape(B, T, d))
    h0 = synth.activations(67, B, d).numpy().astype(np.float64)
    y, hT, parts = O.block_forward(x, blk, h0, "f32", parts=True)
    pf, pc, pg = (O.round_f32(_dq(getattr(blk, n), x)) for n in ("f", "c", "g"))
    H = np.stack([_unrolled_scan(O.sigmoid(pf[:, :t + 1]), O.silu(pc[:, :t + 1]),
                                 np.ones_like(pg[:, :t + 1]), h0)[1] for t in range(T)], axis=1)
    ms = np.mean(H * H, axis=-1, keepdims=True)
    og = O.round_f32(H / np.sqrt(ms + O.EPS_NORM) * blk.gnorm * O.silu(pg))
    np.testing.assert_allclose(parts["o_gate"], og, rtol=2e-7, atol=1e-12)
    np.testing.assert_allclose(hT, O.round_f32(H[:, -1]), rtol=2e-7)
    sig = O.round_f32(O.sigmoid(pg) * H)
    assert np.max(np.abs(sig - og)) > 0.05 * np.max(np.abs(og))
    # g-projection weights zero: g~ = 0, o' = 0, the o-projection of zeros is 0, y1 = x
    blk.g = O.make_tlinear(np.zeros((d, d), np.float32))
    _, _, parts = O.block_forward(x, blk, h0, "f32", parts=True)
    assert np.all(parts["o_gate"] == 0.0)
    np.testing.assert_array_equal(parts["y1"], x)


def test_block_zero_weights_is_identity():
    d, inner, B, T = 32, 48, 2, 6
    blk = _block(43, d, inner)
    for name in ("f", "c", "g", "o", "gate", "up", "down"):
        lin = getattr(blk, name)
        setattr(blk, name, O.make_tlinear(np.zeros((lin.N, lin.K), np.float32)))
    x = O.round_bf16(synth.activations(44, B * T, d).numpy().reshape(B, T, d))
    h0 = synth.activations(45, B, d).numpy().astype(np.float64)
    y, hT = O.block_forward(x, blk, h0, "bf16")
    np.testing.assert_array_equal(y, x)
    # f = sigmoid(0) = 1/2, c = SiLU(0) = 0: h_T = 2^-T h0
    np.testing.assert_array_equal(hT, O.round_f32(h0 * 0.5 ** T))


@pytest.mark.parametrize("dtype,gnorm", [("f32", False), ("bf16", False), ("bf16", True)])
def test_block_prefill_equals_decode_steps(dtype, gnorm):
    d, inner, B, T = 32, 64, 2, 5
    blk = _block(46, d, inner)
    if gnorm:
        blk.gnorm = 1.0 + 0.1 * synth.activations(48, 1, d).numpy().astype(np.float64)[0]
    x = O.store(synth.activations(47, B * T, d).numpy().reshape(B, T, d), dtype)
    h0 = np.zeros((B, d))
    y, hT = O.block_forward(x, blk, h0, dtype)
    h = h0
    ys = []
    for t in range(T):
        yt, h = O.block_forward(x[:, t:t + 1], blk, h, dtype)
        ys.append(yt)
    yd = np.concatenate(ys, axis=1)
    # state is stored in fp32 between decode calls, so agreement is to rounding
    np.testing.assert_allclose(yd, y, rtol=0, atol=2e-2 * np.max(np.abs(y)))
    np.testing.assert_allclose(h, hT, rtol=1e-5, atol=1e-6)


def test_stack_composes_blocks():
    # distinct non-zero initial states per layer, so a stack that handed one
    # layer's state to another would not compose the same way
    d, inner, B, T = 16, 32, 1, 4
    blocks = [_block(50 + l, d, inner) for l in range(3)]
    x = O.round_f32(synth.activations(53, B * T, d).numpy().reshape(B, T, d))
    h0s = O.round_f32(synth.activations(54, 3 * B, d).numpy().reshape(3, B, d) * np.array([1.0, -2.0, 0.5])[:, None, None])
    y, hs = O.stack_forward(x, blocks, h0s, "f32")
    z = x
    for l in range(3):
        z, h = O.block_forward(z, blocks[l], h0s[l], "f32")
        np.testing.assert_array_equal(h, hs[l])
    np.testing.assert_array_equal(z, y)


# ----------------------------------------------------------------- model ends

def test_embed_brute_force_and_range():
    E = synth.activations(70, 7, 5).numpy()
    ids = np.array([[3, 0, 6], [6, 6, 1]])
    x = O.embed(ids, E, "bf16")
    for b in range(2):
        for t in range(3):
            for k in range(5):
                assert x[b, t, k] == O.round_bf16(float(E[ids[b, t], k]))
    np.testing.assert_array_equal(O.embed(ids, E, "f32"), O.round_f32(E[ids]))
    for bad in ([[-1]], [[7]]):
        with pytest.raises(IndexError):
            O.embed(np.array(bad), E, "f32")


def test_greedy_token_brute_force_and_ties():
    rng = np.random.default_rng(71)
    L = rng.integers(-3, 4, size=(40, 9)).astype(np.float64)   # many ties
    tok = O.greedy_token(L)
    for r in range(40):
        best = 0
        for j in range(1, 9):
            if L[r, j] > L[r, best]:
                best = j
        assert tok[r] == best
    assert O.greedy_token(np.array([[-5.0, -5.0, -7.0]]))[0] == 0
    assert O.greedy_token(np.array([[1.0]]))[0] == 0


def test_lm_logits_identity_head_closed_form():
    d = 32
    head = _scaled_eye(d, 1.5)
    x = synth.activations(72, 6, d).numpy()
    np.testing.assert_array_equal(O.lm_logits(x, head, "bf16"), O.round_bf16(_dq(head, x)))


def _zero_block(d, inner):
    z = {n: np.zeros(s, np.float32) for n, s in (("f", (d, d)), ("c", (d, d)), ("g", (d, d)), ("o", (d, d)),
                                                  ("gate", (inner, d)), ("up", (inner, d)), ("down", (d, inner)))}
    return O.make_block(z)


def test_generation_follows_a_permutation():
    # zero blocks are the identity and the head is the identity, so the next
    # token is the position of the largest entry of the current token's
    # embedding row: a table whose row i peaks at perm[i] makes greedy
    # generation follow the permutation
    V = d = 16
    perm = np.random.default_rng(73).permutation(V)
    E = 0.1 * synth.activations(74, V, d).numpy()
    E[np.arange(V), perm] = 3.0
    blocks = [_zero_block(d, 24) for _ in range(2)]
    head = _scaled_eye(d, 1.0)
    prompt = np.array([[5, 2, 9], [0, 0, 3]])
    toks, hs = O.generate_greedy(prompt, 6, E, blocks, head, "bf16")
    for b in range(2):
        t = prompt[b, -1]
        for k in range(6):
            t = perm[t]
            assert toks[b, k] == t
    assert np.all(hs == 0.0)


def test_generation_matches_prefill_of_the_grown_sequence():
    # each generated token is also the greedy token of one prefill over the
    # prompt and the tokens before it (state carried vs recomputed, fp32 runs)
    V, d, inner = 40, 32, 48
    blocks = [_block(75 + l, d, inner) for l in range(2)]
    head = O.make_tlinear(synth.latent_weight(77, V, d).numpy())
    E = synth.activations(78, V, d).numpy()
    prompt = np.array([[3, 17, 8, 8]])
    toks, hs = O.generate_greedy(prompt, 3, E, blocks, head, "f32")
    for k in range(3):
        seq = np.concatenate([prompt, toks[:, :k]], axis=1)
        logits, _ = O.model_forward(seq, E, blocks, head, np.zeros((2, 1, d)), "f32")
        assert O.greedy_token(logits)[0] == toks[0, k]
        srt = np.sort(logits[0])
        assert srt[-1] - srt[-2] > 1e-3   # no near-tie that rounding could flip
    # the carried state after the last fed-back token is the prefill's state over everything
    _, h_all = O.model_forward(np.concatenate([prompt, toks], axis=1), E, blocks, head, np.zeros((2, 1, d)), "f32")
    np.testing.assert_allclose(hs, h_all, rtol=1e-5, atol=1e-6)


# ----------------------------------------------------------------- scan backward

def _scan_loss(pf, pc, pg, h0, do, dhT):
    o, hT = O.mlgru_scan(pf, pc, pg, h0)
    return float(np.sum(o * do) + np.sum(hT * dhT))


def test_scan_backward_matches_central_differences():
    # every gradient against (L(x + e) - L(x - e)) / 2e of the forward oracle
    B, T, d = 2, 7, 3
    pf, pc, pg = (1.5 * a for a in _scan_inputs(90, B, T, d))
    h0 = synth.activations(91, B, d).numpy().astype(np.float64)
    do = synth.activations(92, B * T, d).numpy().astype(np.float64).reshape(B, T, d)
    dhT = synth.activations(93, B, d).numpy().astype(np.float64)
    dpf, dpc, dpg, dh0 = O.mlgru_scan_backward(pf, pc, pg, h0, do, dhT)
    eps = 1e-6
    for arr, grad in ((pf, dpf), (pc, dpc), (pg, dpg)):
        num = np.empty_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            lp = _scan_loss(pf, pc, pg, h0, do, dhT)
            arr[idx] = old - eps
            lm = _scan_loss(pf, pc, pg, h0, do, dhT)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)
    num = np.empty_like(h0)
    for idx in np.ndindex(h0.shape):
        old = h0[idx]
        h0[idx] = old + eps
        lp = _scan_loss(pf, pc, pg, h0, do, dhT)
        h0[idx] = old - eps
        lm = _scan_loss(pf, pc, pg, h0, do, dhT)
        h0[idx] = old
        num[idx] = (lp - lm) / (2 * eps)
    np.testing.assert_allclose(dh0, num, rtol=1e-6, atol=1e-8)


def test_scan_backward_special_cases():
    pf, pc, pg = _scan_inputs(94, B=2, T=9, d=4)
    h0 = synth.activations(95, 2, 4).numpy().astype(np.float64)
    do = synth.activations(96, 18, 4).numpy().astype(np.float64).reshape(2, 9, 4)
    # no upstream gradient: every gradient is zero
    z = O.mlgru_scan_backward(pf, pc, pg, h0, np.zeros_like(do))
    assert all(np.all(a == 0.0) for a in z)
    # forget gate ~0 (f~ = -40): h_t = c_t, so dc~_t = do_t g_t SiLU'(c~_t), dh0 ~ 0
    pf0 = np.full_like(pf, -40.0)
    dpf, dpc, dpg, dh0 = O.mlgru_scan_backward(pf0, pc, pg, h0, do)
    s = O.sigmoid(pc)
    np.testing.assert_allclose(dpc, do * O.sigmoid(pg) * s * (1 + pc * (1 - s)), rtol=1e-12, atol=1e-15)
    assert np.max(np.abs(dh0)) < 1e-15
    # only dhT: lambda is the product of the forget gates from the end
    dpf, dpc, dpg, dh0 = O.mlgru_scan_backward(pf, pc, pg, h0, np.zeros_like(do), np.ones((2, 4)))
    np.testing.assert_allclose(dh0, np.prod(O.sigmoid(pf), axis=1), rtol=1e-12)
    assert np.all(dpg == 0.0)
