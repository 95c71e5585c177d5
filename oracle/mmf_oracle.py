"""Plain CPU oracle for the MatMul-free block forward (FusedBitLinear + MLGRU + GLU).

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously-correct
definition that the CUDA library is checked against. Only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it. The library never calls it, and it shares no code
with the CUDA path (no kernels, headers, tables or helpers): only the seeded
input generators in ``synth`` feed both sides.

Sources (web pages on "Scalable MatMul-free Language Modeling", arXiv 2406.02528):
  [DC]  "MatMul-free language models", DataCamp blog (Chinese edition);
        sections "Replacing MatMul with ternary operations" and
        "Core components: MLGRU and GLU" (incl. the overview figure's panels
        "MatMul vs. scaled ternary accumulation" and "RMS Norm").
  [HL]  hysenlabs project review of ridgerchu/matmulfreellm; sections
        "FusedBitLinear: how ternary weights save the multiplications" and
        "HGRN attention: gated recurrence instead of softmax".
  [AX]  arXiv abstract page of 2406.02528.

Where the pages are silent the plainest reading is taken and stated at the
function. Numerics: fp64 unless a step decides an integer (a quantised code),
where the decision is taken in fp32 exactly as the kernels take it, so that
both sides can agree bit for bit:
  * weight codes: gamma is an fp64 mean cast to fp32, the division W/(gamma+eps)
    is one IEEE fp32 division, rounding is half-to-even;
  * activation codes: the mean square is an fp64 sum cast to fp32, then
    r = sqrt(ms + eps), 1/r, x*(1/r), *gain, 127/max|x^|, x^*s and the rounding
    are single IEEE fp32 operations in that order.

Pins: every function below is checked in tests/test_oracle_pins.py against
closed forms, hand-built cases, brute force or library routines. The
compositions ``mlgru``, ``block_forward`` and ``stack_forward`` are pinned
through special cases only: scaled-identity weights, where every BitLinear
reduces to alpha * q / s and the scan to its unrolled sum; zero weights; the
prefill == decode invariant. The pages print no worked example for them.
The g_norm output gate (``rmsnorm_swish_gate``) is pinned by a hand-worked
two-channel case, g~ = 0 giving o' = 0, the mean-square invariant under a
constant gate, scale invariance, and the identity-weight block.
The model ends (``embed``, ``lm_logits``, ``greedy_token``, ``model_forward``,
``generate_greedy``) are pinned by brute force on small tables, ties, and a
generation that follows a known permutation (zero blocks, identity head).
``mlgru_scan_backward`` is pinned by central finite differences of the
forward oracle in every input, and by special cases (no upstream gradient,
forget gate 0, only a final-state gradient).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

EPS_W = 1e-5      # weight ternarisation epsilon: W / (gamma + EPS_W)
Q_FLOOR = 1e-5    # floor on max|x^| before 127/max|x^|
Q_MAX = 127       # int8 activation code range [-127, 127] (-128 is never produced)
EPS_NORM = 1e-6   # default RMSNorm epsilon (the pages give none)

# ---------------------------------------------------------------------------
# Storage rounding
# ---------------------------------------------------------------------------


def round_f32(x) -> np.ndarray:
    """Round to the nearest fp32 (IEEE, half-to-even); returned as fp64 values."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (8-bit significand), ties to even.

    Written from the format's definition: a normal bf16 number is m * 2^(e-8)
    with an integer 128 <= |m| < 256; below 2^-126 the spacing is fixed at 2^-133.
    Scaling by powers of two is exact in fp64, so the only rounding is np.rint.
    """
    x = np.asarray(x, dtype=np.float64)
    mant, expo = np.frexp(x)                 # x = mant * 2^expo, 0.5 <= |mant| < 1
    normal = np.ldexp(np.rint(np.ldexp(mant, 8)), expo - 8)
    sub = np.ldexp(np.rint(np.ldexp(x, 133)), -133)
    out = np.where(np.abs(x) < 2.0 ** -126, sub, normal)
    return out


def store(x, dtype: str) -> np.ndarray:
    """Round to the run's storage type ("f32" or "bf16")."""
    if dtype == "f32":
        return round_f32(x)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Weights: absmean ternarisation and the 2-bit packed format
# ---------------------------------------------------------------------------


def ternarize(W, gamma: Optional[np.float32] = None):
    """Absmean ternarisation of one latent weight matrix.

    [DC] "Replacing MatMul with ternary operations": the weights are scaled by
    the mean of the absolute values of the matrix's elements and each element
    is rounded to the nearest of -1, 0, 1. Reading: one gamma per whole matrix,
    codes = clip(round(W / (gamma + 1e-5)), -1, 1), ties to even.

    If ``gamma`` is given it is used instead of the matrix's own mean (used to
    compare codes given another implementation's gamma).
    Returns (gamma as np.float32, codes as int8 array of W's shape).
    """
    W32 = np.asarray(W, dtype=np.float32)
    if W32.size == 0:
        raise ValueError("empty weight matrix")
    if gamma is None:
        total = np.sum(np.abs(W32.astype(np.float64)))
        gamma = np.float32(total / W32.size)
    gamma = np.float32(gamma)
    denom = np.float32(gamma + np.float32(EPS_W))       # one fp32 addition
    t = W32 / denom                                      # one IEEE fp32 division
    codes = np.clip(np.rint(t), -1, 1).astype(np.int8)
    return gamma, codes


def pack_codes(codes) -> np.ndarray:
    """Pack ternary codes {-1,0,1} [N, K] (K % 16 == 0) into uint32 [N, K/16].

    Storage format of this library (not from the pages): the stored 2-bit value
    is code + 1 in {0, 1, 2}; the code for column k = 16*j + 4*i + b sits in
    word j at bits [8*b + 2*i, 8*b + 2*i + 2).
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    if K % 16 != 0:
        raise ValueError("K must be a multiple of 16")
    if codes.size and (codes.min() < -1 or codes.max() > 1):
        raise ValueError("codes must be in {-1,0,1}")
    v = (codes.astype(np.int64) + 1).reshape(N, K // 16, 4, 4)   # [n, j, i, b]
    words = np.zeros((N, K // 16), dtype=np.int64)
    for i in range(4):
        for b in range(4):
            words |= v[:, :, i, b] << (8 * b + 2 * i)
    return words.astype(np.uint32)


def unpack_codes(packed, K: int) -> np.ndarray:
    """Inverse of pack_codes: uint32 [N, K/16] -> int8 codes [N, K]."""
    packed = np.asarray(packed, dtype=np.uint32).astype(np.int64)
    N = packed.shape[0]
    out = np.zeros((N, K // 16, 4, 4), dtype=np.int64)
    for i in range(4):
        for b in range(4):
            out[:, :, i, b] = (packed >> (8 * b + 2 * i)) & 3
    if np.any(out == 3):
        raise ValueError("invalid 2-bit field 3 in packed weights")
    return (out.reshape(N, K) - 1).astype(np.int8)


@dataclasses.dataclass
class TLinear:
    """A ternary BitLinear: codes [N,K] int8, per-matrix gamma, optional gain [K] / bias [N].

    With ``cache`` set, the codes are also kept as the -1.0/0.0/+1.0 matrix that
    ternary_accumulate multiplies (4 bytes per weight more memory, no
    conversion per call); the results are the same either way.
    """
    codes: np.ndarray
    gamma: np.float32
    gain: Optional[np.ndarray] = None
    bias: Optional[np.ndarray] = None
    cache: bool = False
    _dense: Optional[np.ndarray] = dataclasses.field(default=None, repr=False, compare=False)

    def weights(self) -> np.ndarray:
        """What ternary_accumulate takes: the cached dense codes, or the int8 codes."""
        if not self.cache:
            return self.codes
        if self._dense is None:
            self._dense = ternary_weights_dense(self.codes)
        return self._dense

    @property
    def N(self) -> int:
        return self.codes.shape[0]

    @property
    def K(self) -> int:
        return self.codes.shape[1]


def make_tlinear(W_latent, gain=None, bias=None, cache: bool = False) -> TLinear:
    gamma, codes = ternarize(W_latent)
    g = None if gain is None else np.asarray(gain, dtype=np.float32)
    b = None if bias is None else np.asarray(bias, dtype=np.float64)
    return TLinear(codes, gamma, g, b, cache)


# ---------------------------------------------------------------------------
# Activations: RMSNorm, per-token absmax int8 quantisation
# ---------------------------------------------------------------------------


def rmsnorm(x, gain=None, eps: float = EPS_NORM) -> np.ndarray:
    """RMSNorm over the last axis, in the fp32 steps listed in the module docstring.

    [DC] overview figure, "RMS Norm" panel: activations are normalised before
    quantisation. [HL] "FusedBitLinear": RMSNorm on the input, then the fused
    bit-op kernel. x^ = x / sqrt(mean(x^2) + eps) * gain. Returns fp32.
    """
    x32 = np.asarray(x, dtype=np.float32)
    K = x32.shape[-1]
    ss = np.sum(np.square(x32.astype(np.float64)), axis=-1)
    ms = (ss / K).astype(np.float32)
    r = np.sqrt(ms + np.float32(eps))
    rinv = (np.float32(1.0) / r).astype(np.float32)
    xhat = x32 * rinv[..., None]
    if gain is not None:
        xhat = xhat * np.asarray(gain, dtype=np.float32)
    return xhat.astype(np.float32)


def absmax_quantize(xhat):
    """Per-token absmax int8 quantisation of normalised activations.

    The pages only say the activations are normalised before quantisation
    ([DC] "RMS Norm" panel); the per-token absmax rule is the reading taken:
    s = 127 / max(max|x^|, 1e-5), q = clip(round_half_even(x^ * s), -128, 127).
    Returns (q int8, s fp32 per token).
    """
    xh = np.asarray(xhat, dtype=np.float32)
    a = np.max(np.abs(xh), axis=-1)
    s = (np.float32(Q_MAX) / np.maximum(a, np.float32(Q_FLOOR))).astype(np.float32)
    q = np.clip(np.rint(xh * s[..., None]), -128, 127).astype(np.int8)
    return q, s


# Largest K for which every partial sum of q[k] * w[k] (|q| <= 128, w in {-1,0,1})
# is an integer below 2^24, i.e. exactly representable in fp32.
F32_EXACT_K = (1 << 24) // 128


def ternary_weights_dense(codes) -> np.ndarray:
    """The ternary codes as a matrix of -1.0 / 0.0 / +1.0, in fp32 when K <= F32_EXACT_K, else fp64."""
    c = np.asarray(codes)
    return c.astype(np.float32 if c.shape[-1] <= F32_EXACT_K else np.float64)


def ternary_accumulate(q, codes) -> np.ndarray:
    """acc[m, n] = sum over k of q[m,k] * w[n,k] with w in {-1,0,1}, exact.

    [DC] "Replacing MatMul with ternary operations": multiplying by -1 negates,
    by 0 drops, by 1 keeps, so every term is -q, 0 or +q and acc is an integer
    sum. It is evaluated as one library matrix product of q with the codes
    written as -1.0 / 0.0 / +1.0: every partial sum, in whatever order the
    library adds, is an integer of magnitude at most 128 * K, which fp32 holds
    exactly for K <= F32_EXACT_K (fp64 beyond), so the result is exact.
    ``codes`` may be int8 codes or the output of ternary_weights_dense.
    """
    c = np.asarray(codes)
    w = c if c.dtype.kind == "f" else ternary_weights_dense(c)
    qf = np.asarray(q).astype(w.dtype)
    acc = qf @ w.T
    return np.rint(acc).astype(np.int64)


def rescale(acc, gamma, s, bias=None) -> np.ndarray:
    """Scaled ternary accumulation: y = acc * gamma / s (+ bias), fp64.

    [DC] overview figure panel "MatMul vs. scaled ternary accumulation".
    """
    y = np.asarray(acc, dtype=np.float64) * np.float64(gamma) / np.asarray(s, dtype=np.float64)[..., None]
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    return y


def bitlinear(x, lin: TLinear, eps: float = EPS_NORM, parts: bool = False):
    """FusedBitLinear forward: RMSNorm -> absmax int8 quant -> ternary accumulate -> rescale.

    [HL] "FusedBitLinear": RMSNorm, quantisation and accumulation against
    ternary weights in one layer. x: [..., K] -> y: [..., N] fp64.
    """
    x = np.asarray(x)
    lead = x.shape[:-1]
    x2 = x.reshape(-1, x.shape[-1])
    xhat = rmsnorm(x2, lin.gain, eps)
    q, s = absmax_quantize(xhat)
    acc = ternary_accumulate(q, lin.weights())
    y = rescale(acc, lin.gamma, s, lin.bias)
    y = y.reshape(*lead, lin.N)
    if parts:
        return y, dict(xhat=xhat, q=q, s=s, acc=acc)
    return y


# ---------------------------------------------------------------------------
# MLGRU token mixer
# ---------------------------------------------------------------------------


def sigmoid(z) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def mlgru_scan(pf, pc, pg, h0):
    """MLGRU gates and recurrence over pre-activations [B, T, d] (fp64).

    [DC] "Core components: MLGRU and GLU": the MLGRU walks the sequence token
    by token, takes the current token and the previous hidden state, and
    updates the state with element-wise operations and gates valued in [0,1].
    [HL] "HGRN attention": forget-gate and candidate paths, recurrence that
    depends only on the current token and the previous state. The pages print
    no formula; the plainest reading used here:
        f_t = sigmoid(f~_t), c_t = SiLU(c~_t), g_t = sigmoid(g~_t)
        h_t = f_t * h_{t-1} + (1 - f_t) * c_t
        o'_t = g_t * h_t
    Returns (o' [B,T,d] fp64, h_T [B,d] fp64). h is carried in fp64 here.
    """
    pf = np.asarray(pf, dtype=np.float64)
    pc = np.asarray(pc, dtype=np.float64)
    pg = np.asarray(pg, dtype=np.float64)
    h = np.array(h0, dtype=np.float64, copy=True)
    T = pf.shape[1]
    o = np.empty_like(pf)
    for t in range(T):
        f = sigmoid(pf[:, t])
        c = silu(pc[:, t])
        g = sigmoid(pg[:, t])
        h = f * h + (1.0 - f) * c
        o[:, t] = g * h
    return o, h


def rmsnorm_swish_gate(h, pg, w=None, eps: float = EPS_NORM) -> np.ndarray:
    """g_norm output gate: RMSNorm of the recurrence state fused with a swish gate (fp64).

    [HL] "HGRN attention": the token mixer's recurrence output passes g_norm,
    a FusedRMSNormSwishGate (normalisation and swish activation in one step),
    before o_proj. The page prints no formula; the plainest reading used here:
        o'_t = h_t / sqrt(mean_n h_t[n]^2 + eps) * w * swish(g~_t),
        swish(z) = z * sigmoid(z) (= SiLU),
    normalised per token over all d channels (one head), w the gate norm's
    gain (ones when None), eps the block's norm epsilon.
    h, pg: [..., d]. Returns o' [..., d] fp64.
    """
    h = np.asarray(h, dtype=np.float64)
    ms = np.mean(np.square(h), axis=-1, keepdims=True)
    y = h / np.sqrt(ms + eps)
    if w is not None:
        y = y * np.asarray(w, dtype=np.float64)
    return y * silu(pg)


def mlgru_scan_gnorm(pf, pc, pg, h0, w=None, eps: float = EPS_NORM):
    """MLGRU recurrence with the g_norm output gate in place of sigmoid(g~) * h.

    The recurrence is the one of ``mlgru_scan`` (f_t = sigmoid(f~_t),
    c_t = SiLU(c~_t), h_t = f_t h_{t-1} + (1 - f_t) c_t, carried in fp64); the
    output is ``rmsnorm_swish_gate(h_t, g~_t, w, eps)`` at every step.
    Returns (o' [B,T,d] fp64, h_T [B,d] fp64).
    """
    pf = np.asarray(pf, dtype=np.float64)
    pc = np.asarray(pc, dtype=np.float64)
    h = np.array(h0, dtype=np.float64, copy=True)
    T = pf.shape[1]
    hs = np.empty_like(pf)
    for t in range(T):
        f = sigmoid(pf[:, t])
        h = f * h + (1.0 - f) * silu(pc[:, t])
        hs[:, t] = h
    return rmsnorm_swish_gate(hs, pg, w, eps), h


@dataclasses.dataclass
class Block:
    """Ternary weights of one MatMul-free block.

    ``gnorm``: gain of the g_norm output gate ([d] fp32). None selects the
    sigmoid output gate o' = sigmoid(g~) * h; a gain selects
    o' = RMSNorm(h) * gnorm * swish(g~) (``rmsnorm_swish_gate``).
    """
    f: TLinear
    c: TLinear
    g: TLinear
    o: TLinear
    gate: TLinear
    up: TLinear
    down: TLinear
    gnorm: Optional[np.ndarray] = None

    @property
    def d(self) -> int:
        return self.f.K

    @property
    def inner(self) -> int:
        return self.gate.N


def make_block(latents: dict, cache: bool = False, gnorm=None) -> Block:
    """latents: dict of name -> fp32 latent [N, K] for f, c, g, o, gate, up, down.

    gnorm: optional [d] gain selecting the g_norm output gate.
    """
    lins = {k: make_tlinear(latents[k], cache=cache) for k in ("f", "c", "g", "o", "gate", "up", "down")}
    g = None if gnorm is None else np.asarray(gnorm, dtype=np.float32).astype(np.float64)
    return Block(**lins, gnorm=g)


def mlgru_preacts(x, blk: Block, dtype: str, eps: float = EPS_NORM):
    """f~, c~, g~ = BitLinear_{f,c,g}(x), each rounded to the storage type."""
    pf = store(bitlinear(x, blk.f, eps), dtype)
    pc = store(bitlinear(x, blk.c, eps), dtype)
    pg = store(bitlinear(x, blk.g, eps), dtype)
    return pf, pc, pg


def mlgru(x, blk: Block, h0, dtype: str, eps: float = EPS_NORM, parts: bool = False):
    """MLGRU token mixer on x [B,T,d]: projections, gated scan, output gate, o-projection.

    The output gate is sigmoid(g~) * h, or the g_norm gate when ``blk.gnorm`` is
    set. Storage points (the kernels store these tensors): f~/c~/g~ and o' in
    the run dtype, the state h in fp32. Returns (o [B,T,d] fp64 unrounded, h_T fp32 values).
    """
    pf, pc, pg = mlgru_preacts(x, blk, dtype, eps)
    if blk.gnorm is None:
        o_gate, hT = mlgru_scan(pf, pc, pg, h0)
    else:
        o_gate, hT = mlgru_scan_gnorm(pf, pc, pg, h0, blk.gnorm, eps)
    o_gate = store(o_gate, dtype)
    o = bitlinear(o_gate, blk.o, eps)
    hT = round_f32(hT)
    if parts:
        return o, hT, dict(pf=pf, pc=pc, pg=pg, o_gate=o_gate)
    return o, hT


def glu(x, blk: Block, dtype: str, eps: float = EPS_NORM, parts: bool = False):
    """MatMul-free GLU channel mixer.

    [DC] "Core components: MLGRU and GLU": the input goes through two separate
    BitLinear layers; one branch passes SiLU and is multiplied element-wise by
    the other; a third BitLinear gives the output. Reading: the SiLU branch is
    "gate", the other "up": p = SiLU(gate(x)) * up(x), stored in the run dtype;
    returns down(p) in fp64.
    """
    u = bitlinear(x, blk.gate, eps)
    v = bitlinear(x, blk.up, eps)
    p = store(silu(u) * v, dtype)
    y = bitlinear(p, blk.down, eps)
    if parts:
        return y, dict(u=u, v=v, p=p)
    return y


def block_forward(x, blk: Block, h0, dtype: str, eps: float = EPS_NORM, parts: bool = False):
    """One MatMul-free block: y1 = x + MLGRU(x); y = y1 + GLU(y1).

    [HL] "HGRN attention": the block input passes RMSNorm first; [DC] names
    the token mixer (MLGRU) and channel mixer (GLU). Reading: pre-norm blocks
    with residual connections; each BitLinear's own RMSNorm is the block norm.
    x [B,T,d] in the run dtype -> (y [B,T,d] stored, h_T [B,d] fp32 values).
    """
    x = store(x, dtype)
    o, hT, p1 = mlgru(x, blk, h0, dtype, eps, parts=True)
    y1 = store(x + o, dtype)
    g, p2 = glu(y1, blk, dtype, eps, parts=True)
    y = store(y1 + g, dtype)
    if parts:
        return y, hT, dict(y1=y1, o=o, **p1, **p2)
    return y, hT


def stack_forward(x, blocks, h0s, dtype: str, eps: float = EPS_NORM):
    """L blocks in sequence; h0s [L,B,d]. Returns (y, h_T [L,B,d])."""
    hs = []
    for l, blk in enumerate(blocks):
        x, h = block_forward(x, blk, h0s[l], dtype, eps)
        hs.append(h)
    return x, np.stack(hs)


# ---------------------------------------------------------------------------
# Model ends: embedding lookup, LM head, greedy next token
# ---------------------------------------------------------------------------


def embed(ids, table, dtype: str) -> np.ndarray:
    """Token embedding: x[m] = E[ids[m]], stored in the run dtype.

    [HL] "Install and model initialisation": the default configuration has an
    embedding of 32000 entries at hidden size 2048. A lookup is a row copy;
    an id outside [0, V) is an error (IndexError).
    """
    ids = np.asarray(ids, dtype=np.int64)
    E = np.asarray(table, dtype=np.float64)
    if ids.size and (ids.min() < 0 or ids.max() >= E.shape[0]):
        raise IndexError("token id outside [0, V)")
    return store(E[ids], dtype)


def lm_logits(x, head: TLinear, dtype: str, eps: float = EPS_NORM) -> np.ndarray:
    """Logits of the language-model head, stored in the run dtype.

    [HL] "FusedBitLinear": every linear projection of the model is a
    FusedBitLinear. Reading: so is the head, logits = BitLinear_head(x)
    ([d] -> [V]); its own RMSNorm is the final norm.
    """
    return store(bitlinear(x, head, eps), dtype)


def greedy_token(logits) -> np.ndarray:
    """Index of the largest logit of each row, the lowest index on ties.

    [HL] "Official generation example" samples the next token (top-p 0.4,
    temperature 0.6); the deterministic reading taken for the on-device loop
    is greedy decoding, the argmax of the stored logits.
    """
    L = np.asarray(logits, dtype=np.float64)
    return np.argmax(L, axis=-1).astype(np.int64)   # first occurrence of the maximum


def model_forward(ids, table, blocks, head: TLinear, h0s, dtype: str, eps: float = EPS_NORM):
    """Embedding -> L blocks -> LM head on the last token of each sequence.

    ids [B, T] -> (logits [B, V] of token T-1, h_T [L, B, d]).
    """
    x = embed(ids, table, dtype)
    y, hs = stack_forward(x, blocks, h0s, dtype, eps)
    return lm_logits(y[:, -1], head, dtype, eps), hs


def generate_greedy(prompt, n: int, table, blocks, head: TLinear, dtype: str, eps: float = EPS_NORM):
    """Greedy generation of n tokens after a prompt [B, T0] (T0 >= 1), state carried.

    The prompt runs as one prefill; each new token is the greedy token of the
    previous step's logits and is fed back as a one-token step.
    Returns (tokens [B, n], h_T [L, B, d]).
    """
    prompt = np.asarray(prompt, dtype=np.int64)
    B = prompt.shape[0]
    d = blocks[0].d
    logits, hs = model_forward(prompt, table, blocks, head, np.zeros((len(blocks), B, d)), dtype, eps)
    out = []
    for _ in range(n):
        tok = greedy_token(logits)
        out.append(tok)
        logits, hs = model_forward(tok[:, None], table, blocks, head, hs, dtype, eps)
    return np.stack(out, axis=1) if out else np.zeros((B, 0), np.int64), hs


# ---------------------------------------------------------------------------
# Training: the MLGRU recurrence backward
# ---------------------------------------------------------------------------


def mlgru_scan_backward(pf, pc, pg, h0, do, dhT=None):
    """Gradients of the MLGRU scan (``mlgru_scan``) for upstream gradients do = dL/do' [B,T,d]
    and dhT = dL/dh_T [B,d] (zero when None), in fp64.

    [DC] "Memory efficiency" / "From optimised GPU to custom FPGA design": the
    models are trained with fused GPU kernels; the pages give no backward
    formula, so this is the exact derivative of the forward reading
        f = sigmoid(f~), c = SiLU(c~), g = sigmoid(g~),
        h_t = f_t h_{t-1} + (1 - f_t) c_t,  o'_t = g_t h_t.
    With lambda_t = dL/dh_t (through o'_t and h_{t+1}):
        lambda_T = do_T g_T + dhT,  lambda_t = do_t g_t + f_{t+1} lambda_{t+1}
        dg~_t = do_t h_t g_t (1 - g_t)
        df~_t = lambda_t (h_{t-1} - c_t) f_t (1 - f_t)
        dc~_t = lambda_t (1 - f_t) SiLU'(c~_t),  SiLU'(z) = s (1 + z (1 - s)), s = sigmoid(z)
        dh0 = f_1 lambda_1
    Returns (dpf, dpc, dpg [B,T,d], dh0 [B,d]).
    """
    pf = np.asarray(pf, dtype=np.float64)
    pc = np.asarray(pc, dtype=np.float64)
    pg = np.asarray(pg, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, T, d = pf.shape
    f, g = sigmoid(pf), sigmoid(pg)
    sc = sigmoid(pc)
    c = pc * sc
    hs = np.empty((B, T + 1, d))
    hs[:, 0] = np.asarray(h0, dtype=np.float64)
    for t in range(T):
        hs[:, t + 1] = f[:, t] * hs[:, t] + (1.0 - f[:, t]) * c[:, t]
    lam = np.zeros((B, d)) if dhT is None else np.array(dhT, dtype=np.float64, copy=True)
    dpf, dpc, dpg = np.empty_like(pf), np.empty_like(pf), np.empty_like(pf)
    for t in range(T - 1, -1, -1):
        lam = lam + do[:, t] * g[:, t]                 # lambda_t
        h, hp = hs[:, t + 1], hs[:, t]
        dpg[:, t] = do[:, t] * h * g[:, t] * (1.0 - g[:, t])
        dpf[:, t] = lam * (hp - c[:, t]) * f[:, t] * (1.0 - f[:, t])
        dpc[:, t] = lam * (1.0 - f[:, t]) * sc[:, t] * (1.0 + pc[:, t] * (1.0 - sc[:, t]))
        lam = f[:, t] * lam                             # the part of lambda_{t-1} through h_t
    return dpf, dpc, dpg, lam
