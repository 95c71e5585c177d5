"""Thin torch-facing binding of libmmf.so: argument marshalling only.

Every step of the computation runs in the library's CUDA kernels. Torch is
used to hold device memory and to name the current CUDA stream. There is no
CPU path: without the built library or without a CUDA tensor, calls fail.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _lib as L

_DT = {torch.float32: L.MMF_F32, torch.bfloat16: L.MMF_BF16}
DEFAULT_EPS = 1e-6


def _vp(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts: Optional[torch.Tensor]) -> None:
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("mmf needs CUDA tensors (there is no CPU path)")
            if not t.is_contiguous():
                raise ValueError("mmf needs contiguous tensors")


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported activation dtype {t.dtype}")
    return _DT[t.dtype]


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace too small: {ws.numel() * ws.element_size()} < {nbytes}")
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def version() -> str:
    return L.load().mmf_version().decode()


def check(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Synchronise and raise if a kernel recorded a device-side error."""
    s = stream if stream is not None else torch.cuda.current_stream()
    L.check(L.load().mmf_check(ctypes.c_void_p(s.cuda_stream)), "mmf_check")


class TLinear:
    """A ternary BitLinear held on the device: packed [N, K/16] (int32 storage of uint32), gamma [1],
    optionally codes [N, K] uint8 (the same codes one byte per weight, see unpack_codes)."""

    def __init__(self, packed: torch.Tensor, gamma: torch.Tensor, N: int, K: int,
                 gain: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                 codes: Optional[torch.Tensor] = None):
        _need_cuda(packed, gamma, gain, bias, codes)
        self.packed, self.gamma, self.gain, self.bias, self.codes = packed, gamma, gain, bias, codes
        self.N, self.K = int(N), int(K)

    def c(self) -> L.TLinear:
        return L.TLinear(self.packed.data_ptr(), self.gamma.data_ptr(),
                         self.gain.data_ptr() if self.gain is not None else None,
                         self.bias.data_ptr() if self.bias is not None else None, self.N, self.K,
                         self.codes.data_ptr() if self.codes is not None else None)


def unpack_codes(lin: TLinear) -> TLinear:
    """The same layer with its codes also held one byte per weight (mmf_unpack_codes), which the
    prefill contraction loads directly instead of expanding the packed words."""
    lib = L.load()
    codes = torch.empty((lin.N, lin.K), dtype=torch.uint8, device=lin.packed.device)
    L.check(lib.mmf_unpack_codes(_vp(lin.packed), lin.N, lin.K, _vp(codes), _stream(lin.packed.device)),
            "mmf_unpack_codes")
    return TLinear(lin.packed, lin.gamma, lin.N, lin.K, lin.gain, lin.bias, codes)


def quantize_weights(W: torch.Tensor, gain: Optional[torch.Tensor] = None,
                     bias: Optional[torch.Tensor] = None) -> TLinear:
    """Absmean-ternarise and pack a latent fp32 weight [N, K] on the device (mmf_quantize_weights)."""
    _need_cuda(W)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 CUDA tensor")
    lib = L.load()
    N, K = W.shape
    packed = torch.empty((N, max(K // 16, 1)), dtype=torch.int32, device=W.device)
    gamma = torch.empty(4, dtype=torch.float32, device=W.device)   # 16-byte slot, element 0 used
    ws = _workspace(lib.mmf_quantize_weights_ws_size(N, K), W.device, None)
    L.check(lib.mmf_quantize_weights(_vp(W), N, K, _vp(packed), _vp(gamma), _vp(ws), ws.numel(),
                                     _stream(W.device)), "mmf_quantize_weights")
    return TLinear(packed, gamma, N, K, gain, bias)


def bitlinear(lin: TLinear, x: torch.Tensor, eps: float = DEFAULT_EPS, debug: bool = False,
              ws: Optional[torch.Tensor] = None):
    """y = BitLinear(x) for x [..., K]; with debug=True also returns (q, s, acc)."""
    _need_cuda(x)
    lib = L.load()
    lead = x.shape[:-1]
    M = int(x.numel() // x.shape[-1]) if x.shape[-1] else 0
    y = torch.empty(*lead, lin.N, dtype=x.dtype, device=x.device)
    w = _workspace(lib.mmf_bitlinear_ws_size(M, lin.K), x.device, ws)
    dbg = None
    if debug:
        q = torch.empty(M, lin.K, dtype=torch.int8, device=x.device)
        s = torch.empty(M, dtype=torch.float32, device=x.device)
        acc = torch.empty(M, lin.N, dtype=torch.int32, device=x.device)
        dbg = L.BitlinearDebug(q.data_ptr(), s.data_ptr(), acc.data_ptr())
    cl = lin.c()
    L.check(lib.mmf_bitlinear(ctypes.byref(cl), _vp(x), _dtype(x), M, _vp(y), eps, _vp(w),
                              w.numel() * w.element_size(), _stream(x.device),
                              ctypes.byref(dbg) if dbg is not None else None), "mmf_bitlinear")
    if debug:
        return y, q, s, acc
    return y


def mlgru_scan(pre: torch.Tensor, h: torch.Tensor, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """pre [B, T, 3, d] -> o' [B, T, d]; h [B, d] fp32 is updated in place to h_T."""
    _need_cuda(pre, h)
    if pre.dim() != 4 or pre.shape[2] != 3:
        raise ValueError("pre must be [B, T, 3, d]")
    B, T, _, d = pre.shape
    if h.dtype != torch.float32 or tuple(h.shape) != (B, d):
        raise ValueError("h must be float32 [B, d]")
    o = torch.empty(B, T, d, dtype=pre.dtype, device=pre.device)
    lib = L.load()
    w = _workspace(lib.mmf_mlgru_scan_ws_size(B, T, d), pre.device, ws)
    L.check(lib.mmf_mlgru_scan(_vp(pre), _dtype(pre), B, T, d, _vp(h), _vp(o), _vp(w), w.numel() * w.element_size(),
                               _stream(pre.device)), "mmf_mlgru_scan")
    return o


def mlgru_scan_gnorm(pre: torch.Tensor, h: torch.Tensor, gain: torch.Tensor, eps: float = DEFAULT_EPS,
                     ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The scan with the g_norm output gate: o' = RMSNorm(h) * gain * swish(g~).

    pre [B, T, 3, d] -> o' [B, T, d]; h [B, d] fp32 is updated in place to h_T;
    gain float32 [d].
    """
    _need_cuda(pre, h, gain)
    if pre.dim() != 4 or pre.shape[2] != 3:
        raise ValueError("pre must be [B, T, 3, d]")
    B, T, _, d = pre.shape
    if h.dtype != torch.float32 or tuple(h.shape) != (B, d):
        raise ValueError("h must be float32 [B, d]")
    if gain.dtype != torch.float32 or tuple(gain.shape) != (d,):
        raise ValueError("gain must be float32 [d]")
    o = torch.empty(B, T, d, dtype=pre.dtype, device=pre.device)
    lib = L.load()
    w = _workspace(lib.mmf_mlgru_scan_gnorm_ws_size(B, T, d), pre.device, ws)
    L.check(lib.mmf_mlgru_scan_gnorm(_vp(pre), _dtype(pre), B, T, d, _vp(h), _vp(gain), eps, _vp(o), _vp(w),
                                     w.numel() * w.element_size(), _stream(pre.device)), "mmf_mlgru_scan_gnorm")
    return o


def mlgru_scan_states(pre: torch.Tensor, h: torch.Tensor, want_o: bool = True):
    """Training forward: (o' [B, T, d] or None, hs [B, T, d] fp32); h [B, d] is updated in place to h_T."""
    _need_cuda(pre, h)
    B, T, _, d = pre.shape
    o = torch.empty(B, T, d, dtype=pre.dtype, device=pre.device) if want_o else None
    hs = torch.empty(B, T, d, dtype=torch.float32, device=pre.device)
    L.check(L.load().mmf_mlgru_scan_states(_vp(pre), _dtype(pre), B, T, d, _vp(h), _vp(o), _vp(hs),
                                           _stream(pre.device)), "mmf_mlgru_scan_states")
    return o, hs


def mlgru_scan_backward(pre: torch.Tensor, h0: torch.Tensor, dout: torch.Tensor,
                        dhT: Optional[torch.Tensor] = None, hs: Optional[torch.Tensor] = None,
                        ws: Optional[torch.Tensor] = None):
    """Gradients of mlgru_scan: (dpre [B, T, 3, d] in pre's dtype, dh0 [B, d] fp32) for
    dout = dL/do' [B, T, d] and dhT = dL/dh_T [B, d] (zero when None); hs: the forward states
    from mlgru_scan_states (recomputed when None)."""
    _need_cuda(pre, h0, dout, dhT, hs)
    B, T, _, d = pre.shape
    if dout.shape != (B, T, d) or dout.dtype != pre.dtype:
        raise ValueError("dout must be [B, T, d] in pre's dtype")
    dpre = torch.empty_like(pre)
    dh0 = torch.empty(B, d, dtype=torch.float32, device=pre.device)
    lib = L.load()
    w = None if hs is not None else _workspace(lib.mmf_mlgru_scan_backward_ws_size(B, T, d), pre.device, ws)
    L.check(lib.mmf_mlgru_scan_backward(_vp(pre), _dtype(pre), B, T, d, _vp(h0), _vp(dout), _vp(dhT), _vp(hs),
                                        _vp(dpre), _vp(dh0), _vp(w), 0 if w is None else w.numel() * w.element_size(),
                                        _stream(pre.device)),
            "mmf_mlgru_scan_backward")
    return dpre, dh0


def glu(gate: TLinear, up: TLinear, down: TLinear, x: torch.Tensor, residual: Optional[torch.Tensor] = None,
        eps: float = DEFAULT_EPS, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = down(SiLU(gate(x)) * up(x)) (+ residual) for x [..., d]."""
    _need_cuda(x, residual)
    lib = L.load()
    d = x.shape[-1]
    M = int(x.numel() // d)
    y = torch.empty_like(x)
    w = _workspace(lib.mmf_glu_ws_size(M, d, gate.N), x.device, ws)
    cg, cu, cd = gate.c(), up.c(), down.c()
    L.check(lib.mmf_glu(ctypes.byref(cg), ctypes.byref(cu), ctypes.byref(cd), _vp(x), _vp(residual), _vp(y), M,
                        _dtype(x), eps, _vp(w), w.numel() * w.element_size(), _stream(x.device)), "mmf_glu")
    return y


class Block:
    """Handle of one MatMul-free block (mmf_block_create); keeps its weight tensors alive."""

    NAMES = ("f", "c", "g", "o", "gate", "up", "down")

    def __init__(self, lins: dict, gnorm: Optional[torch.Tensor] = None):
        """lins: name -> TLinear for NAMES; gnorm: float32 [d] gain selecting the g_norm output gate."""
        self.lins = dict(lins)
        self.d = self.lins["f"].K
        self.inner = self.lins["gate"].N
        if gnorm is not None:
            _need_cuda(gnorm)
            if gnorm.dtype != torch.float32 or tuple(gnorm.shape) != (self.d,) or not gnorm.is_contiguous():
                raise ValueError("gnorm must be a contiguous float32 [d] tensor")
        self.gnorm = gnorm
        bw = L.BlockWeights(*[self.lins[n].c() for n in self.NAMES], _vp(gnorm))
        h = ctypes.c_void_p()
        lib = L.load()
        L.check(lib.mmf_block_create(ctypes.byref(bw), self.d, self.inner, ctypes.byref(h)), "mmf_block_create")
        self.handle = h

    def ws_size(self, B: int, T: int) -> int:
        return int(L.load().mmf_block_ws_size(self.handle, B, T))

    def release_codes(self) -> None:
        """Free the one-byte code copy made by the first prefill call (mmf_block_release_codes)."""
        L.check(L.load().mmf_block_release_codes(self.handle), "mmf_block_release_codes")

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            L.load().mmf_block_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class State:
    """Recurrent MLGRU state h [L, B, d] fp32 owned by the library (mmf_state_create)."""

    def __init__(self, L_: int, B: int, d: int):
        self.L, self.B, self.d = int(L_), int(B), int(d)
        h = ctypes.c_void_p()
        L.check(L.load().mmf_state_create(self.L, self.B, self.d, ctypes.byref(h)), "mmf_state_create")
        self.handle = h

    def reset(self):
        L.check(L.load().mmf_state_reset(self.handle, _stream(torch.device("cuda"))), "mmf_state_reset")

    def get(self) -> torch.Tensor:
        out = torch.empty(self.L, self.B, self.d, dtype=torch.float32)
        L.check(L.load().mmf_state_get(self.handle, ctypes.c_void_p(out.data_ptr()),
                                       _stream(torch.device("cuda"))), "mmf_state_get")
        return out

    def set(self, h: torch.Tensor):
        h = h.detach().to("cpu", torch.float32).contiguous()
        if tuple(h.shape) != (self.L, self.B, self.d):
            raise ValueError("state shape mismatch")
        L.check(L.load().mmf_state_set(self.handle, ctypes.c_void_p(h.data_ptr()),
                                       _stream(torch.device("cuda"))), "mmf_state_set")

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            L.load().mmf_state_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def block_forward(block: Block, layer: int, state: State, x: torch.Tensor, eps: float = DEFAULT_EPS,
                  ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x [B, T, d] -> y [B, T, d] through one block, continuing state layer `layer`."""
    _need_cuda(x)
    B, T, d = x.shape
    y = out if out is not None else torch.empty_like(x)
    w = _workspace(block.ws_size(B, T), x.device, ws)
    L.check(L.load().mmf_block_forward(block.handle, layer, state.handle, _vp(x), _vp(y), B, T, _dtype(x), eps,
                                       _vp(w), w.numel() * w.element_size(), _stream(x.device)),
            "mmf_block_forward")
    return y


def block_forward_debug(block: Block, layer: int, state: State, x: torch.Tensor, eps: float = DEFAULT_EPS,
                        ws: Optional[torch.Tensor] = None):
    """block_forward that also returns the stored intermediates (mmf_block_forward_debug): a dict with
    pre [B, T, 3, d], og [B, T, d], y1 [B, T, d], p [B, T, I], and q[i] / s[i] (int8 codes [M, K] and
    scales [M] of the i-th quantised input: 0 x, 1 o', 2 y1, 3 p)."""
    _need_cuda(x)
    B, T, d = x.shape
    M, I = B * T, block.inner
    dev = x.device
    y = torch.empty_like(x)
    w = _workspace(block.ws_size(B, T), dev, ws)
    out = {"pre": torch.empty(B, T, 3, d, dtype=x.dtype, device=dev),
           "og": torch.empty(B, T, d, dtype=x.dtype, device=dev),
           "y1": torch.empty(B, T, d, dtype=x.dtype, device=dev),
           "p": torch.empty(B, T, I, dtype=x.dtype, device=dev),
           "q": [torch.empty(M, k, dtype=torch.int8, device=dev) for k in (d, d, d, I)],
           "s": [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(4)]}
    dbg = L.BlockDebug(out["pre"].data_ptr(), out["og"].data_ptr(), out["y1"].data_ptr(), out["p"].data_ptr(),
                       (L.c_vp * 4)(*[t.data_ptr() for t in out["q"]]),
                       (L.c_vp * 4)(*[t.data_ptr() for t in out["s"]]))
    L.check(L.load().mmf_block_forward_debug(block.handle, layer, state.handle, _vp(x), _vp(y), B, T, _dtype(x), eps,
                                             _vp(w), w.numel() * w.element_size(), _stream(dev), ctypes.byref(dbg)),
            "mmf_block_forward_debug")
    return y, out


def stack_ws_size(blocks: Sequence[Block], B: int, T: int) -> int:
    return max(b.ws_size(B, T) for b in blocks)


def stack_forward(blocks: Sequence[Block], state: State, x: torch.Tensor, eps: float = DEFAULT_EPS,
                  ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x [B, T, d] through len(blocks) blocks (state layer l for block l)."""
    _need_cuda(x)
    B, T, d = x.shape
    y = out if out is not None else torch.empty_like(x)
    w = _workspace(stack_ws_size(blocks, B, T), x.device, ws)
    arr = (ctypes.c_void_p * len(blocks))(*[b.handle.value for b in blocks])
    L.check(L.load().mmf_stack_forward(arr, len(blocks), state.handle, _vp(x), _vp(y), B, T, _dtype(x), eps,
                                       _vp(w), w.numel() * w.element_size(), _stream(x.device)),
            "mmf_stack_forward")
    return y


# ---------------------------------------------------------------- model ends

def embed(table: torch.Tensor, ids: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x[..., :] = table[ids[...], :] (mmf_embed); table [V, d], ids int32 on the device."""
    _need_cuda(table, ids)
    if table.dim() != 2 or ids.dtype != torch.int32 or not ids.is_contiguous() or not table.is_contiguous():
        raise ValueError("table must be a contiguous [V, d] tensor and ids contiguous int32")
    V, d = table.shape
    x = out if out is not None else torch.empty(*ids.shape, d, dtype=table.dtype, device=table.device)
    L.check(L.load().mmf_embed(_vp(ids), ids.numel(), _vp(table), V, d, _dtype(table), _vp(x),
                               _stream(table.device)), "mmf_embed")
    return x


def argmax(logits: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Greedy next token of each row of logits [..., V] (mmf_argmax): int32, lowest index on ties."""
    _need_cuda(logits)
    if not logits.is_contiguous():
        raise ValueError("logits must be contiguous")
    V = logits.shape[-1]
    ids = out if out is not None else torch.empty(logits.shape[:-1], dtype=torch.int32, device=logits.device)
    L.check(L.load().mmf_argmax(_vp(logits), _dtype(logits), logits.numel() // V, V, _vp(ids),
                                _stream(logits.device)), "mmf_argmax")
    return ids


class Model:
    """Embedding -> blocks -> LM head (a BitLinear d -> V) -> greedy next token.

    table: [V, d] embedding in the run dtype; blocks: Block handles; head: TLinear with K = d.
    Every step is a library call; the torch tensors here are buffers only.
    """

    def __init__(self, table: torch.Tensor, blocks: Sequence[Block], head: TLinear):
        if head.K != table.shape[1] or any(b.d != table.shape[1] for b in blocks):
            raise ValueError("embedding width, block width and head input must agree")
        self.table, self.blocks, self.head = table, list(blocks), head
        self.V, self.d = table.shape

    def forward(self, state: State, ids: torch.Tensor, eps: float = DEFAULT_EPS) -> torch.Tensor:
        """ids [B, T] int32 -> logits [B, V] of each sequence's last token; the state is carried."""
        B, T = ids.shape
        x = embed(self.table, ids)
        y = stack_forward(self.blocks, state, x, eps)
        if T > 1:   # the last token of each sequence: a row lookup into y viewed as [B*T, d]
            last = torch.arange(T - 1, B * T, T, dtype=torch.int32, device=ids.device)
            y = embed(y.reshape(B * T, self.d), last)
        return bitlinear(self.head, y.reshape(B, self.d), eps)

    def generate(self, state: State, prompt: torch.Tensor, n: int, eps: float = DEFAULT_EPS) -> torch.Tensor:
        """Greedy generation of n tokens after prompt [B, T0]: int32 [B, n]."""
        logits = self.forward(state, prompt, eps)
        out = []
        for _ in range(n):
            tok = argmax(logits)
            out.append(tok)
            logits = self.forward(state, tok.reshape(-1, 1), eps)
        return torch.stack(out, 1) if out else torch.empty(prompt.shape[0], 0, dtype=torch.int32,
                                                              device=prompt.device)


# ---------------------------------------------------------------- launch timing

def prof_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (mmf_prof_enable)."""
    L.check(L.load().mmf_prof_enable(1 if on else 0), "mmf_prof_enable")


def prof_reset() -> None:
    L.load().mmf_prof_reset()


def prof_collect() -> dict:
    """{kernel name: (launches, total device ms)} since the last prof_reset()."""
    lib = L.load()
    n = lib.mmf_prof_collect()
    if n < 0:
        raise L.MMFError(5, "mmf_prof_collect", lib.mmf_last_error().decode())
    out = {}
    buf = ctypes.create_string_buffer(128)
    for i in range(n):
        launches = ctypes.c_int64()
        ms = ctypes.c_double()
        L.check(lib.mmf_prof_get(i, buf, 128, ctypes.byref(launches), ctypes.byref(ms)), "mmf_prof_get")
        out[buf.value.decode()] = (int(launches.value), float(ms.value))
    return out
