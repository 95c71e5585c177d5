"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bit-exact: ternary codes (given the GPU's gamma), int32 accumulators (given the
GPU's activation codes). Activation codes: within 1 on <= 0.01% of elements.
Floating outputs: normwise 2e-3, storage-type rounding flips allowed (tests/parity.py).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import (E2E_TOL, TORCH_DT, assert_close, assert_codes_close, make_block, make_layer, packed_to_np, to_np)

pytestmark = pytest.mark.gpu

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")


# ------------------------------------------------------------------ weights

@pytest.mark.parametrize("n,k", [(2048, 2048), (5632, 2048), (2048, 5632), (37, 48), (1, 16), (3, 4096)])
def test_quantize_weights_bit_exact(n, k):
    W = synth.latent_weight(100 + n + k, n, k)
    lin = mmf.quantize_weights(W.cuda())
    g_gpu = np.float32(lin.gamma[0].item())
    g_ref, codes_ref = O.ternarize(W.numpy())
    assert abs(float(g_gpu) - float(g_ref)) <= float(np.spacing(g_ref)), (g_gpu, g_ref)
    _, codes_given = O.ternarize(W.numpy(), gamma=g_gpu)
    codes_gpu = O.unpack_codes(packed_to_np(lin.packed), k)
    np.testing.assert_array_equal(codes_gpu, codes_given)
    if g_gpu == g_ref:
        np.testing.assert_array_equal(codes_gpu, codes_ref)


def test_quantize_weights_is_deterministic():
    W = synth.latent_weight(5, 1024, 1024).cuda()
    a = mmf.quantize_weights(W)
    b = mmf.quantize_weights(W)
    assert torch.equal(a.packed, b.packed) and torch.equal(a.gamma[:1], b.gamma[:1])


# ------------------------------------------------------------------ BitLinear

SWEEP = [(k, n, m) for (k, n) in synth.GEMV_SWEEP_SHAPES for m in synth.GEMV_SWEEP_TOKENS]
RAGGED = [(48, 37, 3), (16, 1, 1), (272, 130, 9), (2048, 2048, 33), (1024, 3072, 130)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k,n,m", SWEEP + RAGGED)
def test_bitlinear_parity(k, n, m, dtype):
    W, lin, olin = make_layer(200 + k + n, n, k)
    x = synth.activations(300 + m, m, k, TORCH_DT[dtype], outlier_p=synth.GEMV_OUTLIER_P,
                          outlier_scale=synth.GEMV_OUTLIER_SCALE)
    y, q, s, acc = mmf.bitlinear(lin, x.cuda(), debug=True)
    torch.cuda.synchronize()
    xn = to_np(x)
    y_ref, parts = O.bitlinear(xn, olin, parts=True)
    np.testing.assert_allclose(to_np(s), parts["s"], rtol=1e-6)
    assert_codes_close(q.cpu().numpy(), parts["q"], "activation codes")
    codes_gpu = O.unpack_codes(packed_to_np(lin.packed), k)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64),
                                  O.ternary_accumulate(q.cpu().numpy(), codes_gpu))
    assert_close(to_np(y), y_ref, dtype, "y")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k,n,m", SWEEP + [(48, 37, 3), (272, 130, 9), (6912, 2560, 16), (1024, 64, 11)])
def test_bitlinear_gain_parity_no_debug(k, n, m, dtype):
    # decode-sized calls without debug outputs, with a non-trivial RMSNorm gain
    W, lin, olin = make_layer(600 + k + n, n, k)
    gain = torch.linspace(0.5, 1.5, k)
    lin = mmf.TLinear(lin.packed, lin.gamma, n, k, gain=gain.cuda())
    olin = O.TLinear(olin.codes, olin.gamma, gain.numpy())
    x = synth.activations(601 + m, m, k, TORCH_DT[dtype], outlier_p=synth.GEMV_OUTLIER_P,
                          outlier_scale=synth.GEMV_OUTLIER_SCALE)
    y = mmf.bitlinear(lin, x.cuda())
    assert_close(to_np(y), O.bitlinear(to_np(x), olin), dtype, "y (gain)")


def test_bitlinear_empty_and_gain_bias():
    k, n = 64, 40
    W, lin, olin = make_layer(17, n, k)
    y = mmf.bitlinear(lin, torch.empty(0, k, device="cuda"))
    assert y.shape == (0, n)
    gain = torch.linspace(-1.5, 2.0, k)
    bias = torch.linspace(-0.3, 0.4, n)
    lin2 = mmf.TLinear(lin.packed, lin.gamma, n, k, gain=gain.cuda(), bias=bias.cuda())
    olin2 = O.TLinear(olin.codes, olin.gamma, gain.numpy(), bias.numpy().astype(np.float64))
    x = synth.activations(18, 7, k)
    y = mmf.bitlinear(lin2, x.cuda())
    assert_close(to_np(y), O.bitlinear(x.numpy(), olin2), "f32", "y with gain and bias")


def test_bitlinear_zero_rows():
    k, n = 128, 64
    _, lin, _ = make_layer(19, n, k)
    x = torch.zeros(5, k, device="cuda")
    x[2] = 1.0
    y, q, s, acc = mmf.bitlinear(lin, x, debug=True)
    assert torch.all(y[[0, 1, 3, 4]] == 0) and torch.all(q[0] == 0)
    assert torch.all(q[2] == 127)


# ------------------------------------------------------------------ MLGRU scan

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
# (8, 300, 2560) has enough 64-channel blocks to fill every SM twice: the
# 64-channel variant; the others run 32-channel CTAs, two per SM
@pytest.mark.parametrize("b,t,d", [(2, 64, 256), (1, 3, 16), (3, 200, 264), (8, 1, 1024), (4, 517, 2048),
                                   (8, 300, 2560)])
def test_scan_parity(b, t, d, dtype):
    pre = synth.preacts(400 + t, b, t, d, TORCH_DT[dtype], scale=2.0)
    h0 = synth.activations(401, b, d)
    h = h0.cuda().clone()
    o = mmf.mlgru_scan(pre.cuda(), h)
    p = to_np(pre)
    o_ref, h_ref = O.mlgru_scan(p[:, :, 0], p[:, :, 1], p[:, :, 2], h0.numpy().astype(np.float64))
    assert_close(to_np(o), O.store(o_ref, dtype), dtype, "o'")
    assert_close(to_np(h), h_ref, "f32", "h_T")


def test_scan_closed_forms_on_gpu():
    b, t, d = 2, 10, 32
    pre = synth.preacts(402, b, t, d)
    pre[:, :, 0] = -1e4   # f = 0 -> h = c
    h = torch.full((b, d), 7.0, device="cuda")
    o = mmf.mlgru_scan(pre.cuda(), h)
    c = O.silu(pre[:, :, 1].numpy().astype(np.float64))
    g = O.sigmoid(pre[:, :, 2].numpy().astype(np.float64))
    assert_close(to_np(o), g * c, "f32", "f=0")
    pre[:, :, 0] = 1e4    # f = 1 -> h = h0
    h = torch.full((b, d), 7.0, device="cuda")
    o = mmf.mlgru_scan(pre.cuda(), h)
    # the kernel's gates carry a few ulp of rounding, so "holds the state" is to rounding
    torch.testing.assert_close(h, torch.full_like(h, 7.0), rtol=1e-5, atol=0)
    assert_close(to_np(o), g * 7.0, "f32", "f=1")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("b,t,d", [(2, 64, 256), (1, 3, 16), (3, 200, 264), (8, 1, 1024), (4, 517, 2048),
                                   (8, 300, 2560)])
def test_scan_gnorm_parity(b, t, d, dtype):
    # the g_norm output gate: both CTA widths, ragged chunks and channel blocks, T = 1
    pre = synth.preacts(420 + t, b, t, d, TORCH_DT[dtype], scale=2.0)
    h0 = synth.activations(421, b, d)
    gain = synth.gains(422, d)
    h = h0.cuda().clone()
    o = mmf.mlgru_scan_gnorm(pre.cuda(), h, gain.cuda())
    mmf.check()
    p = to_np(pre)
    o_ref, h_ref = O.mlgru_scan_gnorm(p[:, :, 0], p[:, :, 1], p[:, :, 2], h0.numpy().astype(np.float64),
                                      gain.numpy())
    assert_close(to_np(o), o_ref, dtype, "o' (g_norm)")
    assert_close(to_np(h), h_ref, "f32", "h_T (g_norm)")


def test_scan_gnorm_closed_forms_on_gpu():
    b, t, d = 2, 150, 64
    pre = synth.preacts(423, b, t, d)
    ones = torch.ones(d, device="cuda")
    # g~ = 0: swish(0) = 0, so o' = 0 exactly whatever the state
    z0 = pre.clone()
    z0[:, :, 2] = 0.0
    o = mmf.mlgru_scan_gnorm(z0.cuda(), torch.full((b, d), 3.0, device="cuda"), ones)
    assert torch.all(o == 0)
    # constant g~ = z, unit gain: each token's mean of o'^2 is swish(z)^2 ms / (ms + eps), ms the
    # mean square of that token's state, read from the sigmoid-gate scan with g~ = 1e4 (o' = h)
    z, eps = 0.8, 1e-3
    zc = pre.clone()
    zc[:, :, 2] = z
    o = mmf.mlgru_scan_gnorm(zc.cuda(), torch.zeros(b, d, device="cuda"), ones, eps=eps)
    zh = pre.clone()
    zh[:, :, 2] = 1e4
    hs = to_np(mmf.mlgru_scan(zh.cuda(), torch.zeros(b, d, device="cuda")))
    ms = np.mean(hs * hs, axis=-1)
    np.testing.assert_allclose(np.mean(to_np(o) ** 2, axis=-1), O.silu(z) ** 2 * ms / (ms + eps), rtol=1e-5)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("b,t,d,with_dhT", [(2, 64, 256, True), (1, 3, 16, False), (3, 200, 264, True),
                                            (8, 1, 1024, True), (4, 517, 2048, False), (8, 300, 2560, True)])
def test_scan_backward_parity(b, t, d, with_dhT, dtype):
    # training: the scan's gradients against the oracle's exact derivative,
    # ragged chunks and channel blocks, T = 1, with and without dL/dh_T
    pre = synth.preacts(440 + t, b, t, d, TORCH_DT[dtype], scale=2.0)
    h0 = synth.activations(441, b, d)
    dout = synth.activations(442 + t, b * t, d, TORCH_DT[dtype]).reshape(b, t, d)
    dhT = synth.activations(443, b, d) if with_dhT else None
    dpre, dh0 = mmf.mlgru_scan_backward(pre.cuda(), h0.cuda(), dout.cuda(), None if dhT is None else dhT.cuda())
    mmf.check()
    p = to_np(pre)
    ref = O.mlgru_scan_backward(p[:, :, 0], p[:, :, 1], p[:, :, 2], h0.numpy().astype(np.float64), to_np(dout),
                                None if dhT is None else dhT.numpy().astype(np.float64))
    g = to_np(dpre)
    for j, name in enumerate(("df~", "dc~", "dg~")):
        assert_close(g[:, :, j], ref[j], dtype, name)
    assert_close(to_np(dh0), ref[3], "f32", "dh0")


def test_scan_wait_gives_up_and_reports(monkeypatch):
    # failure detection without a fault: chunk 1 of CTA 0 is never loaded, so
    # its bounded wait runs out (20 ms); the kernel lets its other copies land
    # and returns, mmf_check reports code 2, and the next scan is correct
    b, t, d = 2, 300, 256
    pre = synth.preacts(404, b, t, d, torch.bfloat16).cuda()
    monkeypatch.setenv("MMF_SCAN_SKIP_CHUNK", "1")
    monkeypatch.setenv("MMF_WAIT_LIMIT_US", "20000")
    mmf.mlgru_scan(pre, torch.zeros(b, d, device="cuda"))
    with pytest.raises(mmf.MMFError) as err:
        mmf.check()
    assert err.value.status == 6 and "code 2" in str(err.value)
    monkeypatch.delenv("MMF_SCAN_SKIP_CHUNK")
    monkeypatch.delenv("MMF_WAIT_LIMIT_US")
    h = torch.zeros(b, d, device="cuda")
    o = mmf.mlgru_scan(pre, h)
    mmf.check()
    p = to_np(pre)
    o_ref, h_ref = O.mlgru_scan(p[:, :, 0], p[:, :, 1], p[:, :, 2], np.zeros((b, d)))
    assert_close(to_np(o), o_ref, "bf16", "o' after the timeout")
    assert_close(to_np(h), h_ref, "f32", "h_T after the timeout")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("b,t,d", [(3, 200, 264), (8, 300, 2560)])
def test_scan_states_then_backward(b, t, d, dtype):
    # the training forward stores the states: o' equals the plain scan's bit for
    # bit, the states match the oracle's, and the backward given them equals the
    # backward that recomputes them, bit for bit
    pre = synth.preacts(460 + t, b, t, d, TORCH_DT[dtype], scale=2.0).cuda()
    h0 = synth.activations(461, b, d).cuda()
    dout = synth.activations(462, b * t, d, TORCH_DT[dtype]).reshape(b, t, d).cuda()
    h1, h2 = h0.clone(), h0.clone()
    o_plain = mmf.mlgru_scan(pre, h1)
    o, hs = mmf.mlgru_scan_states(pre, h2)
    mmf.check()
    assert torch.equal(o, o_plain) and torch.equal(h1, h2)
    p = to_np(pre)
    og, _ = O.mlgru_scan(p[:, :, 0], p[:, :, 1], p[:, :, 2], to_np(h0))
    h_ref = og / O.sigmoid(p[:, :, 2])
    assert_close(to_np(hs), h_ref, "f32", "states")
    d1, dh1 = mmf.mlgru_scan_backward(pre, h0, dout)
    d2, dh2 = mmf.mlgru_scan_backward(pre, h0, dout, hs=hs)
    _, hs_only = mmf.mlgru_scan_states(pre, h0.clone(), want_o=False)
    mmf.check()
    assert torch.equal(d1, d2) and torch.equal(dh1, dh2) and torch.equal(hs_only, hs)


def test_scan_backward_wait_gives_up_and_reports(monkeypatch):
    # chunk 1 of CTA 0 is never loaded by the backward's TMA ring (the forward
    # states pass runs normally): its bounded wait runs out, the kernel lets its
    # other copies land and returns, mmf_check reports code 2, and the next
    # call is correct
    b, t, d = 2, 300, 256
    pre = synth.preacts(450, b, t, d, torch.bfloat16).cuda()
    dout = synth.activations(451, b * t, d, torch.bfloat16).reshape(b, t, d).cuda()
    h0 = torch.zeros(b, d, device="cuda")
    monkeypatch.setenv("MMF_SCAN_SKIP_CHUNK", "1")
    monkeypatch.setenv("MMF_WAIT_LIMIT_US", "20000")
    mmf.mlgru_scan_backward(pre, h0, dout)
    with pytest.raises(mmf.MMFError) as err:
        mmf.check()
    assert err.value.status == 6 and "code 2" in str(err.value)
    monkeypatch.delenv("MMF_SCAN_SKIP_CHUNK")
    monkeypatch.delenv("MMF_WAIT_LIMIT_US")
    dpre, dh0 = mmf.mlgru_scan_backward(pre, h0, dout)
    mmf.check()
    p = to_np(pre)
    ref = O.mlgru_scan_backward(p[:, :, 0], p[:, :, 1], p[:, :, 2], np.zeros((b, d)), to_np(dout))
    assert_close(to_np(dpre)[:, :, 1], ref[1], "bf16", "dc~ after the timeout")
    assert_close(to_np(dh0), ref[3], "f32", "dh0 after the timeout")


def test_scan_chunked_equals_whole():
    b, t, d = 2, 96, 64
    pre = synth.preacts(403, b, t, d).cuda()
    h1 = torch.zeros(b, d, device="cuda")
    o1 = mmf.mlgru_scan(pre, h1)
    h2 = torch.zeros(b, d, device="cuda")
    oa = mmf.mlgru_scan(pre[:, :40].contiguous(), h2)
    ob = mmf.mlgru_scan(pre[:, 40:].contiguous(), h2)
    torch.testing.assert_close(torch.cat([oa, ob], 1), o1, rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(h2, h1, rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------ GLU

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("m,d,inner", [(128, 256, 768), (4, 2048, 5632), (9, 64, 48)])
def test_glu_parity(m, d, inner, dtype):
    _, gate, og = make_layer(500, inner, d)
    _, up, ou = make_layer(501, inner, d)
    _, down, od = make_layer(502, d, inner)
    x = synth.activations(503, m, d, TORCH_DT[dtype])
    res = synth.activations(504, m, d, TORCH_DT[dtype])
    y = mmf.glu(gate, up, down, x.cuda(), residual=res.cuda())
    blk = O.Block(og, og, og, og, og, ou, od)
    y_ref, parts = O.glu(to_np(x), blk, dtype, parts=True)
    assert_close(to_np(y), to_np(res) + y_ref, dtype, "glu y")


# ------------------------------------------------------------------ blocks

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_decode_steps_parity(dtype):
    d, inner, B, T = 256, 768, 4, 6
    blk, oblk = make_block(7001, d, inner)
    x = synth.activations(7002, B * T, d, TORCH_DT[dtype]).reshape(B, T, d)
    st = mmf.State(1, B, d)
    ys = [mmf.block_forward(blk, 0, st, x[:, t:t + 1].contiguous().cuda()) for t in range(T)]
    y = torch.cat(ys, 1)
    h = np.zeros((B, d))
    yr = []
    for t in range(T):
        yt, h = O.block_forward(to_np(x[:, t:t + 1]), oblk, h, dtype)
        yr.append(yt)
    assert_close(to_np(y), np.concatenate(yr, 1), dtype, "decode y", tol=E2E_TOL)
    assert_close(st.get()[0].numpy(), h, "f32", "decode h", tol=E2E_TOL)


@pytest.mark.parametrize("k,n,m", [(2048, 2048, 1), (2048, 5632, 4), (5632, 2048, 16), (272, 130, 9)])
def test_decode_fused_quant_matches_standalone_quantiser(k, n, m, monkeypatch):
    # the decode contraction quantises its token rows itself with the same fp32
    # steps as the standalone quantiser (the whole block on each row for up to
    # 8 tokens, one warp per row above): the fp64 sum of squares may be added in
    # another order, so codes agree except at rounding ties, and the integer
    # accumulators are exact for the codes each path used
    _, lin, olin = make_layer(900 + k + n, n, k)
    x = synth.activations(901 + m, m, k, torch.bfloat16, outlier_p=synth.GEMV_OUTLIER_P,
                          outlier_scale=synth.GEMV_OUTLIER_SCALE).cuda()
    monkeypatch.setenv("MMF_DECODE_FUSED_QUANT", "1")
    fused = mmf.bitlinear(lin, x, debug=True)
    monkeypatch.setenv("MMF_DECODE_FUSED_QUANT", "0")
    split = mmf.bitlinear(lin, x, debug=True)
    assert_codes_close(fused[1].cpu().numpy(), split[1].cpu().numpy(), "fused vs standalone codes")
    np.testing.assert_allclose(to_np(fused[2]), to_np(split[2]), rtol=2e-7)
    codes = O.unpack_codes(packed_to_np(lin.packed), k)
    for y, q, s, acc in (fused, split):
        np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), O.ternary_accumulate(q.cpu().numpy(), codes))
    assert_close(to_np(fused[0]), to_np(split[0]), "bf16", "fused vs standalone y")
    assert_close(to_np(fused[0]), O.bitlinear(to_np(x.cpu()), olin), "bf16", "fused y vs oracle")


def test_block_decode_fused_quant_matches_standalone_quantiser(monkeypatch):
    monkeypatch.setenv("MMF_DECODE_STEP_KERNEL", "0")   # the separate kernels
    d, inner, B = 256, 768, 4
    blk, _ = make_block(7011, d, inner)
    x = synth.activations(7012, B, d, torch.bfloat16).reshape(B, 1, d).cuda()
    h0 = synth.activations(7013, B, d) * 0.5
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MMF_DECODE_FUSED_QUANT", flag)
        st = mmf.State(1, B, d)
        st.set(h0.reshape(1, B, d))
        outs.append((mmf.block_forward(blk, 0, st, x), st.get()))
    # the same arithmetic; only a code at a rounding tie may differ (fp64 sum order)
    assert_close(to_np(outs[0][0]), to_np(outs[1][0]), "bf16", "fused vs standalone block y")
    assert_close(outs[0][1].numpy(), outs[1][1].numpy(), "f32", "fused vs standalone state")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_prefill_unpacked_copy_is_bit_identical(dtype, monkeypatch):
    # a block keeps one-byte copies of its codes for the prefill contraction
    # (TMA-loaded instead of expanded in shared memory): identical results
    d, inner, B, T = 256, 768, 2, 192
    x = synth.activations(7042, B * T, d, TORCH_DT[dtype]).reshape(B, T, d).cuda()
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MMF_PREFILL_UNPACKED", flag)
        blk, _ = make_block(7041, d, inner)
        st = mmf.State(1, B, d)
        outs.append((mmf.block_forward(blk, 0, st, x), st.get()))
    mmf.check()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_block_byte_copy_made_by_first_prefill_call_only():
    # creating a block and decoding with it allocate no one-byte code copy; the
    # first prefill-sized call makes it (7 matrices, N x K bytes each)
    d, inner, B, T = 1024, 2816, 2, 192
    copy_bytes = 4 * d * d + 3 * d * inner
    x = synth.activations(7044, B * T, d, torch.bfloat16).reshape(B, T, d).cuda()
    blk, _ = make_block(7043, d, inner)
    st = mmf.State(1, B, d)
    ws = torch.empty(mmf.stack_ws_size([blk], B, T), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    mmf.block_forward(blk, 0, st, x[:, :1].contiguous(), ws=ws)   # a decode step
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    mmf.block_forward(blk, 0, st, x, ws=ws)                       # first prefill: makes the copy
    torch.cuda.synchronize()
    free2 = torch.cuda.mem_get_info()[0]
    mmf.block_forward(blk, 0, st, x, ws=ws)                       # second prefill: nothing new
    torch.cuda.synchronize()
    free3 = torch.cuda.mem_get_info()[0]
    mmf.check()
    assert free0 - free1 < copy_bytes // 4, (free0, free1)
    assert free1 - free2 >= copy_bytes, (free1, free2, copy_bytes)
    assert abs(free2 - free3) < copy_bytes // 4, (free2, free3)


def test_block_release_codes_frees_the_copy_and_changes_no_result():
    # release the one-byte copy after a prefill: the memory comes back, a
    # decode step afterwards and the next prefill (which makes the copy again)
    # give bit-identical results to a block that kept its copy
    d, inner, B, T = 1024, 2816, 2, 192
    copy_bytes = 4 * d * d + 3 * d * inner
    x = synth.activations(7046, B * T, d, torch.bfloat16).reshape(B, T, d).cuda()
    blk, _ = make_block(7045, d, inner)
    ref, _ = make_block(7045, d, inner)
    st, st_ref = mmf.State(1, B, d), mmf.State(1, B, d)
    ws = torch.empty(mmf.stack_ws_size([blk], B, T), dtype=torch.uint8, device="cuda")
    y0 = mmf.block_forward(blk, 0, st, x, ws=ws)
    r0 = mmf.block_forward(ref, 0, st_ref, x, ws=ws)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    blk.release_codes()
    free_after = torch.cuda.mem_get_info()[0]
    assert free_after - free_before >= copy_bytes, (free_before, free_after, copy_bytes)
    blk.release_codes()   # nothing left to free: a no-op
    xd = x[:, :1].contiguous()
    y1 = mmf.block_forward(blk, 0, st, xd, ws=ws)
    r1 = mmf.block_forward(ref, 0, st_ref, xd, ws=ws)
    y2 = mmf.block_forward(blk, 0, st, x, ws=ws)    # makes the copy again
    r2 = mmf.block_forward(ref, 0, st_ref, x, ws=ws)
    mmf.check()
    assert torch.cuda.mem_get_info()[0] <= free_after - copy_bytes + copy_bytes // 4
    for a, b in ((y0, r0), (y1, r1), (y2, r2)):
        assert torch.equal(a, b)
    assert torch.equal(st.get(), st_ref.get())


@pytest.mark.parametrize("m", [128, 300])
def test_bitlinear_and_glu_with_byte_codes_bit_identical(m):
    # mmf_tlinear.codes (mmf_unpack_codes) lets the prefill contraction load the
    # codes directly: identical outputs and debug values to the packed path
    k, n = 1024, 768
    _, lin, _ = make_layer(911, n, k)
    lin_u = mmf.unpack_codes(lin)
    codes_ref = O.unpack_codes(packed_to_np(lin.packed), k) + 1
    np.testing.assert_array_equal(lin_u.codes.cpu().numpy().astype(np.int64), codes_ref)
    x = synth.activations(912, m, k, torch.bfloat16).cuda()
    for a, b, what in zip(mmf.bitlinear(lin, x, debug=True), mmf.bitlinear(lin_u, x, debug=True),
                          ("y", "q", "s", "acc")):
        assert torch.equal(a, b), what
    _, gate, _ = make_layer(913, 768, k)
    _, up, _ = make_layer(914, 768, k)
    _, down, _ = make_layer(915, k, 768)
    res = synth.activations(916, m, k, torch.bfloat16).cuda()
    y1 = mmf.glu(gate, up, down, x, residual=res)
    y2 = mmf.glu(mmf.unpack_codes(gate), mmf.unpack_codes(up), mmf.unpack_codes(down), x, residual=res)
    assert torch.equal(y1, y2)


def test_block_prefill_then_decode_matches_oracle_bf16():
    d, inner, B, T = 256, 768, 2, 40
    blk, oblk = make_block(7003, d, inner)
    x = synth.activations(7004, B * (T + 3), d, torch.bfloat16).reshape(B, T + 3, d)
    st = mmf.State(1, B, d)
    y0 = mmf.block_forward(blk, 0, st, x[:, :T].contiguous().cuda())
    y1 = [mmf.block_forward(blk, 0, st, x[:, T + i:T + i + 1].contiguous().cuda()) for i in range(3)]
    y = torch.cat([y0] + y1, 1)
    y_ref, h_ref = O.block_forward(to_np(x[:, :T]), oblk, np.zeros((B, d)), "bf16")
    ys = [y_ref]
    h = h_ref
    for i in range(3):
        yt, h = O.block_forward(to_np(x[:, T + i:T + i + 1]), oblk, h, "bf16")
        ys.append(yt)
    assert_close(to_np(y), np.concatenate(ys, 1), "bf16", "prefill+decode y", tol=E2E_TOL)
    assert_close(st.get()[0].numpy(), h, "f32", "prefill+decode h", tol=E2E_TOL)


def test_stack_forward_matches_block_loop():
    d, inner, B, T, L = 128, 256, 2, 24, 3
    pairs = [make_block(7100, d, inner, layer=l) for l in range(L)]
    blocks = [p[0] for p in pairs]
    x = synth.activations(7101, B * T, d, torch.bfloat16).reshape(B, T, d).cuda()
    st1 = mmf.State(L, B, d)
    y1 = mmf.stack_forward(blocks, st1, x)
    st2 = mmf.State(L, B, d)
    z = x
    for l in range(L):
        z = mmf.block_forward(blocks[l], l, st2, z)
    assert torch.equal(y1, z)
    assert torch.equal(st1.get(), st2.get())
    y_ref, h_ref = O.stack_forward(to_np(x.cpu()), [p[1] for p in pairs], np.zeros((L, B, d)), "bf16")
    assert_close(to_np(y1), y_ref, "bf16", "stack y", tol=E2E_TOL)
    assert_close(st1.get().numpy(), h_ref, "f32", "stack h", tol=E2E_TOL)


def test_graft_entry_smoke():
    # the packaged smoke check: a 2 x 64-token prefill (tensor-core contraction)
    # and one decode step of a d=256 block against the oracle
    import importlib.util
    import pathlib
    path = pathlib.Path(__file__).resolve().parents[1] / "__graft_entry__.py"
    spec = importlib.util.spec_from_file_location("graft_entry", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.smoke()
