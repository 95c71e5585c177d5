"""Full-size workloads, in the launch configurations bench.py times, on sampled outputs.

Token rows of a BitLinear are independent, channels of the scan are
independent, and sequences of a block are independent, so the oracle checks
sampled rows / channels / sequences of full-size launches exactly.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import assert_close, assert_codes_close, check_block_stages, make_block, packed_to_np, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")

W370 = synth.STACK_370M


def _rows(seed, n, k):
    return np.sort(np.random.default_rng(seed).choice(n, size=k, replace=False))


@pytest.mark.parametrize("proj,n,k", [("fcg", 3 * W370.d, W370.d), ("gate", W370.inner, W370.d),
                                      ("down", W370.d, W370.inner)])
def test_370m_bitlinear_full_m_sampled_rows(proj, n, k):
    M = W370.batch * W370.seq                      # 16384 tokens: the tcgen05 path
    W = synth.latent_weight(5000 + n, n, k)
    lin = mmf.quantize_weights(W.cuda())
    olin = O.make_tlinear(W.numpy())
    x = synth.activations(5001, M, k, torch.bfloat16)
    y, q, s, acc = mmf.bitlinear(lin, x.cuda(), debug=True)
    rows = _rows(5002, M, 48)
    xr = to_np(x[rows])
    y_ref, parts = O.bitlinear(xr, olin, parts=True)
    assert_codes_close(q[rows].cpu().numpy(), parts["q"], "codes")
    codes = O.unpack_codes(packed_to_np(lin.packed), k)
    np.testing.assert_array_equal(acc[rows].cpu().numpy().astype(np.int64),
                                  O.ternary_accumulate(q[rows].cpu().numpy(), codes))
    assert_close(to_np(y[rows]), y_ref, "bf16", f"{proj} y")


def test_370m_scan_full_size_sampled_channels():
    B, T, d = W370.batch, W370.seq, W370.d
    pre = synth.preacts(5010, B, T, d, torch.bfloat16, scale=2.0)
    h0 = synth.activations(5011, B, d)
    h = h0.cuda().clone()
    o = mmf.mlgru_scan(pre.cuda(), h)
    ch = _rows(5012, d, 24)
    p = to_np(pre[:, :, :, ch])
    o_ref, h_ref = O.mlgru_scan(p[:, :, 0], p[:, :, 1], p[:, :, 2], h0.numpy()[:, ch].astype(np.float64))
    assert_close(to_np(o[:, :, ch]), o_ref, "bf16", "o' sampled channels")
    assert_close(h[:, ch].cpu().numpy(), h_ref, "f32", "h_T sampled channels")


def test_370m_block_full_batch_sampled_sequence():
    B, T, d, I = W370.batch, W370.seq, W370.d, W370.inner
    blk, oblk = make_block(W370.seed, d, I, layer=0)
    x = synth.activations(W370.seed + synth.ACT_SEED_OFFSET, B * T, d, torch.bfloat16).reshape(B, T, d)
    st = mmf.State(1, B, d)
    y, dbg = mmf.block_forward_debug(blk, 0, st, x.cuda())   # M = 16384: the configuration bench.py times
    mmf.check()
    # one full sequence, every token, stage by stage at TOL
    check_block_stages(x, np.zeros((B, d)), y, st.get()[0].numpy(), dbg, oblk, "bf16", "370M block",
                       seqs=slice(5, 6))


@pytest.mark.parametrize("wl,batch", [(synth.STACK_1P3B, 4), (synth.STACK_2P7B, 1), (synth.STACK_2P7B, 8),
                                      (synth.STACK_2P7B, 64)])
def test_decode_step_full_width(wl, batch):
    d, I = wl.d, wl.inner
    blk, oblk = make_block(wl.seed, d, I, layer=0)
    x = synth.activations(wl.seed + 7, batch, d, torch.bfloat16).reshape(batch, 1, d)
    h0 = synth.activations(wl.seed + 8, batch, d) * 0.5
    st = mmf.State(1, batch, d)
    st.set(h0.reshape(1, batch, d))
    y, dbg = mmf.block_forward_debug(blk, 0, st, x.cuda())
    mmf.check()
    check_block_stages(x, h0.numpy().astype(np.float64), y, st.get()[0].numpy(), dbg, oblk, "bf16",
                       f"decode {wl.name} B={batch}")
