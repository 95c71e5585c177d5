"""Teacher-forced per-stage parity inside mmf_block_forward, at the 2e-3 tolerance.

mmf_block_forward_debug hands out every tensor the block stores between its
stages (pre-activations, o', y1, p) and the int8 codes and scales of its four
quantised inputs. Each oracle stage is fed the GPU's own input to that stage,
so every stage is checked on its own at TOL: f|c|g, the gates and scan (or the
decode step's recurrence), o + residual, gate|up with the SiLU gate, down +
residual; the codes within 1 LSB on <= 0.01% of elements and the scales to
fp32 rounding.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import E2E_TOL, TORCH_DT, assert_close, check_block_stages, check_block_tie_forced, make_block, to_np

pytestmark = pytest.mark.gpu

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")


def _run(blk, x, h0, dtype):
    B, T, d = x.shape
    st = mmf.State(1, B, d)
    st.set(torch.tensor(h0, dtype=torch.float32).reshape(1, B, d))
    y, dbg = mmf.block_forward_debug(blk, 0, st, x.cuda())
    mmf.check()
    return y, st.get()[0].numpy(), dbg


def test_tiny_block_fp32_stages_and_end_to_end():
    # the tiny single block, fp32 end to end, h0 = 0: every stage at TOL; the
    # whole block at TOL with only the rounding-tie codes taken from the GPU;
    # and the block without any forcing at the composite tolerance (a code on
    # the other side of a tie moves outputs by about 1/|acc| each)
    w = synth.TINY_BLOCK
    blk, oblk = make_block(w.seed, w.d, w.inner)
    x = synth.activations(w.seed + synth.ACT_SEED_OFFSET, w.batch * w.seq, w.d).reshape(w.batch, w.seq, w.d)
    h0 = np.zeros((w.batch, w.d))
    y, hT, dbg = _run(blk, x, h0, "f32")
    check_block_stages(x, h0, y, hT, dbg, oblk, "f32", "tiny block")
    check_block_tie_forced(x, h0, y, hT, dbg, oblk, "f32", "tiny block")
    y_ref, h_ref = O.block_forward(x.numpy(), oblk, h0, "f32")
    assert_close(to_np(y), y_ref, "f32", "tiny block y (no forcing)", tol=E2E_TOL)
    assert_close(hT, h_ref, "f32", "tiny block h_T (no forcing)", tol=E2E_TOL)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,T", [(3, 100), (2, 64), (1, 5)])
def test_block_prefill_stages(B, T, dtype):
    # M = 300 and 128 take the tensor-core contraction, M = 5 the warp-MMA kernel
    d, inner = 256, 768
    blk, oblk = make_block(8100 + T, d, inner)
    x = synth.activations(8101 + T, B * T, d, TORCH_DT[dtype]).reshape(B, T, d)
    h0 = synth.activations(8102, B, d).numpy().astype(np.float64) * 0.5
    y, hT, dbg = _run(blk, x, h0, dtype)
    check_block_stages(x, h0, y, hT, dbg, oblk, dtype, f"prefill B={B} T={T}")
    check_block_tie_forced(x, h0, y, hT, dbg, oblk, dtype, f"prefill B={B} T={T}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 4, 8, 13])
def test_block_decode_step_stages(B, dtype):
    # one decode step (T = 1): the f|c|g contraction with the recurrence step in
    # its epilogue, teacher-forced on the stored pre-activations and h_{t-1}
    d, inner = 256, 768
    blk, oblk = make_block(8200 + B, d, inner)
    x = synth.activations(8201 + B, B, d, TORCH_DT[dtype]).reshape(B, 1, d)
    h0 = synth.activations(8202 + B, B, d).numpy().astype(np.float64) * 0.5
    y, hT, dbg = _run(blk, x, h0, dtype)
    check_block_stages(x, h0, y, hT, dbg, oblk, dtype, f"decode B={B}")
    check_block_tie_forced(x, h0, y, hT, dbg, oblk, dtype, f"decode B={B}")


def test_block_decode_steps_teacher_forced_each_step():
    # six decode steps in a row, each step checked stage by stage from the
    # GPU's own state and input
    d, inner, B, T = 256, 768, 4, 6
    blk, oblk = make_block(8300, d, inner)
    x = synth.activations(8301, B * T, d, torch.bfloat16).reshape(B, T, d)
    st = mmf.State(1, B, d)
    for t in range(T):
        h_prev = st.get()[0].numpy().astype(np.float64)
        xt = x[:, t:t + 1].contiguous()
        y, dbg = mmf.block_forward_debug(blk, 0, st, xt.cuda())
        check_block_stages(xt, h_prev, y, st.get()[0].numpy(), dbg, oblk, "bf16", f"step {t}")


def test_block_stages_with_gains_and_biases():
    # non-unit RMSNorm gains (f|c|g share one, gate|up share one) and biases on
    # every projection, prefill and decode
    d, inner, B = 256, 768, 3
    shapes = {"f": (d, d), "c": (d, d), "g": (d, d), "o": (d, d), "gate": (inner, d), "up": (inner, d),
              "down": (d, inner)}
    gain_of = {"f": 0, "c": 0, "g": 0, "o": 1, "gate": 2, "up": 2, "down": 3}
    # gain vectors by input: x (f, c, g share it), o', y1 (gate, up share it), p
    gains = [(1.0 + 0.2 * synth.activations(8401 + i, 1, d if i < 3 else inner)[0]) for i in range(4)]
    gains_dev = [g.cuda() for g in gains]   # one device tensor per shared gain
    lins, olins = {}, {}
    for i, name in enumerate(synth.PROJ_NAMES):
        W = synth.latent_weight(synth.sub_seed(8402, 0, i), *shapes[name])
        bias = 0.05 * synth.activations(8403 + i, 1, shapes[name][0])[0]
        j = gain_of[name]
        lins[name] = mmf.quantize_weights(W.cuda(), gain=gains_dev[j], bias=bias.cuda())
        olins[name] = O.make_tlinear(W.numpy(), gain=gains[j].numpy(), bias=bias.numpy())
    blk, oblk = mmf.Block(lins), O.Block(**olins)
    for T in (64, 1):
        x = synth.activations(8410 + T, B * T, d, torch.bfloat16).reshape(B, T, d)
        h0 = synth.activations(8411, B, d).numpy().astype(np.float64) * 0.5
        y, hT, dbg = _run(blk, x, h0, "bf16")
        check_block_stages(x, h0, y, hT, dbg, oblk, "bf16", f"gains and biases T={T}")
        check_block_tie_forced(x, h0, y, hT, dbg, oblk, "bf16", f"gains and biases T={T}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,T", [(3, 100), (1, 5), (4, 1), (9, 1)])
def test_block_gnorm_stages(B, T, dtype):
    # the g_norm output gate (seeded non-unit gain): prefill on the tensor-core
    # (M = 300) and warp-MMA (M = 5) contractions, and decode steps, which run
    # the prefill sequence with T = 1; every stage teacher-forced at TOL
    d, inner = 256, 768
    blk, oblk = make_block(8500 + T + B, d, inner, gnorm=True)
    x = synth.activations(8501 + T, B * T, d, TORCH_DT[dtype]).reshape(B, T, d)
    h0 = synth.activations(8502, B, d).numpy().astype(np.float64) * 0.5
    y, hT, dbg = _run(blk, x, h0, dtype)
    check_block_stages(x, h0, y, hT, dbg, oblk, dtype, f"g_norm B={B} T={T}")
    check_block_tie_forced(x, h0, y, hT, dbg, oblk, dtype, f"g_norm B={B} T={T}")
    # the o projection's codes come from the row kernel that forms o': the
    # standalone quantiser on the same stored o' gives the same codes and scales
    _, q, sc, _ = mmf.bitlinear(blk.lins["o"], dbg["og"].reshape(B * T, d), debug=True)
    assert torch.equal(q, dbg["q"][1]) and torch.equal(sc, dbg["s"][1])


def test_block_gnorm_prefill_then_decode():
    # a g_norm block: a 40-token prompt, then 8 decode steps from the GPU's
    # state, each step teacher-forced; the whole run against the oracle's
    # block at the composite tolerance
    d, inner, B, T, S = 256, 768, 2, 40, 8
    blk, oblk = make_block(8600, d, inner, gnorm=True)
    x = synth.activations(8601, B * (T + S), d, torch.bfloat16).reshape(B, T + S, d)
    st = mmf.State(1, B, d)
    ys = [mmf.block_forward(blk, 0, st, x[:, :T].contiguous().cuda())]
    for t in range(T, T + S):
        h_prev = st.get()[0].numpy().astype(np.float64)
        xt = x[:, t:t + 1].contiguous()
        y, dbg = mmf.block_forward_debug(blk, 0, st, xt.cuda())
        check_block_stages(xt, h_prev, y, st.get()[0].numpy(), dbg, oblk, "bf16", f"g_norm step {t}")
        ys.append(y)
    mmf.check()
    y_ref, h_ref = O.block_forward(x.float().numpy(), oblk, np.zeros((B, d)), "bf16")
    assert_close(to_np(torch.cat(ys, 1)), y_ref, "bf16", "g_norm prompt + decode y", tol=E2E_TOL)
    assert_close(st.get()[0].numpy(), h_ref, "f32", "g_norm prompt + decode h_T", tol=E2E_TOL)


@pytest.mark.parametrize("gnorm", [False, True])
def test_checkpoint_resume_matches_one_prefill(gnorm):
    # prefill half a prompt, save the state to the host, restore it into a
    # fresh state handle and prefill the rest: the second half's output and
    # the final state equal those of one prefill over the whole prompt
    # (recurrent state and outputs are exact; save/restore is a bit copy)
    d, inner, B, T, L = 256, 768, 2, 256, 2
    pairs = [make_block(8700 + l, d, inner, layer=l, gnorm=gnorm) for l in range(L)]
    blocks = [p_[0] for p_ in pairs]
    x = synth.activations(8710, B * T, d, torch.bfloat16).reshape(B, T, d).cuda()
    st = mmf.State(L, B, d)
    y_all = mmf.stack_forward(blocks, st, x)
    h_all = st.get()
    st1 = mmf.State(L, B, d)
    mmf.stack_forward(blocks, st1, x[:, :T // 2].contiguous())
    saved = st1.get()
    st2 = mmf.State(L, B, d)
    st2.set(saved)
    assert torch.equal(st2.get(), saved)   # the round trip is a bit copy
    y2 = mmf.stack_forward(blocks, st2, x[:, T // 2:].contiguous())
    mmf.check()
    # the scan composes its chunks' maps in a different grouping when the
    # sequence is cut, so the state may differ by fp32 rounding; the stored
    # outputs then agree up to the storage rounding that carries into codes
    torch.testing.assert_close(st2.get(), h_all, rtol=1e-5, atol=1e-6)
    assert_close(to_np(y2), to_np(y_all[:, T // 2:]), "bf16", "resumed prefill", tol=E2E_TOL)


@pytest.mark.parametrize("gnorm", [False, True])
@pytest.mark.parametrize("T", [150, 1])
def test_block_stages_ragged_widths(T, gnorm):
    # d = 272 and I = 400 are multiples of 16 but not of 64: the tensor-core
    # contraction does not take them (prefill runs the mma.sync kernel at 300
    # tokens) and the one-launch decode step does not either (decode runs the
    # four contractions); every stage teacher-forced at TOL
    d, inner, B = 272, 400, 2
    blk, oblk = make_block(8800 + T, d, inner, gnorm=gnorm)
    x = synth.activations(8801 + T, B * T, d, torch.bfloat16).reshape(B, T, d)
    h0 = synth.activations(8802, B, d).numpy().astype(np.float64) * 0.5
    y, hT, dbg = _run(blk, x, h0, "bf16")
    check_block_stages(x, h0, y, hT, dbg, oblk, "bf16", f"ragged widths T={T}")
    check_block_tie_forced(x, h0, y, hT, dbg, oblk, "bf16", f"ragged widths T={T}")


def test_block_decode_step_stages_wide_batch():
    # 40 sequences: above the one-launch decode step's batch, and the GLU's
    # gate|up (I = 6912: 54 tiles) takes the tcgen05 kernel at 40 tokens while
    # the other projections stay on mma.sync; every stage teacher-forced
    d, inner, B = 256, 6912, 40
    blk, oblk = make_block(8900, d, inner)
    x = synth.activations(8901, B, d, torch.bfloat16).reshape(B, 1, d)
    h0 = synth.activations(8902, B, d).numpy().astype(np.float64) * 0.5
    y, hT, dbg = _run(blk, x, h0, "bf16")
    check_block_stages(x, h0, y, hT, dbg, oblk, "bf16", "decode B=40")
    check_block_tie_forced(x, h0, y, hT, dbg, oblk, "bf16", "decode B=40")
