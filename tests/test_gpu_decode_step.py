"""The one-launch decode step (decode_step.cu) through the C ABI.

A decode step of up to 8 sequences runs as one cooperative launch over all the
layers of the call. Its stages are checked teacher-forced against the oracle in
test_gpu_stages.py (block calls) and end to end in test_gpu_deep.py (stacks).
Here: agreement with the four-contraction path over several steps and layers,
launches of more than 32 layers, a state used with both dtypes, block and stack
calls interleaved on one state, and failure detection: a bounded wait that runs
out (one CTA made to skip publishing) returns, is reported by mmf_check, and
after mmf_state_reset the next step is correct again. No GPU fault is involved.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import E2E_TOL, TOL, TORCH_DT, assert_close, make_block, to_np

pytestmark = pytest.mark.gpu

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")


def _steps(blocks, B, d, x, steps, monkeypatch, one_launch: bool, h0=None):
    monkeypatch.setenv("MMF_DECODE_STEP_KERNEL", "1" if one_launch else "0")
    L = len(blocks)
    st = mmf.State(L, B, d)
    if h0 is not None:
        st.set(h0)
    ys = []
    cur = x
    for _ in range(steps):
        cur = mmf.stack_forward(blocks, st, cur)
        ys.append(cur)
    mmf.check()
    return torch.stack(ys), st.get()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 3, 8])
def test_decode_step_matches_four_contraction_path(B, dtype, monkeypatch):
    # 3 layers x 4 steps, output fed back; the two paths take the same fp32
    # steps, so they agree to rounding (a code can differ only at a tie of the
    # fp64 sum order); and both against the oracle's own loop at E2E_TOL
    d, inner, L, steps = 320, 2432, 3, 4
    pairs = [make_block(9000 + B, d, inner, layer=l) for l in range(L)]
    blocks = [p[0] for p in pairs]
    x = synth.activations(9001 + B, B, d, TORCH_DT[dtype]).reshape(B, 1, d)
    h0 = (synth.activations(9002 + B, L * B, d) * 0.5).reshape(L, B, d)
    y1, h1 = _steps(blocks, B, d, x.cuda(), steps, monkeypatch, True, h0)
    y0, h0_ = _steps(blocks, B, d, x.cuda(), steps, monkeypatch, False, h0)
    assert_close(to_np(y1), to_np(y0), dtype, "one launch vs four contractions", tol=TOL)
    assert_close(h1.numpy(), h0_.numpy(), "f32", "state", tol=TOL)
    h = [h0[l].numpy().astype(np.float64) for l in range(L)]
    xr = to_np(x)
    ref = []
    for _ in range(steps):
        for l in range(L):
            xr, h[l] = O.block_forward(xr, pairs[l][1], h[l], dtype)
        ref.append(xr)
    assert_close(to_np(y1), np.stack(ref), dtype, "decode loop vs oracle", tol=E2E_TOL)


def test_decode_step_more_than_32_layers(monkeypatch):
    # 34 layers: two launches chained through the workspace
    d, inner, B, L = 256, 768, 2, 34
    blocks = [make_block(9100, d, inner, layer=l)[0] for l in range(L)]
    x = synth.activations(9101, B, d, torch.bfloat16).reshape(B, 1, d).cuda()
    y1, h1 = _steps(blocks, B, d, x, 2, monkeypatch, True)
    y0, h0 = _steps(blocks, B, d, x, 2, monkeypatch, False)
    assert_close(to_np(y1), to_np(y0), "bf16", "34 layers", tol=TOL)
    assert_close(h1.numpy(), h0.numpy(), "f32", "34 layers state", tol=TOL)


def test_decode_step_state_switches_dtype_and_mixes_block_and_stack_calls(monkeypatch):
    monkeypatch.setenv("MMF_DECODE_STEP_KERNEL", "1")
    d, inner, B, L = 256, 768, 4, 2
    pairs = [make_block(9200, d, inner, layer=l) for l in range(L)]
    blocks = [p[0] for p in pairs]
    st = mmf.State(L, B, d)
    h = [np.zeros((B, d)) for _ in range(L)]
    for i, dtype in enumerate(["bf16", "f32", "f32", "bf16"]):
        x = synth.activations(9201 + i, B, d, TORCH_DT[dtype]).reshape(B, 1, d)
        if i % 2 == 0:
            y = mmf.stack_forward(blocks, st, x.cuda())
        else:
            y = mmf.block_forward(blocks[1], 1, st, mmf.block_forward(blocks[0], 0, st, x.cuda()))
        mmf.check()
        xr = to_np(x)
        for l in range(L):
            xr, h[l] = O.block_forward(xr, pairs[l][1], h[l], dtype)
        assert_close(to_np(y), xr, dtype, f"call {i} ({dtype})", tol=E2E_TOL)
    assert_close(st.get().numpy(), np.stack(h), "f32", "state", tol=E2E_TOL)


def test_decode_step_wait_gives_up_and_reports(monkeypatch):
    # CTA 3 never publishes its first stage: every other CTA's wait for those
    # rows runs out after 20 ms (bounded), the launch returns, mmf_check
    # reports code 5; after a state reset the next step matches the oracle
    monkeypatch.setenv("MMF_DECODE_STEP_KERNEL", "1")
    d, inner, B = 256, 768, 2
    blk, oblk = make_block(9300, d, inner)
    x = synth.activations(9301, B, d, torch.bfloat16).reshape(B, 1, d).cuda()
    st = mmf.State(1, B, d)
    monkeypatch.setenv("MMF_DECODE_SKIP_CTA", "3")
    monkeypatch.setenv("MMF_WAIT_LIMIT_US", "20000")
    mmf.block_forward(blk, 0, st, x)
    with pytest.raises(mmf.MMFError) as err:
        mmf.check()
    assert err.value.status == 6 and "code 5" in str(err.value)
    monkeypatch.delenv("MMF_DECODE_SKIP_CTA")
    monkeypatch.delenv("MMF_WAIT_LIMIT_US")
    st.reset()
    y = mmf.block_forward(blk, 0, st, x)
    mmf.check()
    y_ref, h_ref = O.block_forward(to_np(x.cpu()), oblk, np.zeros((B, d)), "bf16")
    assert_close(to_np(y), y_ref, "bf16", "after reset", tol=E2E_TOL)
    assert_close(st.get()[0].numpy(), h_ref, "f32", "state after reset", tol=E2E_TOL)
