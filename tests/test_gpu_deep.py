"""Full-depth slices of the model-shaped stacks against the oracle.

Sequences of a batch are independent and the scan is causal, so one sequence
of a full-batch launch is an exact slice. The GPU runs the whole batch in the
launch configurations the benchmark uses; the oracle checks sequence 0:

  * parity, at TOL: the layers and decode steps listed below are checked
    stage by stage, teacher-forced on the GPU's own inputs and state at that
    layer and step (tests/parity.py: check_block_stages), through the whole
    depth of the stack and the whole decode loop;
  * drift, reported: the oracle also runs sequence 0 on its own (its own
    outputs feed the next layer and the next step), and max|gpu - oracle| /
    max|oracle| and ||gpu - oracle|| / ||oracle|| are recorded per layer and per
    step (written as JSON under $MMF_DRIFT_OUT when set). The block amplifies
    any rounding difference: a change of one unit in the last place of one
    input element of the 370M stack moves the oracle's own output by several
    percent after 24 layers, and a decode loop that feeds its output back is
    chaotic, so free-running drift is a measurement, not a pass/fail criterion.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import check_block_stages, make_block, normwise, record_drift, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")


def _rms(gpu, ref) -> float:
    g, r = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    n = float(np.linalg.norm(r))
    return float(np.linalg.norm(g - r) / n) if n > 0 else 0.0


def _prompt(wl, B, T):
    """[B, T, d] bf16 prompt whose sequence 0 does not depend on B."""
    x0 = synth.activations(wl.seed + synth.ACT_SEED_OFFSET, T, wl.d, torch.bfloat16)
    rest = synth.activations(wl.seed + synth.ACT_SEED_OFFSET + 1, (B - 1) * T, wl.d, torch.bfloat16)
    return torch.cat([x0, rest]).reshape(B, T, wl.d)


def _gpu_by_layer(blocks, obl, st, x, check_layers, what):
    """Run the blocks one at a time over x (whole batch, prefill or one decode step); layers in
    check_layers are teacher-forced stage by stage on sequence 0. Returns sequence 0's output after
    every layer, and the batch's final output."""
    cur = x.cuda()
    B, T, d = x.shape
    ws = torch.empty(mmf.stack_ws_size(blocks, B, T), dtype=torch.uint8, device="cuda")
    outs = []
    for l, blk in enumerate(blocks):
        if l in check_layers:
            h_prev = st.get()[l].numpy().astype(np.float64)
            y, dbg = mmf.block_forward_debug(blk, l, st, cur, ws=ws)
            check_block_stages(cur.cpu(), h_prev, y, st.get()[l].numpy(), dbg, obl[l], "bf16",
                               f"{what} layer {l}", seqs=slice(0, 1))
            del dbg
        else:
            y = mmf.block_forward(blk, l, st, cur, ws=ws)
        outs.append(to_np(y[0:1]))
        cur = y
    mmf.check()
    return outs, cur


def _oracle_prefill(x0, obl, d):
    """Sequence 0 through every layer from zero state, on its own: (outputs per layer, states)."""
    ys, hs = [], []
    cur = to_np(x0)
    for ob in obl:
        cur, h = O.block_forward(cur, ob, np.zeros((1, d)), "bf16")
        ys.append(cur)
        hs.append(h)
    return ys, hs


def _drift(gpu_ys, gpu_h, ref_ys, ref_hs):
    return [{"layer": l, "y_max": normwise(g, r), "y_rms": _rms(g, r), "h_max": normwise(gh, rh),
             "h_rms": _rms(gh, rh)}
            for l, (g, r, gh, rh) in enumerate(zip(gpu_ys, ref_ys, gpu_h, ref_hs))]


def test_370m_stack_sequence0_all_24_layers():
    # every layer teacher-forced at TOL; free-running drift reported next to the
    # oracle's own drift when one input element moves by one bf16 ulp
    wl = synth.STACK_370M
    B, T, d, I, L = wl.batch, wl.seq, wl.d, wl.inner, wl.layers
    pairs = [make_block(wl.seed, d, I, layer=l, cache=True) for l in range(L)]
    blocks, obl = [p[0] for p in pairs], [p[1] for p in pairs]
    x = _prompt(wl, B, T)
    st = mmf.State(L, B, d)
    gpu_ys, _ = _gpu_by_layer(blocks, obl, st, x, range(L), "370M prefill")
    gpu_h = st.get()[:, 0:1].numpy()
    ref_ys, ref_hs = _oracle_prefill(x[0:1], obl, d)
    # the oracle against itself with one element of its input one unit in the last place away
    xp = to_np(x[0:1]).copy()
    k = (T // 2, d // 3)
    xp[0, k[0], k[1]] += 2.0 ** (np.floor(np.log2(abs(xp[0, k[0], k[1]]))) - 7)
    per_ys, per_hs = _oracle_prefill(torch.tensor(xp), obl, d)
    record_drift("stack370m_seq0_prefill", {
        "gpu_vs_oracle": _drift(gpu_ys, gpu_h, ref_ys, ref_hs),
        "oracle_one_ulp_input_change": _drift(per_ys, per_hs, ref_ys, ref_hs)})


def test_1p3b_row0_prefill_2048_then_256_decode_steps():
    # prefill: every 4th layer and the last teacher-forced; decode: 256 steps,
    # output fed back, every layer teacher-forced at steps 0-3 and every 32nd
    wl = synth.STACK_1P3B
    B, T, d, I, L, steps = wl.batch, wl.seq, wl.d, wl.inner, wl.layers, wl.decode_steps
    pairs = [make_block(wl.seed, d, I, layer=l, cache=True) for l in range(L)]
    blocks, obl = [p[0] for p in pairs], [p[1] for p in pairs]
    x = _prompt(wl, B, T)
    st = mmf.State(L, B, d)
    gpu_ys, y_last = _gpu_by_layer(blocks, obl, st, x, set(range(0, L, 4)) | {L - 1}, "1.3B prefill")
    gpu_h = st.get()[:, 0:1].numpy()
    cur = y_last[:, -1:].contiguous()
    ws = torch.empty(mmf.stack_ws_size(blocks, B, 1), dtype=torch.uint8, device="cuda")
    gpu_dec = []
    checked = [t for t in range(steps) if t < 4 or t % 32 == 31]
    for t in range(steps):
        if t in checked:
            _, cur = _gpu_by_layer(blocks, obl, st, cur.cpu(), range(L), f"1.3B decode step {t}")
        else:
            cur = mmf.stack_forward(blocks, st, cur, ws=ws)
        gpu_dec.append(to_np(cur[0:1]))
    mmf.check()
    # free-running oracle: its own prefill of row 0, then its own decode loop (first 32 steps)
    ref_ys, ref_hs = _oracle_prefill(x[0:1], obl, d)
    h = list(ref_hs)
    xr = ref_ys[-1][:, -1:]
    drift_dec = []
    for t in range(32):
        for l, ob in enumerate(obl):
            xr, h[l] = O.block_forward(xr, ob, h[l], "bf16")
        drift_dec.append({"step": t, "y_max": normwise(gpu_dec[t], xr), "y_rms": _rms(gpu_dec[t], xr)})
    record_drift("stack1p3b_row0", {"teacher_forced_decode_steps": checked,
                                    "prefill_by_layer": _drift(gpu_ys, gpu_h, ref_ys, ref_hs),
                                    "decode_by_step": drift_dec})


DECODE_STEPS_2P7B = 8


def test_2p7b_sequence0_prompt_then_decode_at_1_8_64():
    # each batch size: prompt prefill (one stack launch sequence), then 8 decode
    # steps with every layer teacher-forced at every step; B = 1 also checks
    # three layers of the prefill stage by stage
    wl = synth.STACK_2P7B
    T, d, I, L = wl.seq, wl.d, wl.inner, wl.layers
    pairs = [make_block(wl.seed, d, I, layer=l, cache=True) for l in range(L)]
    blocks, obl = [p[0] for p in pairs], [p[1] for p in pairs]
    x1 = _prompt(wl, 1, T)
    ref_ys, ref_hs = _oracle_prefill(x1, obl, d)
    report = {}
    for B in synth.STACK_2P7B_BATCHES:
        x = _prompt(wl, B, T)
        st = mmf.State(L, B, d)
        if B == 1:
            gpu_ys, y = _gpu_by_layer(blocks, obl, st, x, (0, L // 2, L - 1), "2.7B prefill B=1")
            pre_y = gpu_ys[-1]
        else:
            ws = torch.empty(mmf.stack_ws_size(blocks, B, T), dtype=torch.uint8, device="cuda")
            y = mmf.stack_forward(blocks, st, x.cuda(), ws=ws)
            pre_y = to_np(y[0:1])
            del ws
        pre_h = st.get()[:, 0:1].numpy()
        cur = y[:, -1:].contiguous()
        for t in range(DECODE_STEPS_2P7B):
            _, cur = _gpu_by_layer(blocks, obl, st, cur.cpu(), range(L), f"2.7B decode B={B} step {t}")
        report[f"B={B}"] = {"prefill_y_max": normwise(pre_y, ref_ys[-1]), "prefill_y_rms": _rms(pre_y, ref_ys[-1]),
                            "prefill_h_max": max(normwise(pre_h[l], ref_hs[l]) for l in range(L))}
        del st, y, cur
        torch.cuda.empty_cache()
    record_drift("stack2p7b_seq0", report)
