"""Model ends on the GPU: embedding lookup, LM head, greedy next token, greedy generation.

The lookup is a row copy and is compared bit for bit; the argmax is compared
exactly against the oracle's argmax of the same stored logits (the decision is
taken on the stored values on both sides); the head's logits at the BitLinear
tolerance; a whole generation teacher-forced on the GPU's own tokens.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import E2E_TOL, TORCH_DT, assert_close, make_block, make_layer, to_np

pytestmark = pytest.mark.gpu

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("V,d,M", [(32000, 2048, 5), (32000, 1024, 300), (7, 16, 40), (1, 64, 3)])
def test_embed_bit_exact(V, d, M, dtype):
    table = synth.activations(900 + V, V, d, TORCH_DT[dtype]).cuda()
    g = torch.Generator().manual_seed(901)
    ids = torch.randint(0, V, (M,), generator=g, dtype=torch.int32)
    ids[0] = 0
    ids[-1] = V - 1
    x = mmf.embed(table, ids.cuda())
    mmf.check()
    ref = O.embed(ids.numpy(), to_np(table), dtype)
    np.testing.assert_array_equal(to_np(x), ref)


def test_embed_rejects_out_of_range_ids_without_reading_outside():
    V, d = 50, 32
    table = synth.activations(902, V, d).cuda()
    ids = torch.tensor([3, -1, 50, 49], dtype=torch.int32).cuda()
    x = mmf.embed(table, ids)
    with pytest.raises(mmf.MMFError) as err:
        mmf.check()
    assert err.value.status == 1
    xn = to_np(x)
    np.testing.assert_array_equal(xn[[0, 3]], to_np(table)[[3, 49]])
    assert np.all(xn[[1, 2]] == 0.0)
    mmf.check()   # the status word was cleared


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,V", [(1, 32000), (8, 32000), (64, 32000), (3, 37), (5, 1), (2, 100003)])
def test_argmax_exact(M, V, dtype):
    # bf16 logits of N(0,1) have many exact ties among the largest values; a
    # planted tie of the row maximum at two positions checks the lowest index
    logits = synth.activations(903 + V, M, V, TORCH_DT[dtype])
    if V > 10:
        logits[0, V // 2] = 9.0
        logits[0, V // 3] = 9.0
    lg = logits.cuda()
    ids = mmf.argmax(lg)
    mmf.check()
    ref = O.greedy_token(to_np(logits))
    np.testing.assert_array_equal(ids.cpu().numpy(), ref)
    if V > 10:
        assert int(ids[0]) == V // 3


def test_argmax_unaligned_rows_take_the_scalar_path():
    # a row view starting at an odd element: not 16-byte aligned
    base = synth.activations(904, 1, 4001, torch.bfloat16).cuda()
    view = base[0, 1:]
    lg = view.reshape(1, 4000).contiguous()
    np.testing.assert_array_equal(mmf.argmax(lg).cpu().numpy(), O.greedy_token(to_np(lg)))
    lg2 = torch.empty(4001, dtype=torch.bfloat16, device="cuda")[1:].reshape(1, 4000)
    lg2.copy_(lg)
    assert lg2.data_ptr() % 16 != 0
    np.testing.assert_array_equal(mmf.argmax(lg2).cpu().numpy(), O.greedy_token(to_np(lg)))


@pytest.mark.parametrize("M", [1, 4, 16, 64, 300])
def test_lm_head_logits(M):
    # the head of the 2.7B shape: BitLinear 2560 -> 32000 (M = 64 and 300: the
    # tcgen05 kernel, the others the mma.sync kernel)
    _, lin, olin = make_layer(905, 32000, 2560)
    x = synth.activations(906 + M, M, 2560, torch.bfloat16)
    y = mmf.bitlinear(lin, x.cuda())
    mmf.check()
    assert_close(to_np(y), O.lm_logits(to_np(x), olin, "bf16"), "bf16", f"logits M={M}")


def test_greedy_generation_teacher_forced():
    # a 2-block model (d = 256, I = 768, V = 1000): GPU prompt prefill and 8
    # greedy steps; each GPU token is the argmax of the GPU's own logits, and
    # the logits of every step match the oracle's model fed the same tokens
    d, inner, V, B, T0, n = 256, 768, 1000, 2, 12, 8
    pairs = [make_block(960, d, inner, layer=l) for l in range(2)]
    blocks, oblocks = [p[0] for p in pairs], [p[1] for p in pairs]
    _, head, ohead = make_layer(961, V, d)
    table = synth.activations(962, V, d, torch.bfloat16)
    model = mmf.Model(table.cuda(), blocks, head)
    prompt = torch.randint(0, V, (B, T0), generator=torch.Generator().manual_seed(963), dtype=torch.int32)
    st = mmf.State(2, B, d)
    logits = [model.forward(st, prompt.cuda())]
    toks = []
    for _ in range(n):
        t = mmf.argmax(logits[-1])
        toks.append(t)
        logits.append(model.forward(st, t.reshape(B, 1)))
    mmf.check()
    tab = to_np(table)
    h = np.zeros((2, B, d))
    seq = prompt.numpy()
    for k in range(n + 1):
        ref, h = O.model_forward(seq, tab, oblocks, ohead, h, "bf16")
        assert_close(to_np(logits[k]), ref, "bf16", f"logits at step {k}", tol=E2E_TOL)
        if k < n:
            tk = toks[k].cpu().numpy()
            np.testing.assert_array_equal(tk, O.greedy_token(to_np(logits[k])))
            seq = tk[:, None].astype(np.int64)
    # the model's own loop gives the same tokens
    st2 = mmf.State(2, B, d)
    gen = model.generate(st2, prompt.cuda(), n)
    np.testing.assert_array_equal(gen.cpu().numpy(), torch.stack(toks, 1).cpu().numpy())


def test_argmax_nan_and_infinities():
    # a NaN counts as the largest value (first NaN wins), -inf rows pick index 0,
    # +inf beats every finite value; the same decisions as the oracle's argmax
    V = 300
    rows = torch.full((5, V), -float("inf"))
    rows[1, 7] = 1.0
    rows[1, 200] = float("inf")
    rows[2, 50] = float("nan")
    rows[2, 60] = float("nan")
    rows[2, 70] = float("inf")
    rows[3] = synth.activations(907, 1, V)[0]
    rows[3, 299] = float("inf")
    rows[4] = synth.activations(908, 1, V)[0]
    for dtype in ("bf16", "f32"):
        lg = rows.to(TORCH_DT[dtype])
        ids = mmf.argmax(lg.cuda()).cpu().numpy()
        np.testing.assert_array_equal(ids, O.greedy_token(to_np(lg)))
    assert list(ids[:4]) == [0, 200, 50, 299]
