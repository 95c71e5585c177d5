"""tcgen05 (tensor-memory) prefill contraction vs the CPU oracle, through the C ABI.

MMF_GEMM_PATH pins the contraction kernel: both kernels must give the exact
int32 accumulators and the same rescaled outputs.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity import TORCH_DT, assert_close, assert_codes_close, check_block_stages, make_block, make_layer, packed_to_np, to_np

pytestmark = pytest.mark.gpu

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")


@pytest.fixture(params=["tc", "mma"])
def path(request, monkeypatch):
    monkeypatch.setenv("MMF_GEMM_PATH", request.param)
    return request.param


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k,n,m", [(256, 256, 1), (1024, 3072, 130), (2048, 2048, 300), (2816, 1024, 257),
                                   (256, 768, 128), (64, 128, 5), (5632, 2048, 129), (1024, 1024, 2048)])
def test_tc_bitlinear_parity(k, n, m, dtype, path):
    _, lin, olin = make_layer(900 + k + n, n, k)
    x = synth.activations(901 + m, m, k, TORCH_DT[dtype], outlier_p=0.001, outlier_scale=20.0)
    y, q, s, acc = mmf.bitlinear(lin, x.cuda(), debug=True)
    torch.cuda.synchronize()
    y_ref, parts = O.bitlinear(to_np(x), olin, parts=True)
    assert_codes_close(q.cpu().numpy(), parts["q"], "codes")
    codes = O.unpack_codes(packed_to_np(lin.packed), k)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), O.ternary_accumulate(q.cpu().numpy(), codes))
    assert_close(to_np(y), y_ref, dtype, "y")


def test_tc_and_mma_agree_exactly(monkeypatch):
    k, n, m = 1024, 3072, 640
    _, lin, _ = make_layer(950, n, k)
    x = synth.activations(951, m, k, torch.bfloat16).cuda()
    monkeypatch.setenv("MMF_GEMM_PATH", "tc")
    _, _, _, acc_tc = mmf.bitlinear(lin, x, debug=True)
    monkeypatch.setenv("MMF_GEMM_PATH", "mma")
    _, _, _, acc_mma = mmf.bitlinear(lin, x, debug=True)
    assert torch.equal(acc_tc, acc_mma)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,d,inner", [(300, 1024, 2816), (128, 256, 768)])
def test_tc_glu_parity(m, d, inner, dtype, path):
    _, gate, og = make_layer(960, inner, d)
    _, up, ou = make_layer(961, inner, d)
    _, down, od = make_layer(962, d, inner)
    x = synth.activations(963, m, d, TORCH_DT[dtype])
    res = synth.activations(964, m, d, TORCH_DT[dtype])
    y = mmf.glu(gate, up, down, x.cuda(), residual=res.cuda())
    blk = O.Block(og, og, og, og, og, ou, od)
    y_ref = O.glu(to_np(x), blk, dtype)
    assert_close(to_np(y), to_np(res) + y_ref, dtype, "glu y")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tc_block_prefill_parity(dtype, path):
    # one block with every contraction on the pinned kernel, stage by stage at TOL
    d, inner, B, T = 256, 768, 3, 100
    blk, oblk = make_block(970, d, inner)
    x = synth.activations(971, B * T, d, TORCH_DT[dtype]).reshape(B, T, d)
    st = mmf.State(1, B, d)
    y, dbg = mmf.block_forward_debug(blk, 0, st, x.cuda())
    mmf.check()
    check_block_stages(x, np.zeros((B, d)), y, st.get()[0].numpy(), dbg, oblk, dtype, f"block ({path})")


def test_tc_wait_gives_up_and_reports(monkeypatch):
    # failure detection without a fault: CTA 0 never loads its second k-step,
    # so the MMA issuer's bounded wait runs out (20 ms); every role of that CTA
    # leaves its loop, the MMAs and copies already started are drained, tensor
    # memory is released, and mmf_check reports code 1; the next call is exact
    k, n, m = 1024, 1024, 512
    _, lin, olin = make_layer(980, n, k)
    x = synth.activations(981, m, k, torch.bfloat16).cuda()
    monkeypatch.setenv("MMF_GEMM_PATH", "tc")
    monkeypatch.setenv("MMF_TC_SKIP_KSTEP", "1")
    monkeypatch.setenv("MMF_WAIT_LIMIT_US", "20000")
    mmf.bitlinear(lin, x)
    with pytest.raises(mmf.MMFError) as err:
        mmf.check()
    assert err.value.status == 6 and "code 1" in str(err.value)
    monkeypatch.delenv("MMF_TC_SKIP_KSTEP")
    monkeypatch.delenv("MMF_WAIT_LIMIT_US")
    y, q, s, acc = mmf.bitlinear(lin, x, debug=True)
    mmf.check()
    codes = O.unpack_codes(packed_to_np(lin.packed), k)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), O.ternary_accumulate(q.cpu().numpy(), codes))
    assert_close(to_np(y), O.bitlinear(to_np(x.cpu()), olin), "bf16", "y after the timeout")
