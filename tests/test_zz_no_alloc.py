"""mmf_bitlinear_noalloc: the BitLinear entry point for callers that cannot allocate.

Some callers get only their input and output buffers and may not allocate
device memory (a plug-in operator inside another framework, a process whose
device-memory budget is reserved up front). For them the library offers a
variant of mmf_bitlinear whose scratch is a fixed array inside the library.
These tests call it through the C ABI and check it against mmf_bitlinear (the
entry point that takes a workspace), on two calls in a row so that the second
call cannot pass by reading what the first one left in the shared array.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synth
from parity import TORCH_DT, assert_close, to_np

pytestmark = pytest.mark.gpu

mmf = pytest.importorskip("ternary_weight_matmul_fusedbitlinear_b200")
from ternary_weight_matmul_fusedbitlinear_b200 import _lib as L  # noqa: E402

DT_CODE = {"bf16": L.MMF_BF16, "f32": L.MMF_F32}


def _noalloc(lin, x, dtype):
    lib = L.load()
    M = x.shape[0]
    y = torch.empty(M, lin.N, dtype=x.dtype, device=x.device)
    cl = lin.c()
    st = lib.mmf_bitlinear_noalloc(ctypes.byref(cl), ctypes.c_void_p(x.data_ptr()), DT_CODE[dtype], M,
                                   ctypes.c_void_p(y.data_ptr()), 1e-6,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    L.check(st, "mmf_bitlinear_noalloc")
    return y


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("k,n,m", [(2048, 2048, 1), (2048, 5632, 16), (5632, 2048, 4), (1024, 3072, 130)])
def test_noalloc_matches_bitlinear_two_calls_in_a_row(k, n, m, dtype):
    W = synth.latent_weight(1200 + k + n, n, k).cuda()
    lin = mmf.quantize_weights(W)
    for call in range(2):
        x = synth.activations(1300 + 7 * call + m, m, k, TORCH_DT[dtype], outlier_p=0.001).cuda()
        y_ws = mmf.bitlinear(lin, x)          # the entry point that takes a workspace
        y_na = _noalloc(lin, x, dtype)
        torch.cuda.synchronize()
        assert_close(to_np(y_na), to_np(y_ws), dtype, f"call {call + 1}")


def test_noalloc_rejects_sizes_beyond_its_array():
    k, n = 4096, 256
    lin = mmf.quantize_weights(synth.latent_weight(1400, n, k).cuda())
    x = torch.zeros(1024, k, dtype=torch.bfloat16, device="cuda")     # 4 MiB of codes > 2 MiB
    lib = L.load()
    y = torch.empty(1024, n, dtype=torch.bfloat16, device="cuda")
    cl = lin.c()
    st = lib.mmf_bitlinear_noalloc(ctypes.byref(cl), ctypes.c_void_p(x.data_ptr()), L.MMF_BF16, 1024,
                                   ctypes.c_void_p(y.data_ptr()), 1e-6, None)
    assert st == 2
    assert b"scratch" in lib.mmf_last_error()


def test_noalloc_size_limit_boundary():
    # K = 4096: M = 511 tokens fill the array exactly (511*4096 bytes of codes
    # plus two 2048-byte slots for scales and row sums); M = 512 is one too many
    k, n = 4096, 128
    lin = mmf.quantize_weights(synth.latent_weight(1401, n, k).cuda())
    lib = L.load()
    cl = lin.c()
    for m, want in ((511, 0), (512, 2)):
        x = synth.activations(1402 + m, m, k, torch.bfloat16).cuda()
        y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        st = lib.mmf_bitlinear_noalloc(ctypes.byref(cl), ctypes.c_void_p(x.data_ptr()), L.MMF_BF16, m,
                                       ctypes.c_void_p(y.data_ptr()), 1e-6,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == want, (m, st, lib.mmf_last_error())
        if want == 0:
            assert_close(to_np(y), to_np(mmf.bitlinear(lin, x)), "bf16", f"M={m}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_with_gain_and_bias_matches_bitlinear(dtype):
    k, n, m = 1024, 768, 8
    W = synth.latent_weight(1410, n, k).cuda()
    gain = (1.0 + 0.3 * synth.activations(1411, 1, k)[0]).cuda()
    bias = (0.1 * synth.activations(1412, 1, n)[0]).cuda()
    lin = mmf.quantize_weights(W, gain=gain, bias=bias)
    for call in range(2):
        x = synth.activations(1413 + call, m, k, TORCH_DT[dtype]).cuda()
        assert_close(to_np(_noalloc(lin, x, dtype)), to_np(mmf.bitlinear(lin, x)), dtype, f"call {call + 1}")
