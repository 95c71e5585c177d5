"""The C-ABI library loads, exports every declared symbol and validates arguments (no GPU needed)."""
import ctypes
import subprocess

import pytest

from ternary_weight_matmul_fusedbitlinear_b200 import _lib as L


@pytest.fixture(scope="module")
def lib():
    from ternary_weight_matmul_fusedbitlinear_b200 import build
    build.build()
    return L.load()


def test_every_header_function_is_exported(lib):
    names = L.header_functions()
    assert len(names) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(L.SIGNATURES) == set(names)


def test_build_targets_sm100a_only():
    from ternary_weight_matmul_fusedbitlinear_b200 import build
    assert build.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert all("sm_" not in f or "100a" in f for f in build.NVCC_FLAGS)


def test_version_and_error_message(lib):
    assert lib.mmf_version().decode().startswith("mmf ")
    st = lib.mmf_quantize_weights(None, 4, 16, None, None, None, 0, None)
    assert st == 1
    assert b"null" in lib.mmf_last_error()


def _tl(N, K, packed=16, gamma=16):
    return L.TLinear(packed, gamma, None, None, N, K)


def test_bitlinear_validation_codes(lib):
    x = ctypes.c_void_p(4096)
    y = ctypes.c_void_p(8192)
    ws = ctypes.c_void_p(1 << 20)
    bad_k = _tl(8, 24)
    assert lib.mmf_bitlinear(ctypes.byref(bad_k), x, 0, 4, y, 1e-6, ws, 1 << 20, None, None) == 2
    assert b"multiple of 16" in lib.mmf_last_error()
    mis = _tl(8, 32, packed=18)
    assert lib.mmf_bitlinear(ctypes.byref(mis), x, 0, 4, y, 1e-6, ws, 1 << 20, None, None) == 3
    ok = _tl(8, 32)
    assert lib.mmf_bitlinear(ctypes.byref(ok), x, 0, 4, y, 1e-6, ws, 16, None, None) == 4      # workspace
    assert lib.mmf_bitlinear(ctypes.byref(ok), x, 7, 4, y, 1e-6, ws, 1 << 20, None, None) == 1  # dtype
    assert lib.mmf_bitlinear(ctypes.byref(ok), x, 0, -1, y, 1e-6, ws, 1 << 20, None, None) == 1
    assert lib.mmf_bitlinear(ctypes.byref(ok), x, 0, 4, y, 0.0, ws, 1 << 20, None, None) == 1   # eps
    # M = 0 is a no-op that touches nothing
    assert lib.mmf_bitlinear(ctypes.byref(ok), None, 0, 0, None, 1e-6, None, 0, None, None) == 0


def test_scan_and_glu_validation(lib):
    p = ctypes.c_void_p(4096)
    assert lib.mmf_mlgru_scan(p, 0, 2, 3, 12, p, p, p, 1 << 20, None) == 2          # d % 8
    assert lib.mmf_mlgru_scan(p, 0, -1, 3, 16, p, p, p, 1 << 20, None) == 1
    assert lib.mmf_mlgru_scan(None, 0, 0, 3, 16, None, None, None, 0, None) == 0  # B = 0 no-op
    assert lib.mmf_mlgru_scan(p, 0, 2, 300, 64, p, p, p, 16, None) == 4              # workspace
    assert lib.mmf_mlgru_scan_ws_size(8, 2048, 1024) >= lib.mmf_mlgru_scan_ws_size(1, 256, 32) > 16
    gate, up, down = _tl(64, 32), _tl(64, 32), _tl(32, 64)
    bad_up = _tl(48, 32)
    assert lib.mmf_glu(ctypes.byref(gate), ctypes.byref(bad_up), ctypes.byref(down), p, None, p, 4, 0, 1e-6, p,
                       1 << 20, None) == 2
    up_gain = L.TLinear(16, 16, 32, None, 64, 32)
    assert lib.mmf_glu(ctypes.byref(gate), ctypes.byref(up_gain), ctypes.byref(down), p, None, p, 4, 0, 1e-6, p,
                       1 << 20, None) == 2
    assert b"share one gain" in lib.mmf_last_error()


def test_block_create_validation(lib):
    d, I = 32, 64
    sq = lambda: _tl(d, d)
    w = L.BlockWeights(sq(), sq(), sq(), sq(), _tl(I, d), _tl(I, d), _tl(d, I))
    h = ctypes.c_void_p()
    assert lib.mmf_block_create(ctypes.byref(w), d, I, ctypes.byref(h)) == 0
    assert h.value
    assert lib.mmf_block_ws_size(h, 2, 8) > 0
    lib.mmf_block_destroy(h)
    w.c = L.TLinear(16, 16, 32, None, d, d)  # c has its own gain
    assert lib.mmf_block_create(ctypes.byref(w), d, I, ctypes.byref(h)) == 2
    w.c = _tl(d, d)
    w.down = _tl(d, 48)
    assert lib.mmf_block_create(ctypes.byref(w), d, I, ctypes.byref(h)) == 2


def test_state_accessors_on_null_handle(lib):
    assert lib.mmf_state_layer(None, 0) is None
    assert lib.mmf_state_reset(None, None) == 1


def test_workspace_sizes_grow_with_size(lib):
    assert lib.mmf_bitlinear_ws_size(16, 2048) < lib.mmf_bitlinear_ws_size(64, 2048)
    assert lib.mmf_glu_ws_size(4, 1024, 2816) > 4 * 2816
    assert lib.mmf_quantize_weights_ws_size(2048, 2048) >= 8


def test_gnorm_scan_validation(lib):
    p = ctypes.c_void_p(4096)
    ws = lib.mmf_mlgru_scan_gnorm_ws_size(2, 300, 64)
    assert ws >= 4 * 2 * 300 * 64 + 4 * 2 * 300 * 2
    assert lib.mmf_mlgru_scan_gnorm(p, 0, 2, 3, 12, p, p, 1e-6, p, p, 1 << 20, None) == 2       # d % 8
    assert lib.mmf_mlgru_scan_gnorm(p, 0, 2, 3, 16, p, p, 0.0, p, p, 1 << 20, None) == 1        # eps
    assert lib.mmf_mlgru_scan_gnorm(p, 0, 2, 3, 16, p, None, 1e-6, p, p, 1 << 20, None) == 1    # gain
    assert lib.mmf_mlgru_scan_gnorm(p, 0, 2, 3, 16, p, ctypes.c_void_p(4100), 1e-6, p, p, 1 << 20, None) == 3
    assert lib.mmf_mlgru_scan_gnorm(p, 0, 2, 300, 64, p, p, 1e-6, p, p, ws - 1, None) == 4      # workspace
    assert lib.mmf_mlgru_scan_gnorm(None, 0, 0, 3, 16, None, None, 1e-6, None, None, 0, None) == 0  # B = 0


def test_model_end_validation(lib):
    p = ctypes.c_void_p(4096)
    assert lib.mmf_embed(p, 4, p, 100, 24, 1, p, None) == 2                # d % 16
    assert lib.mmf_embed(p, -1, p, 100, 32, 1, p, None) == 1
    assert lib.mmf_embed(p, 4, p, 0, 32, 1, p, None) == 1                  # V
    assert lib.mmf_embed(p, 4, ctypes.c_void_p(4098), 100, 32, 1, p, None) == 3
    assert lib.mmf_embed(None, 4, p, 100, 32, 1, p, None) == 1
    assert lib.mmf_embed(None, 0, None, 100, 32, 1, None, None) == 0       # M = 0
    assert lib.mmf_argmax(p, 1, 2, 0, p, None) == 1                        # V
    assert lib.mmf_argmax(None, 1, 2, 10, p, None) == 1
    assert lib.mmf_argmax(None, 1, 0, 10, None, None) == 0                 # M = 0
    assert lib.mmf_argmax(p, 5, 2, 10, p, None) == 1                       # dtype


def test_block_gnorm_gain_validation_and_workspace(lib):
    d, I = 32, 64
    sq = lambda: _tl(d, d)
    w = L.BlockWeights(sq(), sq(), sq(), sq(), _tl(I, d), _tl(I, d), _tl(d, I), None)
    h = ctypes.c_void_p()
    assert lib.mmf_block_create(ctypes.byref(w), d, I, ctypes.byref(h)) == 0
    plain = lib.mmf_block_ws_size(h, 2, 8)
    lib.mmf_block_destroy(h)
    w.gnorm = 4104   # not 16-byte aligned
    assert lib.mmf_block_create(ctypes.byref(w), d, I, ctypes.byref(h)) == 3
    w.gnorm = 4096
    assert lib.mmf_block_create(ctypes.byref(w), d, I, ctypes.byref(h)) == 0
    # the g_norm scan's scratch (v in fp32 and the partial sums) comes on top
    assert lib.mmf_block_ws_size(h, 2, 8) >= plain + lib.mmf_mlgru_scan_gnorm_ws_size(2, 8, d) - 256
    lib.mmf_block_destroy(h)


def test_scan_backward_validation(lib):
    p = ctypes.c_void_p(4096)
    q = ctypes.c_void_p(1 << 20)
    ws = lib.mmf_mlgru_scan_backward_ws_size(2, 300, 64)
    assert ws >= 4 * 2 * 300 * 64
    assert lib.mmf_mlgru_scan_backward(p, 0, 2, 3, 12, p, p, None, None, p, q, p, 1 << 20, None) == 2      # d % 8
    assert lib.mmf_mlgru_scan_backward(p, 0, 2, 3, 16, None, p, None, None, p, q, p, 1 << 20, None) == 1   # null h0
    assert lib.mmf_mlgru_scan_backward(p, 0, 2, 3, 16, p, p, None, None, p, p, p, 1 << 20, None) == 1      # h0 = dh0
    assert lib.mmf_mlgru_scan_backward(p, 0, 2, 3, 16, p, p, ctypes.c_void_p(4104), None, p, q, p, 1 << 20, None) == 3
    assert lib.mmf_mlgru_scan_backward(p, 0, 2, 300, 64, p, p, None, None, p, q, p, ws - 1, None) == 4      # workspace
    assert lib.mmf_mlgru_scan_backward(None, 0, 0, 3, 16, None, None, None, None, None, None, None, 0, None) == 0
    # with the forward states given no scratch is needed; a wrong-size workspace is then not an error
    assert lib.mmf_mlgru_scan_backward(p, 0, 2, 3, 12, p, p, None, p, p, q, None, 0, None) == 2          # d % 8 still
    assert lib.mmf_mlgru_scan_states(p, 0, 2, 3, 16, p, None, None, None) == 1                          # null hs
    assert lib.mmf_mlgru_scan_states(p, 0, 2, 3, 16, p, ctypes.c_void_p(4100), p, None) == 3            # misaligned o
