"""ctypes declarations of the C ABI in include/mmf.h (no arithmetic here)."""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libmmf.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG_DIR), "include", "mmf.h")

MMF_OK = 0
STATUS_NAMES = {
    0: "MMF_OK", 1: "MMF_ERR_INVALID_ARG", 2: "MMF_ERR_UNSUPPORTED_SHAPE", 3: "MMF_ERR_MISALIGNED",
    4: "MMF_ERR_WORKSPACE", 5: "MMF_ERR_CUDA", 6: "MMF_ERR_TIMEOUT", 7: "MMF_ERR_NOMEM",
}
MMF_F32, MMF_BF16 = 0, 1

c_vp = ctypes.c_void_p
c_i32 = ctypes.c_int32
c_sz = ctypes.c_size_t
c_f = ctypes.c_float


class TLinear(ctypes.Structure):
    _fields_ = [("packed", c_vp), ("gamma", c_vp), ("gain", c_vp), ("bias", c_vp), ("N", c_i32), ("K", c_i32),
                ("codes", c_vp)]


class BitlinearDebug(ctypes.Structure):
    _fields_ = [("q", c_vp), ("scale", c_vp), ("acc", c_vp)]


class BlockDebug(ctypes.Structure):
    _fields_ = [("pre", c_vp), ("og", c_vp), ("y1", c_vp), ("p", c_vp), ("q", c_vp * 4), ("scale", c_vp * 4)]


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, TLinear) for n in ("f", "c", "g", "o", "gate", "up", "down")] + [("gnorm", ctypes.c_void_p)]


# name -> (restype, argtypes)
SIGNATURES = {
    "mmf_version": (ctypes.c_char_p, []),
    "mmf_last_error": (ctypes.c_char_p, []),
    "mmf_check": (ctypes.c_int, [c_vp]),
    "mmf_quantize_weights_ws_size": (c_sz, [c_i32, c_i32]),
    "mmf_quantize_weights": (ctypes.c_int, [c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "mmf_unpack_codes": (ctypes.c_int, [c_vp, c_i32, c_i32, c_vp, c_vp]),
    "mmf_bitlinear_ws_size": (c_sz, [c_i32, c_i32]),
    "mmf_bitlinear": (ctypes.c_int, [ctypes.POINTER(TLinear), c_vp, ctypes.c_int, c_i32, c_vp, c_f, c_vp, c_sz,
                                     c_vp, ctypes.POINTER(BitlinearDebug)]),
    "mmf_mlgru_scan_ws_size": (c_sz, [c_i32, c_i32, c_i32]),
    "mmf_mlgru_scan": (ctypes.c_int, [c_vp, ctypes.c_int, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "mmf_mlgru_scan_gnorm_ws_size": (c_sz, [c_i32, c_i32, c_i32]),
    "mmf_mlgru_scan_backward_ws_size": (c_sz, [c_i32, c_i32, c_i32]),
    "mmf_mlgru_scan_backward": (ctypes.c_int, [c_vp, ctypes.c_int, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                               c_vp, c_vp, c_sz, c_vp]),
    "mmf_mlgru_scan_states": (ctypes.c_int, [c_vp, ctypes.c_int, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "mmf_mlgru_scan_gnorm": (ctypes.c_int, [c_vp, ctypes.c_int, c_i32, c_i32, c_i32, c_vp, c_vp, c_f, c_vp, c_vp, c_sz,
                                            c_vp]),
    "mmf_embed": (ctypes.c_int, [c_vp, c_i32, c_vp, c_i32, c_i32, ctypes.c_int, c_vp, c_vp]),
    "mmf_argmax": (ctypes.c_int, [c_vp, ctypes.c_int, c_i32, c_i32, c_vp, c_vp]),
    "mmf_glu_ws_size": (c_sz, [c_i32, c_i32, c_i32]),
    "mmf_glu": (ctypes.c_int, [ctypes.POINTER(TLinear)] * 3 + [c_vp, c_vp, c_vp, c_i32, ctypes.c_int, c_f, c_vp,
                                                             c_sz, c_vp]),
    "mmf_block_create": (ctypes.c_int, [ctypes.POINTER(BlockWeights), c_i32, c_i32, ctypes.POINTER(c_vp)]),
    "mmf_block_destroy": (None, [c_vp]),
    "mmf_block_release_codes": (ctypes.c_int, [c_vp]),
    "mmf_state_create": (ctypes.c_int, [c_i32, c_i32, c_i32, ctypes.POINTER(c_vp)]),
    "mmf_state_destroy": (None, [c_vp]),
    "mmf_state_reset": (ctypes.c_int, [c_vp, c_vp]),
    "mmf_state_layer": (c_vp, [c_vp, c_i32]),
    "mmf_state_get": (ctypes.c_int, [c_vp, c_vp, c_vp]),
    "mmf_state_set": (ctypes.c_int, [c_vp, c_vp, c_vp]),
    "mmf_block_ws_size": (c_sz, [c_vp, c_i32, c_i32]),
    "mmf_block_forward": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, c_vp, c_i32, c_i32, ctypes.c_int, c_f, c_vp, c_sz,
                                         c_vp]),
    "mmf_block_forward_debug": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, c_vp, c_i32, c_i32, ctypes.c_int, c_f, c_vp,
                                               c_sz, c_vp, ctypes.POINTER(BlockDebug)]),
    "mmf_stack_forward": (ctypes.c_int, [ctypes.POINTER(c_vp), c_i32, c_vp, c_vp, c_vp, c_i32, c_i32, ctypes.c_int,
                                         c_f, c_vp, c_sz, c_vp]),
    "mmf_bitlinear_noalloc": (ctypes.c_int, [ctypes.POINTER(TLinear), c_vp, ctypes.c_int, c_i32, c_vp, c_f, c_vp]),
    "mmf_prof_enable": (ctypes.c_int, [c_i32]),
    "mmf_prof_collect": (c_i32, []),
    "mmf_prof_get": (ctypes.c_int, [c_i32, ctypes.c_char_p, c_sz, ctypes.POINTER(ctypes.c_int64),
                                    ctypes.POINTER(ctypes.c_double)]),
    "mmf_prof_reset": (None, []),
}

_lib = None


class MMFError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def load() -> ctypes.CDLL:
    """Load libmmf.so; raises ImportError (never falls back) if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m ternary_weight_matmul_fusedbitlinear_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != MMF_OK:
        msg = load().mmf_last_error().decode(errors="replace")
        raise MMFError(status, where, msg)


def header_functions() -> list[str]:
    """Names of every function the public header declares."""
    import re
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mmf_[a-z0-9_]+)\s*\(", text)))
