"""MatMul-free block forward (FusedBitLinear + MLGRU + GLU) for NVIDIA B200.

The computation lives in libmmf.so (hand-written CUDA for sm_100a behind the C
ABI of include/mmf.h); this package only marshals torch tensors into it. The
library must be built (``python -m ternary_weight_matmul_fusedbitlinear_b200.build``);
there is no CPU fallback.
"""
from .api import (  # noqa: F401
    DEFAULT_EPS, Block, State, TLinear, bitlinear, block_forward, block_forward_debug, check, glu, mlgru_scan,
    mlgru_scan_gnorm, mlgru_scan_states, mlgru_scan_backward, quantize_weights, unpack_codes, embed, argmax, Model,
    stack_forward, stack_ws_size, version, prof_enable, prof_reset, prof_collect,
)
from ._lib import LIB_PATH, MMFError, load  # noqa: F401
