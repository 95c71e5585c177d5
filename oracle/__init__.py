"""CPU oracle for the MatMul-free block forward.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU legs of bench.py. The CUDA library never imports or calls anything here.
"""
from .mmf_oracle import *  # noqa: F401,F403
from . import mmf_oracle  # noqa: F401
