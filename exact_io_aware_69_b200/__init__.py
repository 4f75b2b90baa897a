"""Exact scaled-dot-product attention for B200 (sm_100a).

The computation lives in the CUDA library ``libfa.so`` behind the C ABI of
``include/fa.h``; ``exact_io_aware_69_b200.fa`` is its ctypes binding and
``exact_io_aware_69_b200.inputs`` the seeded synthetic-input generator.
"""

__all__ = ["fa", "inputs", "build"]
