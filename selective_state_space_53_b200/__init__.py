"""B200-native Mamba-3 SSM layer core.

The compute path is ``libm3.so`` (hand-written sm_100a CUDA kernels behind a
C ABI, declared in include/m3.h).  ``selective_state_space_53_b200.m3`` is the
thin ctypes binding; ``inputs`` draws seeded synthetic layer inputs.  Submodules
are imported on demand so that ``inputs`` can be used without a GPU.
"""

__all__ = ["inputs", "m3"]
