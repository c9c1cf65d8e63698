"""Masked (absorbing) discrete-diffusion denoise forward on B200.

The compute path lives in the CUDA library `libdg.so` (sources in `csrc/`,
C-ABI in `include/dg.h`); `binding` marshals arguments to it with ctypes and
loads it lazily, so `metrics` and the workload helpers import without a GPU.
"""
__all__ = ["binding", "metrics"]
