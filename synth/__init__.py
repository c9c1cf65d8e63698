"""Seeded synthetic inputs shared by the CUDA path's callers and the oracle.

Workload shapes (`workloads`), a device-independent counter-based generator
(`gen`), the model's weight/input naming (`model_inputs`) and the FP8 storage
format of expert weights (`fp8`).  Nothing here computes any step of the model.
"""
from . import gen, model_inputs, workloads  # noqa: F401
from .workloads import Workload, get  # noqa: F401
