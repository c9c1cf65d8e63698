"""Shared set-up for the GPU parity tests: build a model from a workload's seeded weights."""
import torch

from masked_discrete_diffusion_b200 import binding, build
from synth import model_inputs


def make_model(w, max_batch=None, max_prompt=None):
    build.build()
    tensors = model_inputs.weight_set(w, "cuda")
    cfg = binding.make_config(w, max_batch, max_prompt)
    return binding.Model(cfg, tensors)


def max_abs_rel(a, b):
    """max |a - b| / max |b| (b the oracle)."""
    import numpy as np
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))
