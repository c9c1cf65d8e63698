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


def storage_tol(g, key, stated, index=None):
    """Tolerance for a deep workload's output `key`: the stated one, or twice the
    distance between the oracle's bf16-storage run (key + "_s16") and its fp64 run,
    whichever is larger.  A bf16 path's own rounding is a perturbation of the same
    size as that run's, and both are amplified alike through the layers."""
    a, b = g[key + "_s16"], g[key]
    if index is not None:
        a, b = a[index], b[index]
    return max(stated, 2.0 * max_abs_rel(a, b))
