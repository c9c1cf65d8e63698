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
    """Tolerance for a deep workload's output `key`: the stated one where the oracle's
    bf16-storage run (key + "_s16") stays within 1e-2 of its fp64 run (bf16 storage is
    not amplified there), else 1.5x that distance (never below the stated one).  A bf16
    path stores bf16 where that run does, so its error is a perturbation of the same
    size, amplified alike through the layers."""
    a, b = g[key + "_s16"], g[key]
    if index is not None:
        a, b = a[index], b[index]
    dist = max_abs_rel(a, b)
    return stated if dist < 1e-2 else max(stated, 1.5 * dist)
