"""Oracle: the Entropy-Bound (EB) sampler step and the block loop, in plain Python.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Passages followed:
* "DiffusionGemma 技术报告" (full translation page), §3.3 "DiffusionGemma 采样器",
  paragraph "熵有界的 token 精炼": positions are accepted in ascending order of
  entropy until an error bound is reached.
* Explainer page "DiffusionGemma 深度解析", section "Entropy Bound (EB) 采样器":
  low-entropy positions are updated first, high-entropy ones are left for later
  steps; section on absorbing diffusion: the reverse process starts from an all
  [MASK] canvas and replaces [MASK] until none is left.
* The workload's rule: the bound is a cumulative entropy <= gamma, at least
  ceil(masked / steps_left) positions are committed, each committed position
  takes its argmax token, ties in entropy go to the lower position.

Reading of the cumulative sum (bit-exact by construction): each entropy h (fp32,
clamped to [0, inf), NaN treated as +inf) becomes q = min(floor(h * 2^48), 2^54)
as an integer; gamma becomes min(floor(gamma * 2^48), 2^62).  The accepted
prefix is the longest whose integer sum is <= the integer bound.
"""
from __future__ import annotations

import math

import numpy as np

Q_SHIFT = 48
Q_CAP = 1 << 54
G_CAP = 1 << 62


def entropy_key(h) -> float:
    """Clamped entropy the sampler orders and sums (fp32 value as a Python float)."""
    h = float(np.float32(h))
    if math.isnan(h):
        return math.inf
    return max(h, 0.0)


def q48(h: float) -> int:
    if math.isinf(h):
        return Q_CAP
    return min(math.floor(h * (1 << Q_SHIFT)), Q_CAP)


def gamma_q48(gamma: float) -> int:
    g = float(np.float32(gamma))
    if math.isinf(g):
        return G_CAP
    return min(math.floor(g * (1 << Q_SHIFT)), G_CAP)


def eb_step(H, argmax, canvas, mask, steps_left: int, gamma: float):
    """One sampler step on one canvas.

    H [C] fp32 entropies, argmax [C] ids, canvas [C] ids, mask [C] (1 = [MASK]).
    Returns (canvas', mask', n_committed, k_gamma).  Inputs are not modified.
    """
    canvas = np.array(canvas, dtype=np.int64).copy()
    mask = np.array(mask, dtype=np.uint8).copy()
    masked = [i for i in range(len(mask)) if mask[i]]
    m = len(masked)
    if m == 0:
        return canvas, mask, 0, 0
    order = sorted(masked, key=lambda i: (entropy_key(H[i]), i))
    bound = gamma_q48(gamma)
    acc, k_gamma = 0, 0
    for i in order:
        q = q48(entropy_key(H[i]))
        if acc + q > bound:
            break
        acc += q
        k_gamma += 1
    floor_n = -(-m // steps_left)          # ceil(m / steps_left)
    n = min(m, max(k_gamma, floor_n))
    for i in order[:n]:
        canvas[i] = int(argmax[i])
        mask[i] = 0
    return canvas, mask, n, k_gamma


def generate_block(forward, C: int, mask_id: int, T: int, gamma: float):
    """Denoise one canvas from all [MASK] with T forwards.

    forward(canvas, steps_left) -> (H [C] fp32, argmax [C]).  Step k (0-based)
    runs at steps_left s = T - k; the loop stops early once nothing is masked.
    Returns (canvas, trajectory) where trajectory lists per step
    (s, H, argmax, canvas_after, mask_after, n_committed).
    """
    canvas = np.full(C, mask_id, dtype=np.int64)
    mask = np.ones(C, dtype=np.uint8)
    traj = []
    for k in range(T):
        if not mask.any():
            break
        s = T - k
        H, am = forward(canvas, s)
        canvas, mask, n, _ = eb_step(H, am, canvas, mask, s, gamma)
        traj.append((s, np.asarray(H), np.asarray(am), canvas.copy(), mask.copy(), n))
    return canvas, traj
