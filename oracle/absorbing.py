"""Oracle: the absorbing (mask) forward process, used for invariant checks.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Explainer page "DiffusionGemma 深度解析", section on absorbing diffusion
("吸收扩散") and its worked example: at step t of T every token independently
becomes [MASK] (id = vocab size) with probability t / T; t = 0 masks nothing,
t = T masks everything.

The uniform draws are an input (integers k in [0, 65536), read as k / 65536),
so the decision "k / 65536 < t / T" is taken exactly as k * T < t * 65536.
"""
from __future__ import annotations

import numpy as np


def absorb(x, t: int, T: int, mask_id: int, u16):
    """Return (x_noisy, absorbed) for tokens x [..] and draws u16 [..] in [0, 65536)."""
    x = np.asarray(x, dtype=np.int64)
    u16 = np.asarray(u16, dtype=np.int64)
    absorbed = u16 * T < t * 65536
    out = x.copy()
    out[absorbed] = mask_id
    return out, absorbed
