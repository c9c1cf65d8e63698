"""NVFP4 storage of routed-expert weights (workloads whose dtype is "bf16_fp4exp").

Storage format of the workload (two-level scaling: a per-tensor scale and one scale per
16 consecutive input columns):
- per expert tensor (one layer's gate, up or down weights of all experts) one fp32
  tensor scale s_t = 2^k, the smallest power of two with 6 * 448 * s_t >= 8 sigma
  (sigma: the workload's weight standard deviation), so that weights within 8 sigma
  need no block scale above the largest E4M3 value;
- per weight row, each block of 16 consecutive input columns has one E4M3 block scale
  s_b = the E4M3 rounding (nearest, ties to even) of max |w| over the block / (6 s_t),
  or 2^-9 (the smallest E4M3 subnormal) where that rounds to 0;
- each weight is stored as the E2M1 code of w / (s_b s_t) rounded to nearest, ties to
  even, saturating at +-6; two codes per byte, element 2i in the low nibble and element
  2i + 1 in the high nibble.
E2M1: sign bit (bit 3), 2 exponent bits (bias 1) and 1 mantissa bit, no infinities or
NaN; the eight magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are codes 0..7 in order.  The
represented weight is e2m1(code) * s_b * s_t, exact in fp32 (at most 2 significant
bits times 4 times a power of two).

Every step is exact in fp64 or a correctly rounded fp64 division followed by a
rounding to the grid, so the bytes and scales are the same on the host and on a GPU.
This is a weight format; it holds none of the model's arithmetic.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import gen
from .fp8 import e4m3_decode, e4m3_encode, e4m3_round
from .workloads import Workload

BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0
E4M3_MIN_SUB = 2.0 ** -9
GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # E2M1 magnitudes of codes 0..7


def tensor_scale(sigma: float) -> float:
    """s_t = 2^k, the smallest power of two with 6 * 448 * s_t >= 8 sigma."""
    return 2.0 ** math.ceil(math.log2(8.0 * sigma / (E2M1_MAX * E4M3_MAX)))


def e2m1_round(x: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 value (ties to even), saturating at +-6; fp64 in, fp64 out.

    The quantum of the binade holding |x| is 2^(e - 1) with e = max(exponent, 0)
    (one mantissa bit; below 1 the subnormal step 0.5), so rounding |x| / quantum to
    the nearest integer, ties to even, lands on the grid with an even mantissa bit."""
    a = torch.clamp(x.abs(), max=E2M1_MAX)
    mant, ex = torch.frexp(a)  # a = mant * 2^ex, mant in [0.5, 1)
    e = (ex - 1).clamp(min=0)
    quantum = torch.ldexp(torch.ones_like(a), e - 1)
    r = torch.clamp(torch.round(a / quantum) * quantum, max=E2M1_MAX)
    return torch.where(x < 0, -r, r)


def e2m1_encode(v: torch.Tensor) -> torch.Tensor:
    """4-bit codes (uint8, 0..15) of exact E2M1 values v (fp64)."""
    grid = torch.tensor(GRID, dtype=torch.float64, device=v.device)
    mag = (v.abs()[..., None] == grid).to(torch.int32).argmax(dim=-1)
    return (((v < 0).to(torch.int32) << 3) | mag).to(torch.uint8)


def e2m1_decode(c: torch.Tensor) -> torch.Tensor:
    """fp64 values of 4-bit E2M1 codes."""
    grid = torch.tensor(GRID, dtype=torch.float64, device=c.device)
    c = c.to(torch.int64)
    v = grid[c & 7]
    return torch.where((c >> 3) == 1, -v, v)


def quantize_rows(w: torch.Tensor, s_t: float):
    """w [rows, cols] (cols % 32 == 0) -> (packed codes uint8 [rows, cols / 2], E4M3 block
    scale bytes uint8 [rows, cols / 16])."""
    rows, cols = w.shape
    blk = w.to(torch.float64).reshape(rows, cols // BLOCK, BLOCK)
    amax = blk.abs().amax(dim=2)
    sb = e4m3_round(amax / (E2M1_MAX * s_t))
    sb = torch.where(sb > 0, sb, torch.full_like(sb, E4M3_MIN_SUB))
    codes = e2m1_encode(e2m1_round(blk / (sb[..., None] * s_t))).reshape(rows, cols)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).to(torch.uint8)
    return packed, e4m3_encode(sb)


def unpack(packed: torch.Tensor) -> torch.Tensor:
    """uint8 [rows, cols / 2] -> 4-bit codes uint8 [rows, cols] (low nibble first)."""
    lo, hi = packed & 0xF, packed >> 4
    return torch.stack((lo, hi), dim=-1).reshape(packed.shape[0], -1)


def _rows2d(shape):
    return int(np.prod(shape[:-1])), int(shape[-1])


def quantised(w: Workload, name: str, shape, sigma: float, device="cpu"):
    """(packed codes uint8 [..., cols / 2], block scales uint8 [..., cols / 16], tensor
    scale fp32 [1]) of an expert tensor of the given shape (cols last)."""
    R, K = _rows2d(shape)
    s_t = tensor_scale(sigma)
    packed = torch.empty(R, K // 2, dtype=torch.uint8, device=device)
    scales = torch.empty(R, K // BLOCK, dtype=torch.uint8, device=device)
    step = max(1, (1 << 22) // K)
    for r in range(0, R, step):
        n = min(step, R - r)
        # on the target device: every step is exact or a correctly rounded fp64
        # division, so the bytes are the same wherever they are computed
        v = gen.normal_values(w.seed, name, r * K, n * K, sigma, device).reshape(n, K)
        packed[r:r + n], scales[r:r + n] = quantize_rows(v, s_t)
    st = torch.tensor([s_t], dtype=torch.float32, device=device)
    return (packed.reshape(tuple(shape[:-1]) + (K // 2,)),
            scales.reshape(tuple(shape[:-1]) + (K // BLOCK,)), st)


def dequantised(w: Workload, name: str, shape, sigma: float, start_row: int = 0,
                n_rows=None) -> np.ndarray:
    """Represented values e2m1(code) * s_b * s_t (fp64) of rows [start_row, +n_rows) of
    the leading dimension."""
    shape = tuple(shape)
    n_rows = shape[0] - start_row if n_rows is None else n_rows
    inner = int(np.prod(shape[1:-1])) if len(shape) > 2 else 1
    K = shape[-1]
    R0, R = start_row * inner, n_rows * inner
    s_t = tensor_scale(sigma)
    v = gen.normal_values(w.seed, name, R0 * K, R * K, sigma, "cpu").reshape(R, K)
    packed, sb = quantize_rows(v, s_t)
    codes = unpack(packed)
    vals = (e2m1_decode(codes).reshape(R, K // BLOCK, BLOCK)
            * e4m3_decode(sb)[..., None] * s_t)
    return vals.reshape((n_rows,) + shape[1:]).numpy()
