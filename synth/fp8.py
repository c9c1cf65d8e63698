"""FP8 E4M3 storage of routed-expert weights (workloads whose dtype is "bf16_fp8exp").

Storage format of the workload: for every routed-expert weight row, each block of
128 consecutive input columns has one fp32 scale = max |w| over the block / 448
(1 for an all-zero block); the stored byte is the E4M3 code of w / scale rounded
to nearest, ties to even, saturating at +-448.  The represented weight is
code_value * scale.  E4M3 ("fn"): 1 sign bit, 4 exponent bits (bias 7), 3
mantissa bits, no infinities, largest finite 448, smallest normal 2^-6,
subnormal step 2^-9; byte 0x7F / 0xFF is NaN and never produced.

Every step is exact in fp64 or a correctly rounded fp32 division, so CPU and GPU
produce identical bytes and scales.  This is a weight format; it holds none of
the model's arithmetic.
"""
from __future__ import annotations

import numpy as np
import torch

from . import gen
from .workloads import Workload

BLOCK = 128
E4M3_MAX = 448.0


def e4m3_round(x: torch.Tensor) -> torch.Tensor:
    """Nearest E4M3 value (ties to even), saturating at +-448; fp64 in, fp64 out."""
    a = torch.clamp(x.abs(), max=E4M3_MAX)
    mant, ex = torch.frexp(a)                       # a = mant * 2^ex, mant in [0.5, 1)
    e = (ex - 1).clamp(min=-6)                      # exponent of the quantum's binade
    quantum = torch.ldexp(torch.ones_like(a), e - 3)
    r = torch.round(a / quantum) * quantum          # exact: power-of-two scaling
    return torch.where(x < 0, -r, r)


def e4m3_encode(v: torch.Tensor) -> torch.Tensor:
    """Byte codes (uint8) of exact E4M3 values v (fp64)."""
    a = v.abs()
    sign = (v < 0).to(torch.int32) << 7
    mant, ex = torch.frexp(a)
    e = ex - 1
    normal = a >= 2.0 ** -6
    m_norm = ((a / torch.ldexp(torch.ones_like(a), e) - 1.0) * 8).round().to(torch.int32)
    code_norm = ((e + 7).clamp(min=0).to(torch.int32) << 3) | m_norm
    code_sub = (a / 2.0 ** -9).round().to(torch.int32)
    code = torch.where(normal, code_norm, code_sub)
    return (sign | code).to(torch.uint8)


def e4m3_decode(b: torch.Tensor) -> torch.Tensor:
    """fp64 values of E4M3 byte codes."""
    b = b.to(torch.int32)
    s = torch.where((b >> 7) == 1, -1.0, 1.0).to(torch.float64)
    e = (b >> 3) & 0xF
    m = (b & 7).to(torch.float64)
    one = torch.ones_like(m)
    normal = torch.ldexp(one + m / 8, e - 7)
    sub = m * 2.0 ** -9
    return s * torch.where(e == 0, sub, normal)


def quantize_rows(w: torch.Tensor):
    """w [rows, cols] fp32 (cols % 128 == 0) -> (codes uint8 [rows, cols], scales fp32 [rows, cols/128])."""
    rows, cols = w.shape
    blk = w.reshape(rows, cols // BLOCK, BLOCK)
    amax = blk.abs().amax(dim=2)
    scale = torch.where(amax > 0, amax / torch.tensor(E4M3_MAX, dtype=torch.float32,
                                                        device=w.device), torch.ones_like(amax))
    x = (blk / scale[..., None]).to(torch.float64)
    codes = e4m3_encode(e4m3_round(x)).reshape(rows, cols)
    return codes, scale


def _rows2d(shape):
    return int(np.prod(shape[:-1])), int(shape[-1])


def quantised(w: Workload, name: str, shape, device="cpu"):
    """(codes uint8 with `shape`, scales fp32 [..., cols/128]) of an expert tensor."""
    R, K = _rows2d(shape)
    codes = torch.empty(R, K, dtype=torch.uint8, device=device)
    scales = torch.empty(R, K // BLOCK, dtype=torch.float32, device=device)
    step = max(1, (1 << 24) // K)
    for r in range(0, R, step):
        n = min(step, R - r)
        v = gen.normal_values(w.seed, name, r * K, n * K, w.init_std, device).reshape(n, K)
        codes[r:r + n], scales[r:r + n] = quantize_rows(v)
    return (codes.reshape(shape), scales.reshape(tuple(shape[:-1]) + (K // BLOCK,)))


def dequantised(w: Workload, name: str, shape, start_row: int = 0, n_rows=None) -> np.ndarray:
    """Represented values code * scale (fp64) of rows [start_row, +n_rows) of the leading dim."""
    shape = tuple(shape)
    n_rows = shape[0] - start_row if n_rows is None else n_rows
    inner = int(np.prod(shape[1:-1])) if len(shape) > 2 else 1
    K = shape[-1]
    R0, R = start_row * inner, n_rows * inner
    v = gen.normal_values(w.seed, name, R0 * K, R * K, w.init_std, "cpu").reshape(R, K)
    codes, scales = quantize_rows(v)
    vals = e4m3_decode(codes).reshape(R, K // BLOCK, BLOCK) * scales.to(torch.float64)[..., None]
    return vals.reshape((n_rows,) + shape[1:]).numpy()
