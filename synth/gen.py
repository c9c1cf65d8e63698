"""Seeded, device-independent generator for synthetic weights and inputs.

Every value is a pure function of (seed, tensor name, flat element index), so the
CPU (oracle side) and the GPU (CUDA-path side) obtain bit-identical tensors
without either side reading the other's output.

Random bits: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014): state_i = key + (i + 1) * 0x9E3779B97F4A7C15
(mod 2^64), output = mix64(state_i).  The key of a tensor is mix64 of
(seed * 2^32 + CRC-32 of its name).

Weights: an Irwin-Hall(4) sum of the four 16-bit fields of the output, centred
and scaled to the requested standard deviation (an approximately normal draw).
All integer steps are exact and the single fp32 multiply is correctly rounded on
every IEEE device, so CPU and CUDA results agree bit for bit.  The stored dtype
(fp32, or bf16 by round-to-nearest-even) is part of the input definition.

This module holds none of the model's arithmetic.
"""
from __future__ import annotations

import math
import zlib

import numpy as np
import torch

_M64 = (1 << 64) - 1


def _signed(x: int) -> int:
    x &= _M64
    return x - (1 << 64) if x >= (1 << 63) else x


_GOLDEN = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_GOLDEN_S, _C1_S, _C2_S = _signed(_GOLDEN), _signed(_C1), _signed(_C2)


def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (mod 2^64)."""
    z &= _M64
    z = ((z ^ (z >> 30)) * _C1) & _M64
    z = ((z ^ (z >> 27)) * _C2) & _M64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor holding 64 raw bits."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _C1_S
    z = (z ^ _srl(z, 27)) * _C2_S
    return z ^ _srl(z, 31)


def tensor_key(seed: int, name: str) -> int:
    return mix64_int((seed << 32) + zlib.crc32(name.encode()))


def raw_bits(seed: int, name: str, start: int, count: int, device="cpu") -> torch.Tensor:
    """SplitMix64 outputs for flat indices [start, start + count) of a tensor (int64)."""
    key = tensor_key(seed, name)
    idx = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _mix64(idx * _GOLDEN_S + _signed(key))


# Standard deviation of a sum of four independent uniform 16-bit integers.
_IH4_STD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)
_CHUNK = {"cpu": 1 << 22, "cuda": 1 << 26}


def normal_values(seed: int, name: str, start: int, count: int, std: float,
                  device="cpu") -> torch.Tensor:
    """Approximately N(0, std^2) fp32 values for flat indices [start, start+count)."""
    scale = torch.tensor(np.float32(std / _IH4_STD), dtype=torch.float32, device=device)
    out = torch.empty(count, dtype=torch.float32, device=device)
    step = _CHUNK["cuda" if torch.device(device).type == "cuda" else "cpu"]
    for off in range(0, count, step):
        n = min(step, count - off)
        z = raw_bits(seed, name, start + off, n, device)
        s = (z & 0xFFFF) + (_srl(z, 16) & 0xFFFF) + (_srl(z, 32) & 0xFFFF) + _srl(z, 48)
        out[off:off + n] = (s - 131070).to(torch.float32) * scale
    return out


_STORE = {"f32": torch.float32, "bf16": torch.bfloat16}


def weight(seed: int, name: str, shape, std: float, store: str, device="cpu",
           start_row: int = 0, n_rows: int | None = None) -> torch.Tensor:
    """Stored values of a weight tensor (or of rows [start_row, start_row+n_rows) of it).

    `shape` is the full tensor shape; the leading dimension is the row index.
    """
    shape = tuple(int(s) for s in shape)
    row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    n_rows = shape[0] - start_row if n_rows is None else n_rows
    v = normal_values(seed, name, start_row * row, n_rows * row, std, device)
    return v.to(_STORE[store]).reshape((n_rows,) + shape[1:])


def fill_weight_(out: torch.Tensor, seed: int, name: str, std: float,
                 start_row: int = 0) -> torch.Tensor:
    """Write rows [start_row, start_row + out.shape[0]) of tensor `name` into `out`."""
    row = int(np.prod(out.shape[1:])) if out.dim() > 1 else 1
    n = out.shape[0]
    step_rows = max(1, _CHUNK["cuda" if out.is_cuda else "cpu"] // row)
    for r in range(0, n, step_rows):
        m = min(step_rows, n - r)
        v = normal_values(seed, name, (start_row + r) * row, m * row, std, out.device)
        out[r:r + m].copy_(v.reshape((m,) + tuple(out.shape[1:])).to(out.dtype))
    return out


def tokens(seed: int, name: str, count: int, vocab: int, device="cpu") -> torch.Tensor:
    """`count` token ids uniform in [0, vocab) (int32)."""
    z = raw_bits(seed, name, 0, count, device)
    return torch.remainder(_srl(z, 1), vocab).to(torch.int32)


def uniform_u16(seed: int, name: str, count: int, device="cpu") -> torch.Tensor:
    """`count` integers uniform in [0, 65536) (int64)."""
    return raw_bits(seed, name, 0, count, device) & 0xFFFF
