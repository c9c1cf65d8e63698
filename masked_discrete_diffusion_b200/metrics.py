"""Inference-efficiency metrics of block-wise diffusion decoding.

"DiffusionGemma 技术报告" (full translation page), §3.4 "推理效率指标":
with K canvases, N_k denoising forwards and C_k valid tokens in canvas k,
  total tokens            = sum_k C_k
  total denoising steps   = sum_k N_k
  effective denoise steps = sum_k C_k N_k / sum_k C_k      (token-weighted mean)
  tokens per forward      = sum_k C_k / (sum_k N_k + K - 1)
where the K - 1 term counts the forwards that append each finished canvas to the
KV cache.  §6, paragraph on batch-1 serving throughput: TPS = TPF / t_fwd.
"""
from __future__ import annotations


def total_tokens(C_k) -> int:
    return int(sum(C_k))


def total_steps(N_k) -> int:
    return int(sum(N_k))


def effective_steps(C_k, N_k) -> float:
    tot = sum(C_k)
    return sum(c * n for c, n in zip(C_k, N_k)) / tot if tot else 0.0


def tokens_per_forward(C_k, N_k) -> float:
    K = len(C_k)
    den = sum(N_k) + K - 1
    return sum(C_k) / den if den > 0 else 0.0


def tokens_per_second(tpf: float, t_fwd_s: float) -> float:
    return tpf / t_fwd_s


def canvas_tokens_per_second(batch: int, canvas: int, block_seconds: float) -> float:
    """Canvas tokens completed per second when a block of `batch` canvases takes
    `block_seconds` of device time (all of its forwards and sampler steps)."""
    return batch * canvas / block_seconds
