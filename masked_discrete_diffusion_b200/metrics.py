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


def forward_cost(cfg, batch: int, window: int, unique_experts=None):
    """Algorithmic bytes and FLOPs of one canvas forward (all layers + LM head).

    Bytes: weights of the routed experts actually used (unique_experts[l] per layer,
    all E if None), every dense weight (QKV, O, router, shared expert), the LM head,
    the embedding rows gathered, and the cached prompt window's keys and values
    read once.  Intermediate activations and the never-stored logits are not
    counted.  FLOPs: 2 x multiply-adds of every projection over the B*C canvas
    rows (k routed experts per row) plus 4 Hq C (W + C) h per layer for attention,
    plus the LM head.
    """
    L, d, h = cfg.n_layers, cfg.d_model, cfg.head_dim
    Hq, Hkv, E, k = cfg.n_q_heads, cfg.n_kv_heads, cfg.n_experts, cfg.top_k
    I, Is, V, C = cfg.expert_inter, cfg.shared_inter, cfg.vocab, cfg.canvas
    wb = 4 if cfg.dtype == 0 else 2
    if cfg.dtype == 2:    # FP8 codes + an fp32 scale per 128 inputs
        expert_bytes = 3 * I * d + 3 * I * d // 128 * 4
    elif cfg.dtype == 3:  # NVFP4 codes (half a byte) + an E4M3 scale per 16 inputs
        expert_bytes = 3 * I * d // 2 + 3 * I * d // 16
    else:
        expert_bytes = 3 * I * d * wb
    qkv = (Hq + 2 * Hkv) * h
    dense = (qkv * d + d * Hq * h + E * d + 3 * Is * d) * wb
    if unique_experts is None:
        unique_experts = [E] * L
    n = batch * C
    kv_bytes = L * batch * Hkv * window * h * 2 * (8 if cfg.dtype == 0 else 2)
    bytes_ = (sum(unique_experts) * expert_bytes + L * dense + V * d * wb + n * d * wb
              + kv_bytes)
    flops_layer = 2 * n * (qkv * d + d * Hq * h + E * d + k * 3 * I * d + 3 * Is * d) \
        + 4 * Hq * C * (window + C) * h * batch
    flops = L * flops_layer + 2 * n * d * V
    return {"bytes": float(bytes_), "flops": float(flops), "expert_bytes": float(expert_bytes)}
