"""Workload shapes for the masked-diffusion denoise forward.

Each workload is a model stand-in (dimensions, precision) plus an input recipe
(batch, prompt length, number of denoise steps T, entropy bound gamma, seed).
The dimensions the pages fix come from the explainer page "DiffusionGemma
深度解析", list "核心架构参数" (30 layers, sliding window 1024, 256-token
canvas, 262K vocabulary, 128 experts with top-8 routing plus one shared
expert); the hidden sizes are stand-ins the pages do not give.

This module only describes shapes; it holds none of the model's arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    expert_inter: int
    shared_inter: int
    vocab: int            # real tokens; the [MASK] id equals vocab
    window: int           # sliding attention window over the prompt
    canvas: int           # C, tokens denoised in parallel
    rope_base: float
    rms_eps: float
    logit_scale: float
    dtype: str            # "f32" | "bf16" | "bf16_fp8exp" | "bf16_fp4exp"
    batch: int
    prompt_len: int
    T: int                # denoise forwards per block
    gamma: float          # entropy bound of the sampler
    seed: int = 0
    init_std: float = 0.02
    sc_inter: int = 0     # self-conditioning FFW inner size (0: no self-conditioning)
    sc_std: float = 0.02  # standard deviation of the self-conditioning FFW's weights

    @property
    def mask_id(self) -> int:
        return self.vocab

    @property
    def kv_window(self) -> int:
        return min(self.prompt_len, self.window)

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# Tiny fp32 model: the exact-trajectory case (T = 4).
TINY_F32 = Workload(
    name="tiny-f32", n_layers=2, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16,
    n_experts=8, top_k=2, expert_inter=128, shared_inter=128, vocab=512, window=1024,
    canvas=32, rope_base=10000.0, rms_eps=1e-6, logit_scale=8.0, dtype="f32",
    batch=1, prompt_len=32, T=4, gamma=1.0)

# One Gemma-4-26B-A4B-shaped layer plus the 262,144-token LM head, BF16.
LAYER1_BF16 = Workload(
    name="layer1-bf16", n_layers=1, d_model=2048, n_q_heads=16, n_kv_heads=8, head_dim=128,
    n_experts=128, top_k=8, expert_inter=768, shared_inter=2048, vocab=262144, window=1024,
    canvas=256, rope_base=10000.0, rms_eps=1e-6, logit_scale=8.0, dtype="bf16",
    batch=1, prompt_len=1024, T=12, gamma=1.0)

# Full 30-layer stand-in, batch 1, prompt 1024: the throughput workload.
FULL30_BF16 = LAYER1_BF16.with_(name="full30-bf16", n_layers=30)

# Same model, 8 independent canvases with 8192-token prompts (window 1024).
FULL30_B8_P8192 = FULL30_BF16.with_(name="full30-b8-p8192", batch=8, prompt_len=8192)


def full30_fp8exp(batch: int) -> Workload:
    """Same model with FP8 E4M3 expert weights, prompt 4096, the given batch."""
    return FULL30_BF16.with_(name=f"full30-fp8exp-b{batch}", dtype="bf16_fp8exp",
                             batch=batch, prompt_len=4096)


# Small bf16 model for fast parity tests of the tensor-core path: several tiles per
# GEMM with ragged tails (B*C = 288 rows), a prompt longer than the window
# (160 > 128), experts receiving more than 256 rows, 4 vocabulary tiles.
SMALL_BF16 = Workload(
    name="small-bf16", n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
    n_experts=8, top_k=4, expert_inter=128, shared_inter=192, vocab=1024, window=128,
    canvas=96, rope_base=10000.0, rms_eps=1e-6, logit_scale=8.0, dtype="bf16",
    batch=3, prompt_len=160, T=6, gamma=1.0)

# FP8-expert variants for parity tests: the small model, and one full-size layer with
# the FP8 workload's 4096-token prompt.
SMALL_FP8 = SMALL_BF16.with_(name="small-fp8exp", dtype="bf16_fp8exp")
LAYER1_FP8 = LAYER1_BF16.with_(name="layer1-fp8exp-p4096", dtype="bf16_fp8exp", prompt_len=4096)

# Ragged shapes of the full-size kernels: a prompt shorter than the window and not a
# multiple of the 64-key tile (200), two canvases, and a canvas that is not a multiple
# of the 128-row query tile (96).
LAYER1_P200_B2 = LAYER1_BF16.with_(name="layer1-bf16-p200-b2", prompt_len=200, batch=2)
LAYER1_P200_B2_C96 = LAYER1_P200_B2.with_(name="layer1-bf16-p200-b2-c96", canvas=96)

# NVFP4-expert variants (E2M1 codes, an E4M3 scale per 16 input columns and a
# power-of-two scale per tensor): the small model and one full-size layer.
SMALL_FP4 = SMALL_BF16.with_(name="small-fp4exp", dtype="bf16_fp4exp")
LAYER1_FP4 = LAYER1_BF16.with_(name="layer1-fp4exp", dtype="bf16_fp4exp")


def full30_fp4exp(batch: int) -> Workload:
    """The 30-layer model with NVFP4 expert weights, prompt 1024, the given batch."""
    return FULL30_BF16.with_(name=f"full30-fp4exp-b{batch}", dtype="bf16_fp4exp", batch=batch)


# One FP8-expert layer at the batches where each expert holds several 128-row token
# chunks (the tensor-bound part of the FP8 sweep).
LAYER1_FP8_B16 = LAYER1_FP8.with_(name="layer1-fp8exp-p4096-b16", batch=16)
LAYER1_FP8_B64 = LAYER1_FP8.with_(name="layer1-fp8exp-p4096-b64", batch=64)

# Self-conditioning variants (the Report's decoder input z = FFW(p0 E)): the FFW inner
# size of the full-size model is the shared expert's.
TINY_F32_SC = TINY_F32.with_(name="tiny-f32-sc", sc_inter=128, sc_std=4.0)
SMALL_BF16_SC = SMALL_BF16.with_(name="small-bf16-sc", sc_inter=192, sc_std=1.0)
LAYER1_BF16_SC = LAYER1_BF16.with_(name="layer1-bf16-sc", sc_inter=2048)
FULL30_BF16_SC = FULL30_BF16.with_(name="full30-bf16-sc", sc_inter=2048)

WORKLOADS = {w.name: w for w in (TINY_F32, SMALL_BF16, LAYER1_BF16, FULL30_BF16,
                                 FULL30_B8_P8192, SMALL_FP8, LAYER1_FP8, LAYER1_P200_B2,
                                 LAYER1_P200_B2_C96, LAYER1_FP8_B16, LAYER1_FP8_B64,
                                 TINY_F32_SC, SMALL_BF16_SC, LAYER1_BF16_SC, FULL30_BF16_SC,
                                 SMALL_FP4, LAYER1_FP4)}
for _b in (1, 4, 16, 32, 64):
    WORKLOADS[f"full30-fp8exp-b{_b}"] = full30_fp8exp(_b)
    WORKLOADS[f"full30-fp4exp-b{_b}"] = full30_fp4exp(_b)


def get(name: str) -> Workload:
    return WORKLOADS[name]
