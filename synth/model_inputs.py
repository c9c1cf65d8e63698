"""Names, shapes and seeded values of a workload's weights and inputs.

Weight tensors (row-major, the leading index is the output row):
  tok_emb        [V + 1, d]     token embedding; row V is the [MASK] embedding
  lm_head        [V, d]         untied LM head (the [MASK] id is not a class)
  l{l}.wqkv      [(Hq + 2 Hkv) h, d]  rows: the Hq query heads, then Hkv key heads,
                                then Hkv value heads, head-major, h rows per head
  l{l}.wo        [d, Hq h]
  l{l}.router    [E, d]
  l{l}.gate      [E, I, d]      routed experts, SwiGLU gate projection
  l{l}.up        [E, I, d]      routed experts, SwiGLU up projection
  l{l}.down      [E, d, I]      routed experts, down projection
  l{l}.sgate     [I_s, d]       shared expert
  l{l}.sup       [I_s, d]
  l{l}.sdown     [d, I_s]
Every tensor is drawn i.i.d. (approximately) N(0, init_std^2) and stored in the
workload's dtype.  In the FP8-expert workloads the three routed-expert tensors are
additionally quantised (see `synth.fp8` and `synth.nvfp4`).

Inputs: prompt[b] holds `prompt_len` tokens uniform in [0, V).
"""
from __future__ import annotations

import torch

from . import gen
from .workloads import Workload


def layer_specs(w: Workload, l: int):
    d, h, E, I, Is = w.d_model, w.head_dim, w.n_experts, w.expert_inter, w.shared_inter
    return [
        (f"l{l}.wqkv", (w.qkv_rows, d)),
        (f"l{l}.wo", (d, w.n_q_heads * h)),
        (f"l{l}.router", (E, d)),
        (f"l{l}.gate", (E, I, d)),
        (f"l{l}.up", (E, I, d)),
        (f"l{l}.down", (E, d, I)),
        (f"l{l}.sgate", (Is, d)),
        (f"l{l}.sup", (Is, d)),
        (f"l{l}.sdown", (d, Is)),
    ]


def global_specs(w: Workload):
    out = [("tok_emb", (w.vocab + 1, w.d_model)), ("lm_head", (w.vocab, w.d_model))]
    if w.sc_inter > 0:  # the self-conditioning FFW
        out += [("sc.gate", (w.sc_inter, w.d_model)), ("sc.up", (w.sc_inter, w.d_model)),
                ("sc.down", (w.d_model, w.sc_inter))]
    return out


def all_specs(w: Workload):
    out = list(global_specs(w))
    for l in range(w.n_layers):
        out += layer_specs(w, l)
    return out


def store_dtype(w: Workload) -> str:
    return "f32" if w.dtype == "f32" else "bf16"


def std_of(w: Workload, name: str) -> float:
    """Standard deviation a tensor is drawn with: the self-conditioning FFW's own (test
    workloads raise it so that the signal reaches the next forward), else init_std."""
    return w.sc_std if name.startswith("sc.") else w.init_std


def weight(w: Workload, name: str, shape, device="cpu", start_row=0, n_rows=None):
    """Stored (un-quantised) values of one weight tensor or a row range of it."""
    return gen.weight(w.seed, name, shape, std_of(w, name), store_dtype(w), device,
                      start_row, n_rows)


def prompt(w: Workload, device="cpu", first: int = 0) -> torch.Tensor:
    """[B, P] int32 prompt tokens uniform in [0, V) for canvases first .. first + B - 1."""
    rows = [gen.tokens(w.seed, f"prompt.b{b}", w.prompt_len, w.vocab, device)
            for b in range(first, first + w.batch)]
    return torch.stack(rows) if rows else torch.empty(0, w.prompt_len, dtype=torch.int32)


def block_tokens(w: Workload, device="cpu", first: int = 0) -> torch.Tensor:
    """[B, C] int32 tokens uniform in [0, V): finished blocks to append to canvases
    first .. first + B - 1 (stand-ins for denoised canvases)."""
    rows = [gen.tokens(w.seed, f"block.b{b}", w.canvas, w.vocab, device)
            for b in range(first, first + w.batch)]
    return torch.stack(rows)


def is_fp8_expert(w: Workload, name: str) -> bool:
    return (w.dtype == "bf16_fp8exp" and name.startswith("l")
            and name.split(".")[-1] in ("gate", "up", "down"))


def is_fp4_expert(w: Workload, name: str) -> bool:
    return (w.dtype == "bf16_fp4exp" and name.startswith("l")
            and name.split(".")[-1] in ("gate", "up", "down"))


def weight_set(w: Workload, device="cpu") -> dict:
    """Every weight tensor of the workload, keyed by name, in its stored dtype."""
    dt = torch.float32 if store_dtype(w) == "f32" else torch.bfloat16
    out = {}
    for name, shape in all_specs(w):
        if is_fp8_expert(w, name):
            from . import fp8
            q, s = fp8.quantised(w, name, shape, device)
            out[name], out[name.rsplit(".", 1)[0] + "." + name.split(".")[-1] + "_scale"] = q, s
            continue
        if is_fp4_expert(w, name):
            from . import nvfp4
            q, s, st = nvfp4.quantised(w, name, shape, std_of(w, name), device)
            out[name], out[name + "_scale"], out[name + "_tscale"] = q, s, st
            continue
        t = torch.empty(shape, dtype=dt, device=device)
        gen.fill_weight_(t, w.seed, name, std_of(w, name))
        out[name] = t
    return out
