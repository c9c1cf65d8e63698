"""Oracle: the masked-diffusion denoise forward, written out plainly in fp64 numpy.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
bench's CPU-baseline leg may import this module; the CUDA path never does.

The model (passages followed):
* Block-parallel generation of a 256-token canvas conditioned on a causal KV
  cache of the prompt: "DiffusionGemma 技术报告" (full translation page),
  §3.1 "块自回归生成" (KV-cache initialisation, canvas denoising conditioned on
  the cache) and §3.2 "推理时的去噪框架" (decoder forward, bidirectional
  attention inside the canvas).
* Gemma-4-style MoE decoder with a timestep embedding, 30 layers, sliding
  window 1024, 128 experts top-8 plus one shared expert, 262K vocabulary:
  explainer page "DiffusionGemma 深度解析", architecture paragraph and list
  "核心架构参数".
* Canvas starts all [MASK] (absorbing diffusion): explainer page, section on
  absorbing diffusion ("吸收扩散").

Readings of what the pages leave open (RoPE form, timestep embedding,
norm gains, router normalisation, joint softmax over window and canvas, ...)
are fixed in the docstrings below and listed in the design notes.

Precision: weights are read as their stored values (fp32 / bf16 / dequantised
FP8 / dequantised NVFP4) and widened to fp64; every activation and reduction is fp64.  Per-row
entropies are rounded to fp32 at the end, which is the precision the sampler
decides in.

Storage variant (Weights(..., storage="bf16")): the same forward with every
tensor a bf16 model multiplies kept in bf16: the activations rounded where they
are stored (normalised rows entering a projection, q / k / v after RoPE, the
attention output, the SwiGLU hidden rows) and FP8 expert weights dequantised to
bf16 (bf16 weights and dequantised NVFP4 weights are already exact in bf16); residual
stream, router and every sum
stay fp64.  It measures how far bf16 storage alone moves the outputs of a
workload (its sensitivity), from which the tolerances of the deep workloads are
derived.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from synth import model_inputs
from synth.workloads import Workload


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------
def round_bf16(a: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value of fp64 values: 8 significant bits, ties to even.

    a = m 2^e with 0.5 <= |m| < 1; m 2^8 rounded half-to-even to an integer keeps
    8 significant bits (a carry to 256 gives the next power of two).  Exact in fp64;
    the exponent range is not limited (the activations here are far from it).
    """
    m, e = np.frexp(np.asarray(a, dtype=np.float64))
    return np.ldexp(np.round(m * 256.0), e - 8)


def _keep(a: np.ndarray) -> np.ndarray:
    return a


class Weights:
    """Stored weight values as fp64 arrays, generated on demand from the seed.

    `keep_layers` caches every layer (tiny models); otherwise one layer at a
    time is held, so a 30-layer model never needs its full size in RAM.
    `storage` = "fp64" (the oracle) or "bf16" (the storage variant).
    """

    def __init__(self, w: Workload, keep_layers: bool = False, storage: str = "fp64"):
        if storage not in ("fp64", "bf16"):
            raise ValueError(f"storage must be fp64 or bf16, not {storage!r}")
        self.w = w
        self.keep = keep_layers
        self.store = round_bf16 if storage == "bf16" else _keep
        self._cache: dict[str, np.ndarray] = {}

    def _load(self, name, shape, start_row=0, n_rows=None) -> np.ndarray:
        if model_inputs.is_fp8_expert(self.w, name):
            from synth import fp8
            a = fp8.dequantised(self.w, name, shape, start_row, n_rows).astype(np.float64)
            return self.store(a)
        if model_inputs.is_fp4_expert(self.w, name):
            from synth import nvfp4
            a = nvfp4.dequantised(self.w, name, shape, model_inputs.std_of(self.w, name),
                                  start_row, n_rows)
            return self.store(a)
        t = model_inputs.weight(self.w, name, shape, "cpu", start_row, n_rows)
        return t.to(torch.float64).numpy()

    def get(self, name: str, shape) -> np.ndarray:
        if name in self._cache:
            return self._cache[name]
        a = self._load(name, shape)
        if self.keep or not name.startswith("l"):
            self._cache[name] = a
        return a

    def rows(self, name: str, shape, start_row: int, n_rows: int) -> np.ndarray:
        if name in self._cache:
            return self._cache[name][start_row:start_row + n_rows]
        return self._load(name, shape, start_row, n_rows)

    def layer(self, l: int) -> "LayerWeights":
        return LayerWeights(self, l)


class LayerWeights:
    def __init__(self, ws: Weights, l: int):
        w = ws.w
        self.ws, self.l, self.w = ws, l, w
        self.store = ws.store
        specs = dict(model_inputs.layer_specs(w, l))
        self.specs = specs
        qkv = ws.get(f"l{l}.wqkv", specs[f"l{l}.wqkv"])
        nq, nk = w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim
        self.wq, self.wk, self.wv = qkv[:nq], qkv[nq:nq + nk], qkv[nq + nk:]
        self.wo = ws.get(f"l{l}.wo", specs[f"l{l}.wo"])
        self.router = ws.get(f"l{l}.router", specs[f"l{l}.router"])
        self.sgate = ws.get(f"l{l}.sgate", specs[f"l{l}.sgate"])
        self.sup = ws.get(f"l{l}.sup", specs[f"l{l}.sup"])
        self.sdown = ws.get(f"l{l}.sdown", specs[f"l{l}.sdown"])

    def expert(self, e: int):
        """(W_gate [I, d], W_up [I, d], W_down [d, I]) of routed expert e."""
        l, s = self.l, self.specs
        return tuple(self.ws.rows(f"l{l}.{k}", s[f"l{l}.{k}"], e, 1)[0]
                     for k in ("gate", "up", "down"))


# ----------------------------------------------------------------------------
# building blocks
# ----------------------------------------------------------------------------
def rmsnorm(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps), gain fixed at 1 (no learned scale is modelled)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotary embedding, rotate-half form, on x [n, heads, h] at absolute positions pos [n].

    Pair (i, i + h/2) is rotated by the angle pos * base^(-2i/h).
    """
    h = x.shape[-1]
    half = h // 2
    theta = base ** (-2.0 * np.arange(half, dtype=np.float64) / h)
    ang = pos.astype(np.float64)[:, None] * theta[None, :]          # [n, half]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def timestep_embedding(tau: float, d: int) -> np.ndarray:
    """Sinusoidal embedding of the diffusion time tau in (0, 1].

    e[i] = sin(1000 tau w_i), e[d/2 + i] = cos(1000 tau w_i), w_i = 10000^(-i/(d/2)).
    """
    half = d // 2
    omega = 10000.0 ** (-np.arange(half, dtype=np.float64) / half)
    a = 1000.0 * tau * omega
    return np.concatenate([np.sin(a), np.cos(a)])


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(h)) v per query head, restricted to allowed keys.

    q [nq, Hq, h]; k, v [nk, Hkv, h]; allowed [nq, nk] bool.  Query head j reads
    key/value head j // (Hq / Hkv) (grouped-query attention).
    """
    nq, Hq, h = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    out = np.empty_like(q)
    for j in range(Hq):
        kv = j // group
        s = (q[:, j, :] @ k[:, kv, :].T) / math.sqrt(h)
        s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, j, :] = p @ v[:, kv, :]
    return out


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def swiglu(u: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray,
           store=_keep) -> np.ndarray:
    """down(silu(gate u) * up u) for rows u [n, d] (hidden rows kept through `store`)."""
    return store(silu(u @ wg.T) * (u @ wu.T)) @ wd.T


def route(u: np.ndarray, router: np.ndarray, top_k: int):
    """Softmax over all experts, top-k (ties to the lower expert id), renormalised.

    Returns (idx [n, k] int, gate [n, k] fp64, logits [n, E]).
    """
    logits = u @ router.T
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    E = p.shape[1]
    idx = np.empty((p.shape[0], top_k), dtype=np.int64)
    for t in range(p.shape[0]):
        order = sorted(range(E), key=lambda e: (-p[t, e], e))
        idx[t] = order[:top_k]
    g = np.take_along_axis(p, idx, axis=1)
    g = g / g.sum(axis=1, keepdims=True)
    return idx, g, logits


def moe(u: np.ndarray, lw: LayerWeights, top_k: int):
    """Routed experts plus the shared expert (weight 1) on normalised rows u [n, d].

    The router reads u itself; the expert inputs are u as stored (lw.store).
    """
    idx, g, logits = route(u, lw.router, top_k)
    st = lw.store
    us = st(u)
    y = swiglu(us, lw.sgate, lw.sup, lw.sdown, st)
    for e in range(lw.w.n_experts):
        rows, slot = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        wg, wu, wd = lw.expert(e)
        y[rows] += g[rows, slot][:, None] * swiglu(us[rows], wg, wu, wd, st)
    return y, idx, g, logits


def decoder_layer(x, pos, lw: LayerWeights, kv_prev, allowed, w: Workload):
    """One pre-norm block: x += attn(RMSNorm x); x += MoE(RMSNorm x).

    kv_prev = (K [n0, Hkv, h], V [n0, Hkv, h]) keys placed before this block's own
    keys; `allowed` [n, n0 + n] is the attention mask.  Returns (x, k, v, route_info).
    """
    n = x.shape[0]
    H, Hk, h = w.n_q_heads, w.n_kv_heads, w.head_dim
    st = lw.store
    xn = st(rmsnorm(x, w.rms_eps))
    q = (xn @ lw.wq.T).reshape(n, H, h)
    k = (xn @ lw.wk.T).reshape(n, Hk, h)
    v = st((xn @ lw.wv.T).reshape(n, Hk, h))
    q, k = st(rope(q, pos, w.rope_base)), st(rope(k, pos, w.rope_base))
    K = np.concatenate([kv_prev[0], k], axis=0)
    V = np.concatenate([kv_prev[1], v], axis=0)
    o = st(attention(q, K, V, allowed))
    x = x + o.reshape(n, H * h) @ lw.wo.T
    u = rmsnorm(x, w.rms_eps)
    y, idx, g, rlog = moe(u, lw, w.top_k)
    return x + y, k, v, (idx, g, rlog)


# ----------------------------------------------------------------------------
# prefill (causal encoder over the prompt) and the canvas forward
# ----------------------------------------------------------------------------
def causal_window_mask(P: int, window: int) -> np.ndarray:
    """Prompt row j sees keys i with j - window < i <= j (the window includes itself)."""
    i = np.arange(P)
    return (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - window)


def embed(ws: Weights, tokens: np.ndarray) -> np.ndarray:
    w = ws.w
    E = ws.get("tok_emb", (w.vocab + 1, w.d_model))
    return E[np.asarray(tokens, dtype=np.int64)].copy()


def prefill_layer_by_layer(ws: Weights, prompt: np.ndarray):
    """Causal pass over one prompt [P]; yields (layer, K_window, V_window, lw).

    K is kept after RoPE; the window is the last min(P, window) positions.
    """
    w = ws.w
    P = prompt.shape[0]
    W = min(P, w.window)
    x = embed(ws, prompt)
    pos = np.arange(P)
    allowed = causal_window_mask(P, w.window)
    empty = np.zeros((0, w.n_kv_heads, w.head_dim))
    for l in range(w.n_layers):
        lw = ws.layer(l)
        x, k, v, _ = decoder_layer(x, pos, lw, (empty, empty), allowed, w)
        yield l, k[P - W:], v[P - W:], lw


def prefill(ws: Weights, prompt: np.ndarray):
    """List over layers of (K, V) windows, each [W, Hkv, h]."""
    return [(k, v) for _, k, v, _ in prefill_layer_by_layer(ws, prompt)]


def canvas_layer(x, lw, kv, P: int, w: Workload):
    """One layer of the canvas forward: keys = prompt window then all canvas rows."""
    C = x.shape[0]
    W = kv[0].shape[0]
    pos = P + np.arange(C)
    allowed = np.ones((C, W + C), dtype=bool)
    return decoder_layer(x, pos, lw, kv, allowed, w)


def canvas_input(ws: Weights, canvas: np.ndarray, s: int, T: int, z=None) -> np.ndarray:
    """Embedding of the canvas tokens ([MASK] has its own row) plus temb(s / T), plus the
    self-conditioning signal z [C, d] when given."""
    w = ws.w
    x = embed(ws, canvas) + timestep_embedding(s / T, w.d_model)[None, :]
    return x if z is None else x + z


def selfcond_mix(ws: Weights, logits: np.ndarray) -> np.ndarray:
    """y = p0 E: the clean-token probabilities p0 = softmax(logits) (temperature 1, the
    V real tokens) times the token embedding rows of those tokens
    ("DiffusionGemma 技术报告" (full translation page), §3.2 "去噪迭代": the
    self-conditioning signal is a feed-forward network of p0 times the embedding matrix;
    §6: the embedding product runs over the whole vocabulary in full precision)."""
    w = ws.w
    l = np.asarray(logits, dtype=np.float64)
    m = l.max(axis=1, keepdims=True)
    p = np.exp(l - m)
    p /= p.sum(axis=1, keepdims=True)
    E = ws.get("tok_emb", (w.vocab + 1, w.d_model))[:w.vocab]
    return ws.store(p) @ E           # p0 kept through `store` (a bf16 model stores it)


def selfcond(ws: Weights, logits: np.ndarray) -> np.ndarray:
    """z = FFW(p0 E) with FFW(y) = W_down (silu(W_gate y) * W_up y), the next forward's
    self-conditioning input (same section; the FFW's form is this model's SwiGLU)."""
    w = ws.w
    d, I = w.d_model, w.sc_inter
    y = ws.store(selfcond_mix(ws, logits))
    return swiglu(y, ws.get("sc.gate", (I, d)), ws.get("sc.up", (I, d)),
                  ws.get("sc.down", (d, I)), ws.store)


def lm_head_stats(ws: Weights, x: np.ndarray, vocab_chunk: int = 16384, want_logits=False):
    """Final RMSNorm, logits = logit_scale * xn W_lm^T, and per-row statistics.

    Returns dict with H (fp32 entropy in nats, -sum p log p at temperature 1),
    argmax (lowest id on ties), lse, margin (top-1 minus top-2 logit) and
    optionally the logits [n, V].
    """
    w = ws.w
    xn = ws.store(rmsnorm(x, w.rms_eps))
    V = w.vocab
    logits = np.empty((x.shape[0], V))
    for c0 in range(0, V, vocab_chunk):
        n = min(vocab_chunk, V - c0)
        W = ws.rows("lm_head", (V, w.d_model), c0, n)
        logits[:, c0:c0 + n] = w.logit_scale * (xn @ W.T)
    stats = entropy_stats(logits)
    if want_logits:
        stats["logits"] = logits
    return stats


def entropy_stats(logits: np.ndarray):
    """Per-row softmax entropy (nats), argmax, log-sum-exp, top-2 margin and sigma,
    the standard deviation of the logits under the row's own softmax p (the
    first-order gain of the entropy: dH = -Cov_p(l, dl), so |dH| <= sigma max|dl|)."""
    m = logits.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(logits - m).sum(axis=1, keepdims=True))
    logp = logits - lse
    p = np.exp(logp)
    H = -(p * logp).sum(axis=1)
    mean = (p * logits).sum(axis=1, keepdims=True)
    sigma = np.sqrt((p * (logits - mean) ** 2).sum(axis=1))
    am = logits.argmax(axis=1)
    top2 = np.partition(logits, -2, axis=1)[:, -2:]
    return {"H": H.astype(np.float32), "H64": H, "argmax": am.astype(np.int64),
            "lse": lse[:, 0], "margin": top2[:, 1] - top2[:, 0], "sigma": sigma}


def denoise_forward(ws: Weights, kv_layers, canvas: np.ndarray, s: int, T: int, P: int,
                    want_logits=False, want_hidden=False, z=None):
    """Decoder forward over one canvas [C] at steps-left s (self-conditioning input z, or
    none); returns lm_head_stats."""
    w = ws.w
    x = canvas_input(ws, canvas, s, T, z)
    routes = []
    for l in range(w.n_layers):
        x, _, _, r = canvas_layer(x, ws.layer(l), kv_layers[l], P, w)
        routes.append(r)
    st = lm_head_stats(ws, x, want_logits=want_logits)
    st["routes"] = routes
    if want_hidden:
        st["hidden"] = x
    return st


def prefill_then_forward(ws: Weights, prompt: np.ndarray, canvas: np.ndarray, s: int,
                         T: int, want_logits=False, z=None):
    """Prefill of one prompt and one canvas forward, interleaved layer by layer.

    Layer l of the canvas forward needs only the canvas state after layer l-1
    and layer l's prompt window, so running the two passes layer by layer gives
    the same values as running them one after the other while each layer's
    weights are generated once.
    """
    w = ws.w
    P = prompt.shape[0]
    x = canvas_input(ws, canvas, s, T, z)
    kv_layers, routes = [], []
    for l, kw, vw, lw in prefill_layer_by_layer(ws, prompt):
        kv_layers.append((kw, vw))
        x, _, _, r = canvas_layer(x, lw, (kw, vw), P, w)
        routes.append(r)
    st = lm_head_stats(ws, x, want_logits=want_logits)
    st["routes"] = routes
    st["kv"] = kv_layers
    return st


class CanvasForwards:
    """The successive forwards of one block over a fixed context (cache kv of P
    positions), carrying the self-conditioning signal between them when the model has
    one: z = 0 at the block's first forward, afterwards z = selfcond(the previous
    forward's logits) ("DiffusionGemma 技术报告" (full translation page), §3.2
    "解码器前向传播" and "去噪迭代").  `zs` records the z each forward received."""

    def __init__(self, ws: Weights, kv, P: int):
        self.ws, self.kv, self.P = ws, kv, P
        self.z = None
        self.zs = []

    def logits(self, canvas, s: int, T: int):
        w = self.ws.w
        self.zs.append(self.z)
        st = denoise_forward(self.ws, self.kv, canvas, s, T, self.P, want_logits=True, z=self.z)
        if w.sc_inter > 0:
            self.z = selfcond(self.ws, st["logits"])
        return st

    def entropy_bound(self, T: int):
        """forward(canvas, s) -> (H, argmax) for oracle.sampler.generate_block."""
        def forward(canvas, s):
            st = self.logits(canvas, s, T)
            return st["H"], st["argmax"]
        return forward

    def annealed(self, N: int):
        """forward(canvas, k) -> logits for oracle.anneal.generate_block."""
        return lambda canvas, k: self.logits(canvas, N - k, N)["logits"]


def generate_block(ws: Weights, prompt: np.ndarray, T: int, gamma: float):
    """One all-[MASK] canvas denoised by the Entropy-Bound block loop after the causal
    pass over the prompt (with self-conditioning when the model has it).  Returns
    oracle.sampler.generate_block's (canvas, trajectory)."""
    from oracle import sampler
    w = ws.w
    kv = prefill(ws, np.asarray(prompt, dtype=np.int64))
    fw = CanvasForwards(ws, kv, len(prompt))
    return sampler.generate_block(fw.entropy_bound(T), w.canvas, w.mask_id, T, gamma)


def generate_blocks(ws: Weights, prompt: np.ndarray, n_blocks: int, T: int, gamma: float):
    """Block-autoregressive generation: block k is denoised from all [MASK] conditioned
    on the causal pass over the prompt followed by blocks 0 .. k-1, and then joins the
    context ("DiffusionGemma 技术报告" (full translation page), §3.1 "块自回归生成":
    the context is encoded causally, each finished block is appended before the next).

    Returns (blocks [n_blocks, C], trajectories per block as generate_block gives them).
    """
    from oracle import sampler
    w = ws.w
    context = np.asarray(prompt, dtype=np.int64)
    blocks, trajs = [], []
    for _ in range(n_blocks):
        kv = prefill(ws, context)
        fw = CanvasForwards(ws, kv, len(context))
        canvas, traj = sampler.generate_block(fw.entropy_bound(T), w.canvas, w.mask_id, T,
                                              gamma)
        blocks.append(canvas)
        trajs.append(traj)
        context = np.concatenate([context, canvas])
    return np.stack(blocks), trajs


def generate_block_annealed(ws: Weights, prompt: np.ndarray, seed: int, params=None):
    """One canvas denoised by the Report's default sampler (entropy-bounded refinement
    with temperature annealing and adaptive stopping over a uniform-noise canvas,
    "DiffusionGemma 技术报告" (full translation page), §3.2 and §3.3), conditioned on
    the causal pass over the prompt.  Step k's forward takes the time input
    t = (N - k) / N.  Returns oracle.anneal.generate_block's (result, trajectory).
    """
    from oracle import anneal
    p = params or anneal.Params()
    w = ws.w
    kv = prefill(ws, np.asarray(prompt, dtype=np.int64))
    fw = CanvasForwards(ws, kv, len(prompt))
    return anneal.generate_block(fw.annealed(p.N), w.canvas, w.vocab, seed, p)
