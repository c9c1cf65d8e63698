"""Oracle: the Report's default sampler — entropy-bounded token refinement with
temperature annealing and adaptive stopping, over a uniform (multinomial) diffusion
canvas.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Passages followed ("DiffusionGemma 技术报告" (full translation page)):
* §3.2 "画布初始化": a canvas is refined for at most N steps of size 1/N, starting at
  t = 1 from tokens drawn uniformly from the vocabulary.
* §3.2 "多项式扩散": the iteration is uniform (multinomial) diffusion, not masking, so a
  token accepted at an earlier step may still change; tokens of earlier canvases are
  frozen.
* §3.3 "熵有界的 token 精炼": tokens are sampled from the temperature-scaled marginals
  of every position; positions are accepted in ascending order of entropy while the
  mutual-information bound stays within the tolerance b = 0.1; every other position is
  re-noised to a uniformly random token.
* §3.3 "温度退火": the temperature moves linearly along the denoising time t in [0, 1]
  from tau_max = 0.8 to tau_min = 0.4.
* §3.3 "自适应停止启发式" (and §3.1 footnote 3): the loop ends before N steps once the
  mean predicted entropy over the canvas is below e_stop = 0.005 and the most likely
  token sequence is the same at two consecutive steps; N = 48 (§3.4, Figure 5).

Readings of what the pages leave open (the same list stands beside the CUDA path):
 A1 step k (0-based) runs at t_k = (N - k) / N: the first forward at t = 1, the last at
    1 / N; the decoder's time input is t_k (steps left s = N - k over N).
 A2 tau(t) = tau_min + (tau_max - tau_min) t (tau_max at the noisy end), in fp64.
 A3 the entropies that are ordered, bounded and averaged are those of the tempered
    distribution softmax(l / tau), the distribution the tokens are drawn from.
 A4 mutual-information bound of the entropy-bounded sampler: a set S of positions is
    accepted when sum_{i in S} H_i - max_{i in S} H_i <= b.  Along the ascending
    (entropy, position) order the accepted set is the longest prefix meeting it, so
    the first position is always accepted and the prefix length is one more than the
    number of leading entropies whose sum stays <= b (at most C).  Sums are exact
    integers of the fixed-point entropies min(floor(h 2^48), 2^54) (NaN -> inf,
    negative -> 0), the bound is min(floor(b 2^48), 2^62).
 A5 each position outside the accepted prefix takes a fresh uniformly drawn token.
 A6 the stop test runs after every step: sum_i q(H_i) < C q(e_stop) with the same
    fixed-point entropies (the sum saturates at 2^63, e_stop <= 16 so the right side
    stays below 2^62), and the argmax sequence equals that of the previous step (never
    true at the first step).  When it passes, or after step N - 1, the canvas's result
    is the argmax sequence of that step's forward.
 A7 draws are SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014), counter-based: the c-th output of the generator started
    at state key is mix64(key + (c + 1) G), G = 0x9E3779B97F4A7C15.  A canvas's seed
    gives three stream keys, key_j = mix64(seed + j G) for j = 1 (initial canvas),
    2 (Gumbel noise), 3 (re-noising).
      initial token of position i:        stream 1, c = i
      Gumbel noise of (k, i, tokens 2p, 2p + 1):
                                           stream 2, c = (k C + i) ceil(V / 2) + p
      re-noise token of (k, i):            stream 3, c = k C + i
    A token from 64 bits z is floor(hi32(z) V / 2^32) (multiply-shift).  One output z
    of stream 2 serves two tokens: the 23-bit field f = bits 63..41 of z for the even
    token, bits 31..9 for the odd one; the Gumbel variate is -log(-log u) with
    u = (f + 1/2) 2^-23 (exact in fp32).  The drawn token is argmax_v (l_v / tau + g_v),
    the lowest id on exact ties (Gumbel-max: a draw from softmax(l / tau)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

G = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1
Q_SHIFT = 48
Q_CAP = 1 << 54
B_CAP = 1 << 62
SUM_CAP = 1 << 63
STREAM_INIT, STREAM_GUMBEL, STREAM_RENOISE = 1, 2, 3


@dataclass(frozen=True)
class Params:
    """Sampler constants (§3.3): N steps at most, MI tolerance b, temperatures at
    t = 1 and t = 0, mean-entropy threshold of the adaptive stop."""
    N: int = 48
    b: float = 0.1
    tau_max: float = 0.8
    tau_min: float = 0.4
    e_stop: float = 0.005


# ---------------------------------------------------------------------------
# SplitMix64 (A7)
# ---------------------------------------------------------------------------
def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on uint64 arrays (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def splitmix_outputs(state: int, count: int) -> np.ndarray:
    """The first `count` outputs of the sequential generator started at `state`:
    state += G, output mix64(state)."""
    out = np.empty(count, dtype=np.uint64)
    s = state & _M64
    for j in range(count):
        s = (s + G) & _M64
        out[j] = mix64(np.uint64(s))
    return out


def stream_key(seed: int, stream: int) -> int:
    return int(mix64(np.uint64((seed + stream * G) & _M64)))


def draw(key: int, counters) -> np.ndarray:
    """Outputs number `counters` (0-based) of the generator started at `key`."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(key) + (c + np.uint64(1)) * np.uint64(G))


def token_from_bits(z: np.ndarray, V: int) -> np.ndarray:
    hi = np.asarray(z, dtype=np.uint64) >> np.uint64(32)
    return ((hi * np.uint64(V)) >> np.uint64(32)).astype(np.int64)   # V < 2^32: no wrap


def gumbel_from_field(f: np.ndarray) -> np.ndarray:
    """Gumbel variate of a 23-bit field f: -log(-log u), u = (f + 1/2) 2^-23."""
    u = (np.asarray(f, dtype=np.float64) + 0.5) * 2.0 ** -23
    return -np.log(-np.log(u))


def fields_of_bits(z: np.ndarray) -> np.ndarray:
    """The two 23-bit fields of each output: [..., 2] = (bits 63..41, bits 31..9)."""
    z = np.asarray(z, dtype=np.uint64)
    m = np.uint64((1 << 23) - 1)
    return np.stack([z >> np.uint64(41), (z >> np.uint64(9)) & m], axis=-1)


def initial_canvas(seed: int, C: int, V: int) -> np.ndarray:
    """x_1: C uniform tokens (§3.2 canvas initialisation)."""
    return token_from_bits(draw(stream_key(seed, STREAM_INIT), np.arange(C)), V)


def gumbel_row(seed: int, k: int, i: int, C: int, V: int) -> np.ndarray:
    """Gumbel noise of all V tokens at step k, position i (token v from output
    (k C + i) ceil(V / 2) + floor(v / 2) of stream 2, field v mod 2)."""
    half = (V + 1) // 2
    c0 = (k * C + i) * half
    f = fields_of_bits(draw(stream_key(seed, STREAM_GUMBEL), np.arange(c0, c0 + half)))
    return gumbel_from_field(f.reshape(-1)[:V])


def renoise_tokens(seed: int, k: int, C: int, V: int) -> np.ndarray:
    """The re-noise token every position of the canvas would take at step k."""
    return token_from_bits(draw(stream_key(seed, STREAM_RENOISE), np.arange(k * C, k * C + C)), V)


# ---------------------------------------------------------------------------
# temperature, tempered statistics, Gumbel-max (A1 - A3, A7)
# ---------------------------------------------------------------------------
def step_time(k: int, N: int) -> float:
    """t of step k (A1)."""
    return (N - k) / N


def temperature(k: int, p: Params) -> float:
    """tau(t_k) = tau_min + (tau_max - tau_min) t_k (A2), the constants read as fp32."""
    tmax, tmin = float(np.float32(p.tau_max)), float(np.float32(p.tau_min))
    return tmin + (tmax - tmin) * step_time(k, p.N)


def tempered_stats(logits: np.ndarray, tau: float):
    """Entropy (nats) and argmax of softmax(l / tau) per row of logits [n, V]."""
    z = np.asarray(logits, dtype=np.float64) / tau
    m = z.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(z - m).sum(axis=1, keepdims=True))
    logp = z - lse
    H = -(np.exp(logp) * logp).sum(axis=1)
    return {"H": H.astype(np.float32), "H64": H, "argmax": z.argmax(axis=1).astype(np.int64)}


def gumbel_max(zrow: np.ndarray, g: np.ndarray):
    """(argmax of z + g, lowest id on ties; gap between the best and second best)."""
    y = np.asarray(zrow, dtype=np.float64) + g
    v = int(np.argmax(y))
    top2 = np.partition(y, -2)[-2:] if y.shape[0] > 1 else np.array([-np.inf, y[0]])
    return v, float(top2[1] - top2[0])


def sample_tokens(logits: np.ndarray, tau: float, seed: int, k: int):
    """Gumbel-max draw of every position of one canvas from softmax(l / tau):
    (tokens [C], gaps [C])."""
    C, V = logits.shape
    tok = np.empty(C, dtype=np.int64)
    gap = np.empty(C)
    for i in range(C):
        tok[i], gap[i] = gumbel_max(np.asarray(logits[i], dtype=np.float64) / tau,
                                    gumbel_row(seed, k, i, C, V))
    return tok, gap


# ---------------------------------------------------------------------------
# acceptance, re-noising and the stop test (A4 - A6)
# ---------------------------------------------------------------------------
def entropy_key(h) -> float:
    h = float(np.float32(h))
    if math.isnan(h):
        return math.inf
    return max(h, 0.0)


def q48(h: float) -> int:
    if math.isinf(h):
        return Q_CAP
    return min(math.floor(h * (1 << Q_SHIFT)), Q_CAP)


def b_q48(b: float) -> int:
    v = float(np.float32(b))
    if math.isinf(v):
        return B_CAP
    return min(math.floor(v * (1 << Q_SHIFT)), B_CAP)


def order(H) -> list:
    """Positions by ascending (entropy, position)."""
    return sorted(range(len(H)), key=lambda i: (entropy_key(H[i]), i))


def accepted_count(H, b: float) -> int:
    """Length of the accepted prefix under the MI bound (A4)."""
    bound, acc, lead = b_q48(b), 0, 0
    for i in order(H):
        acc += q48(entropy_key(H[i]))
        if acc > bound:
            break
        lead += 1
    return min(len(H), lead + 1)


def refine(H, sampled, seed: int, k: int, V: int, b: float):
    """One refinement of one canvas: the accepted prefix keeps its drawn tokens, every
    other position is re-noised (A4, A5).  Returns (canvas [C], n_accepted)."""
    C = len(H)
    n = accepted_count(H, b)
    out = renoise_tokens(seed, k, C, V)
    for i in order(H)[:n]:
        out[i] = int(sampled[i])
    return out, n


def entropy_sum_q(H) -> int:
    return min(sum(q48(entropy_key(h)) for h in H), SUM_CAP)


def stop_test(H, argmax, prev_argmax, e_stop: float) -> bool:
    """Adaptive stop after a step (A6); prev_argmax None at the first step."""
    e = float(np.float32(e_stop))
    if not (0.0 <= e <= 16.0):
        raise ValueError("e_stop must be in [0, 16]")
    low = entropy_sum_q(H) < len(H) * q48(e)
    stable = prev_argmax is not None and np.array_equal(np.asarray(argmax), np.asarray(prev_argmax))
    return bool(low and stable)


def generate_block(forward, C: int, V: int, seed: int, p: Params = Params()):
    """Denoise one canvas with the annealed entropy-bounded sampler.

    forward(canvas [C], k) -> logits [C, V] (fp64, temperature 1) of step k, whose
    time input is t_k = (N - k) / N.  Returns (result [C], trajectory) with one entry
    per forward: dict(k, tau, H, argmax, sampled, gap, canvas (after the step),
    n_accepted, stop).
    """
    canvas = initial_canvas(seed, C, V)
    prev, traj = None, []
    for k in range(p.N):
        tau = temperature(k, p)
        logits = forward(canvas, k)
        st = tempered_stats(logits, tau)
        sampled, gap = sample_tokens(logits, tau, seed, k)
        stop = stop_test(st["H"], st["argmax"], prev, p.e_stop)
        if stop or k == p.N - 1:
            new, n = st["argmax"].copy(), C
        else:
            new, n = refine(st["H"], sampled, seed, k, V, p.b)
        traj.append({"k": k, "tau": tau, "H": st["H"], "H64": st["H64"],
                     "argmax": st["argmax"], "sampled": sampled, "gap": gap,
                     "canvas": new.copy(), "n_accepted": n, "stop": stop})
        canvas, prev = new, st["argmax"]
        if stop:
            break
    return canvas, traj
