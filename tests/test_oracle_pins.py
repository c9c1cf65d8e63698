"""Pins of the oracle against what the pages and the mathematics fix.

Each test checks one oracle function against something other than itself: a
closed form, a brute-force loop, a special case that reduces to a library
routine the oracle does not call, an invariant, or values the pages print.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import scipy.stats

from oracle import absorbing, model, sampler
from synth import gen, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# --------------------------------------------------------------- attention
def brute_attention(q, k, v, allowed):
    nq, Hq, h = q.shape
    Hkv = k.shape[1]
    out = np.zeros_like(q)
    for i in range(nq):
        for j in range(Hq):
            kv = j // (Hq // Hkv)
            keys = [t for t in range(k.shape[0]) if allowed[i, t]]
            sc = [sum(q[i, j, c] * k[t, kv, c] for c in range(h)) / math.sqrt(h) for t in keys]
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            z = sum(ex)
            for c in range(h):
                out[i, j, c] = sum(e * v[t, kv, c] for e, t in zip(ex, keys)) / z
    return out


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (2, 2), (4, 1)])
def test_attention_matches_bruteforce(Hq, Hkv):
    nq, nk, h = 5, 7, 4
    q = rng.normal(size=(nq, Hq, h))
    k = rng.normal(size=(nk, Hkv, h))
    v = rng.normal(size=(nk, Hkv, h))
    allowed = rng.random((nq, nk)) < 0.6
    allowed[:, 0] = True
    np.testing.assert_allclose(model.attention(q, k, v, allowed),
                               brute_attention(q, k, v, allowed), rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    q = rng.normal(size=(3, 2, 4))
    k = np.tile(rng.normal(size=(1, 1, 4)), (6, 1, 1))     # all keys equal
    v = rng.normal(size=(6, 1, 4))
    out = model.attention(q, k, v, np.ones((3, 6), bool))
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0), out.shape), atol=1e-14)
    allowed = np.zeros((3, 6), bool)
    allowed[:, 4] = True                                     # a single key
    out = model.attention(q, rng.normal(size=(6, 1, 4)), v, allowed)
    np.testing.assert_allclose(out, np.broadcast_to(v[4], out.shape), atol=1e-14)


# --------------------------------------------------------------- RoPE
def test_rope_identity_norm_relative():
    h, base = 16, 10000.0
    x = rng.normal(size=(1, 3, h))
    np.testing.assert_allclose(model.rope(x, np.array([0]), base), x, atol=0)
    pos = np.array([5, 37, 1000])
    y = model.rope(np.repeat(x, 3, 0), pos, base)
    # every rotated pair keeps its length
    half = h // 2
    n0 = x[..., :half] ** 2 + x[..., half:] ** 2
    n1 = y[..., :half] ** 2 + y[..., half:] ** 2
    np.testing.assert_allclose(n1, np.broadcast_to(n0, n1.shape), rtol=1e-12)
    # q(m) . k(n) depends on m - n only
    q, k = rng.normal(size=(1, 1, h)), rng.normal(size=(1, 1, h))
    for m, n, d in [(3, 1, 10), (100, 7, 250)]:
        a = (model.rope(q, np.array([m]), base) * model.rope(k, np.array([n]), base)).sum()
        b = (model.rope(q, np.array([m + d]), base) * model.rope(k, np.array([n + d]), base)).sum()
        assert abs(a - b) < 1e-9


def test_rope_pair_frequencies():
    """Unit vector on pair i at position p ends up at angle p * base^(-2i/h)."""
    h, base, p = 8, 10000.0, 3
    for i in range(h // 2):
        e = np.zeros((1, 1, h))
        e[0, 0, i] = 1.0
        y = model.rope(e, np.array([p]), base)[0, 0]
        ang = math.atan2(y[i + h // 2], y[i])
        want = math.remainder(p * base ** (-2 * i / h), 2 * math.pi)
        assert abs(math.remainder(ang - want, 2 * math.pi)) < 1e-12
        others = [c for c in range(h) if c not in (i, i + h // 2)]
        assert np.all(y[others] == 0)


# --------------------------------------------------------------- RMSNorm
def test_rmsnorm_closed_form():
    x = rng.normal(size=(4, 64)) * 3.0
    eps = 1e-6
    y = model.rmsnorm(x, eps)
    ms = (x * x).mean(axis=1)
    np.testing.assert_allclose((y * y).mean(axis=1), ms / (ms + eps), rtol=1e-12)
    assert np.all(np.sign(y) == np.sign(x))


# --------------------------------------------------------------- timestep embedding
def test_timestep_embedding_pins():
    d = 64
    e = model.timestep_embedding(math.pi / 2000.0, d)     # 1000*tau*w_0 = pi/2
    assert abs(e[0] - 1.0) < 1e-15 and abs(e[d // 2]) < 1e-15
    for tau in (0.25, 1.0):
        e = model.timestep_embedding(tau, d)
        np.testing.assert_allclose(e[:d // 2] ** 2 + e[d // 2:] ** 2, 1.0, rtol=1e-14)
        # the slowest pair turns at 1000*tau*10000^(-(d/2-1)/(d/2))
        w_last = 10000.0 ** (-(d // 2 - 1) / (d // 2))
        assert abs(math.atan2(e[d // 2 - 1], e[-1]) - 1000 * tau * w_last) < 1e-12


# --------------------------------------------------------------- MoE
class _FakeLayer:
    def __init__(self, E, d, I, Is, w):
        self.w = w
        self.store = lambda a: a   # the fp64 oracle keeps activations as computed
        self.router = rng.normal(size=(E, d))
        self.experts = [(rng.normal(size=(I, d)) * 0.3, rng.normal(size=(I, d)) * 0.3,
                         rng.normal(size=(d, I)) * 0.3) for _ in range(E)]
        self.sgate, self.sup = rng.normal(size=(Is, d)) * 0.3, rng.normal(size=(Is, d)) * 0.3
        self.sdown = rng.normal(size=(d, Is)) * 0.3

    def expert(self, e):
        return self.experts[e]


def _dense_moe(u, L, top_k):
    """All experts evaluated for every row; non-selected gates are zero."""
    n, E = u.shape[0], len(L.experts)
    logits = u @ L.router.T
    p = scipy.special.softmax(logits, axis=1)
    y = np.zeros_like(u)
    for t in range(n):
        top = np.lexsort((np.arange(E), -p[t]))[:top_k]
        gates = np.zeros(E)
        gates[top] = p[t, top] / p[t, top].sum()
        for e in range(E):
            wg, wu, wd = L.experts[e]
            a = u[t] @ wg.T
            hdn = a * scipy.special.expit(a) * (u[t] @ wu.T)
            y[t] += gates[e] * (wd @ hdn)
        a = u[t] @ L.sgate.T
        y[t] += L.sdown @ (a * scipy.special.expit(a) * (u[t] @ L.sup.T))
    return y


@pytest.mark.parametrize("E,k", [(8, 2), (6, 6), (1, 1)])
def test_moe_topk_equals_dense(E, k):
    d, I, Is = 12, 10, 9
    w = workloads.TINY_F32.with_(n_experts=E, top_k=k)
    L = _FakeLayer(E, d, I, Is, w)
    u = rng.normal(size=(7, d))
    y, idx, g, _ = model.moe(u, L, k)
    np.testing.assert_allclose(y, _dense_moe(u, L, k), rtol=1e-11, atol=1e-12)
    if k == E:   # full mixture: gates are the plain softmax
        for t in range(7):
            full = scipy.special.softmax(u[t] @ L.router.T)
            np.testing.assert_allclose(g[t][np.argsort(idx[t])], full, rtol=1e-12)


def test_router_ties_go_to_lower_expert():
    router = np.zeros((6, 2))
    router[[1, 3, 4]] = [1.0, 0.0]
    idx, g, _ = model.route(np.array([[2.0, 0.0]]), router, 2)
    assert list(idx[0]) == [1, 3]
    np.testing.assert_allclose(g[0], [0.5, 0.5])


# --------------------------------------------------------------- entropy / LM-head statistics
def test_entropy_uniform_two_level_gap():
    V = 512
    st = model.entropy_stats(np.full((1, V), 3.25))
    assert abs(st["H64"][0] - math.log(V)) < 1e-12
    assert st["argmax"][0] == 0
    # two-level logits: n_a entries at a, n_b at b
    a, b, na = 2.0, -1.0, 5
    lg = np.full((1, V), b)
    lg[0, 100:100 + na] = a
    Z = na * math.exp(a) + (V - na) * math.exp(b)
    Hc = math.log(Z) - (a * na * math.exp(a) + b * (V - na) * math.exp(b)) / Z
    st = model.entropy_stats(lg)
    assert abs(st["H64"][0] - Hc) < 1e-12 and st["argmax"][0] == 100
    # a 100-nat gap leaves essentially no uncertainty
    lg = np.zeros((1, V))
    lg[0, 7] = 100.0
    st = model.entropy_stats(lg)
    assert 0.0 <= st["H64"][0] < 1e-38 and st["argmax"][0] == 7


def test_entropy_matches_library_and_bounds():
    lg = rng.normal(size=(6, 300)) * 4.0
    st = model.entropy_stats(lg)
    want = scipy.stats.entropy(scipy.special.softmax(lg, axis=1), axis=1)
    np.testing.assert_allclose(st["H64"], want, rtol=1e-12)
    assert np.all(st["H64"] >= 0) and np.all(st["H64"] <= math.log(300) + 1e-12)
    np.testing.assert_allclose(st["lse"], scipy.special.logsumexp(lg, axis=1), rtol=1e-13)
    assert st["H"].dtype == np.float32


# --------------------------------------------------------------- sampler
def _brute_sampler(H, am, canvas, mask, s, gamma):
    """Independent restatement with exact rational prefix sums."""
    masked = [i for i in range(len(mask)) if mask[i]]
    m = len(masked)
    if m == 0:
        return list(canvas), list(mask), 0
    keys = {i: max(float(np.float32(H[i])), 0.0) for i in masked}
    order = sorted(masked, key=lambda i: (keys[i], i))
    g = Fraction(float(np.float32(gamma)))
    best = 0
    for n in range(m + 1):
        if sum((Fraction(keys[i]) for i in order[:n]), Fraction(0)) <= g:
            best = n
        else:
            break
    n = min(m, max(best, math.ceil(m / s)))
    c2, m2 = list(canvas), list(mask)
    for i in order[:n]:
        c2[i], m2[i] = am[i], 0
    return c2, m2, n


@pytest.mark.parametrize("trial", range(40))
def test_sampler_matches_bruteforce(trial):
    r = np.random.default_rng(100 + trial)
    C = int(r.integers(1, 13))
    H = (r.random(C) * r.choice([0.05, 0.3, 2.0])).astype(np.float32)
    if trial % 3 == 0:
        H = np.round(H * 8).astype(np.float32) / 8           # force exact ties
    am = r.integers(0, 50, C)
    mask = (r.random(C) < 0.8).astype(np.uint8)
    canvas = np.where(mask == 1, 50, r.integers(0, 50, C))
    s = int(r.integers(1, 6))
    gamma = float(r.choice([0.0, 0.1, 0.5, 1.0, 3.0]))
    c, mk, n, _ = sampler.eb_step(H, am, canvas, mask, s, gamma)
    c2, m2, n2 = _brute_sampler(H, am, canvas, mask, s, gamma)
    assert n == n2 and list(c) == c2 and list(mk) == m2


def test_sampler_special_cases():
    C = 20
    H = (np.arange(C, dtype=np.float32) + 1) / 7
    am = np.arange(C) + 100
    mask = np.ones(C, np.uint8)
    canvas = np.full(C, 999)
    for s in (1, 2, 3, 7):
        _, _, n, _ = sampler.eb_step(H, am, canvas, mask, s, 0.0)
        assert n == (C if s == 1 else math.ceil(C / s))        # gamma = 0 -> the minimum
    _, mk, n, _ = sampler.eb_step(H, am, canvas, mask, 9, float("inf"))
    assert n == C and not mk.any()
    # equal entropies: lower positions first
    c, mk, n, _ = sampler.eb_step(np.full(C, 0.5, np.float32), am, canvas, mask, 4, 0.0)
    assert n == 5 and list(np.nonzero(mk == 0)[0]) == [0, 1, 2, 3, 4]
    # nothing masked: no-op
    c, mk, n, _ = sampler.eb_step(H, am, canvas, np.zeros(C, np.uint8), 3, 1.0)
    assert n == 0 and list(c) == list(canvas)


def test_block_invariants_with_synthetic_entropies():
    C, T, V = 64, 6, 1000
    step = {"k": 0}

    def fake_forward(canvas, s):
        step["k"] += 1
        u = gen.uniform_u16(7, f"fake.{step['k']}", 2 * C).numpy()
        return (u[:C] / 4096.0).astype(np.float32), u[C:] % V

    canvas, traj = sampler.generate_block(fake_forward, C, V, T, 1.0)
    prev_mask = np.ones(C, np.uint8)
    prev_canvas = np.full(C, V)
    for s, H, am, c, mk, n in traj:
        assert np.all(mk <= prev_mask)                                   # never re-masked
        kept = prev_mask == 0
        assert np.all(c[kept] == prev_canvas[kept])                      # committed stay put
        new = (prev_mask == 1) & (mk == 0)
        assert np.all(c[new] == am[new])                                 # commits take argmax
        assert mk.sum() <= C * (s - 1) // T                              # masked <= C(s-1)/T
        order = sorted(np.nonzero(prev_mask)[0], key=lambda i: (H[i], i))
        assert set(order[:n]) == set(np.nonzero(new)[0])                 # a sorted prefix
        prev_mask, prev_canvas = mk, c
    assert not (canvas == V).any() and len(traj) <= T


# --------------------------------------------------------------- absorbing process
def test_absorbing_example_endpoints():
    g = json.load(open(os.path.join(GOLDEN, "absorbing_example.json")))
    u = gen.uniform_u16(0, "absorb.example", len(g["sentence"])).numpy()
    x0, _ = absorbing.absorb(g["sentence"], 0, g["T"], g["vocab"], u)
    xT, _ = absorbing.absorb(g["sentence"], g["T"], g["T"], g["vocab"], u)
    assert list(x0) == g["at_t0"] and list(xT) == g["at_tT"]


def test_absorbing_fraction_and_monotone():
    n, T = 200000, 10
    u = gen.uniform_u16(3, "absorb.frac", n).numpy()
    prev = np.zeros(n, bool)
    for t in range(T + 1):
        _, a = absorbing.absorb(np.zeros(n, np.int64), t, T, 99, u)
        p = t / T
        assert abs(a.mean() - p) <= 4 * math.sqrt(p * (1 - p) / n) + 1e-12
        assert np.all(a >= prev)
        prev = a


# --------------------------------------------------------------- masks and composition
def _tiny(**kw):
    return model.Weights(workloads.TINY_F32.with_(**kw), keep_layers=True)


def test_prefill_causal_and_window():
    P = 12
    base = np.arange(P) * 7 % 500
    ws = _tiny()                                       # window 1024: all P rows are kept
    kv = model.prefill(ws, base)
    for j in (5, 9):
        alt = base.copy()
        alt[j] = (alt[j] + 1) % 500
        kv2 = model.prefill(ws, alt)
        K1, K2 = kv[1][0], kv2[1][0]                  # layer 1 keys
        assert np.array_equal(K1[:j], K2[:j])          # causal: earlier rows unchanged
        assert not np.allclose(K1[j:j + 2], K2[j:j + 2])
    # window 4: the cache keeps positions 8..11; layer-1 row i depends on tokens i-3 .. i
    ws4 = _tiny(window=4)
    kv = model.prefill(ws4, base)
    assert kv[1][0].shape[0] == 4
    alt = base.copy()
    alt[4] = (alt[4] + 1) % 500
    assert np.array_equal(kv[1][0], model.prefill(ws4, alt)[1][0])
    alt = base.copy()
    alt[7] = (alt[7] + 1) % 500
    K2 = model.prefill(ws4, alt)[1][0]
    assert np.array_equal(kv[1][0][3], K2[3])          # position 11 is 4 away from 7
    assert not np.allclose(kv[1][0][:3], K2[:3])


def test_canvas_is_bidirectional():
    ws = _tiny()
    w = ws.w
    prompt = np.arange(w.prompt_len) % w.vocab
    kv = model.prefill(ws, prompt)
    c = np.full(w.canvas, w.mask_id)
    a = model.denoise_forward(ws, kv, c, 3, w.T, w.prompt_len)["H64"]
    c2 = c.copy()
    c2[20] = 5
    b = model.denoise_forward(ws, kv, c2, 3, w.T, w.prompt_len)["H64"]
    assert np.all(a[:20] != b[:20]) and np.all(a[21:] != b[21:])


def test_zero_blocks_reduce_to_embedding_head():
    """With Wo and all FFN outputs zero every layer is the identity."""
    ws = _tiny()
    w = ws.w
    for l in range(w.n_layers):
        for name, shape in [(f"l{l}.wo", (w.d_model, w.n_q_heads * w.head_dim)),
                            (f"l{l}.sdown", (w.d_model, w.shared_inter)),
                            (f"l{l}.down", (w.n_experts, w.d_model, w.expert_inter))]:
            ws._cache[name] = np.zeros(shape)
    prompt = np.arange(w.prompt_len) % w.vocab
    kv = model.prefill(ws, prompt)
    c = (np.arange(w.canvas) * 3) % (w.vocab + 1)
    st = model.denoise_forward(ws, kv, c, 2, w.T, w.prompt_len, want_logits=True)
    E = ws.get("tok_emb", (w.vocab + 1, w.d_model))
    x = E[c] + model.timestep_embedding(2 / w.T, w.d_model)
    xn = x / np.sqrt((x * x).mean(1, keepdims=True) + w.rms_eps)
    want = w.logit_scale * xn @ ws.get("lm_head", (w.vocab, w.d_model)).T
    np.testing.assert_allclose(st["logits"], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st["H64"], scipy.stats.entropy(scipy.special.softmax(want, 1), axis=1),
                               rtol=1e-11)


# --------------------------------------------------------------- layer composition
class _FixedWeights(model.Weights):
    """Weights whose tensors are given (constructed by hand), not drawn from the seed."""

    def __init__(self, w, tensors):
        super().__init__(w, keep_layers=True)
        self.t = tensors

    def get(self, name, shape):
        assert self.t[name].shape == tuple(shape), name
        return self.t[name]

    def rows(self, name, shape, start_row, n_rows):
        return self.t[name][start_row:start_row + n_rows]


def _composition_weights(swap_kv=False):
    """d = 8, four query heads over two key/value heads (h = 2), one layer.

    Query and router weights are zero, so every attention score is 0 (uniform
    attention: the mean of V over the allowed keys) and the router ties; the key
    rows are non-zero and differ from the value rows, so a q | k | v split that
    read the key rows as values would change the output.  Values: head 0 = xn[0:2],
    head 1 = xn[2:4]; Wo = I; routed experts zero; shared expert with gate = up =
    down = I, so it adds silu(u) * u for u = RMSNorm(x) after attention."""
    w = workloads.TINY_F32.with_(name="composition", n_layers=1, d_model=8, n_q_heads=4,
                                 n_kv_heads=2, head_dim=2, n_experts=2, top_k=1,
                                 expert_inter=4, shared_inter=8, vocab=16)
    wq = np.zeros((8, 8))
    wk = np.zeros((4, 8))
    wk[:, 4:8] = 2.0 * np.eye(4)
    wv = np.zeros((4, 8))
    wv[:, 0:4] = np.eye(4)
    if swap_kv:
        wk, wv = wv, wk
    t = {"l0.wqkv": np.concatenate([wq, wk, wv]), "l0.wo": np.eye(8),
         "l0.router": np.zeros((2, 8)), "l0.gate": np.zeros((2, 4, 8)),
         "l0.up": np.zeros((2, 4, 8)), "l0.down": np.zeros((2, 8, 4)),
         "l0.sgate": np.eye(8), "l0.sup": np.eye(8), "l0.sdown": np.eye(8)}
    return _FixedWeights(w, t)


def _composition_expected(x, keys_xn, eps):
    """Closed form of the constructed layer: pre-norm attention (mean of the value
    heads over the keys, query heads 0, 1 -> kv head 0 and 2, 3 -> kv head 1), then
    pre-norm shared expert silu(u) * u, each added to the residual."""
    v0 = keys_xn[:, 0:2].mean(axis=0)
    v1 = keys_xn[:, 2:4].mean(axis=0)
    x1 = x + np.concatenate([v0, v0, v1, v1])[None, :]
    u = x1 / np.sqrt((x1 * x1).mean(axis=1, keepdims=True) + eps)
    return x1 + u * u / (1.0 + np.exp(-u))


def _composition_rows():
    # rows whose RMS is far from 1 (so a missing or misplaced norm shows)
    return np.array([[3.0, -1.0, 0.5, 2.0, -4.0, 1.5, 0.25, -2.5],
                     [0.1, 0.4, -0.3, 0.2, 0.05, -0.6, 0.7, -0.15],
                     [-7.0, 2.0, 9.0, -1.0, 4.0, 3.0, -5.0, 6.0]])


def test_decoder_layer_composition_closed_form():
    """Pre-norm residual order, values from the normalised rows, the q | k | v row split
    and the grouped-query head map, against a closed form (all rows see all rows)."""
    ws = _composition_weights()
    w = ws.w
    x = _composition_rows()
    xn = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + w.rms_eps)
    empty = np.zeros((0, 2, 2))
    out, k, v, _ = model.decoder_layer(x, np.arange(3), ws.layer(0), (empty, empty),
                                       np.ones((3, 3), dtype=bool), w)
    np.testing.assert_allclose(out, _composition_expected(x, xn, w.rms_eps), rtol=1e-12,
                               atol=1e-12)
    np.testing.assert_allclose(v.reshape(3, 4), xn[:, 0:4], rtol=1e-12, atol=1e-12)
    # variants a reading error would produce all differ from the constructed layer:
    # values read from the key rows, a post-norm block, values from the raw rows
    out_swap = model.decoder_layer(x, np.arange(3), _composition_weights(swap_kv=True).layer(0),
                                   (empty, empty), np.ones((3, 3), dtype=bool), w)[0]
    assert np.abs(out_swap - out).max() > 0.1
    x1 = x + np.concatenate([xn[:, 0:2].mean(0)] * 2 + [xn[:, 2:4].mean(0)] * 2)
    post = x1 / np.sqrt((x1 * x1).mean(1, keepdims=True) + w.rms_eps)
    assert np.abs(_composition_expected(post, post, w.rms_eps) - out).max() > 0.1
    assert np.abs(_composition_expected(x, x, w.rms_eps) - out).max() > 0.1


def test_canvas_layer_one_softmax_over_window_and_canvas():
    """Canvas rows attend to the cached window and every canvas row in ONE softmax: with
    zero scores the value is the mean over all 2 + 3 keys (separate softmaxes over the
    window and the canvas would average the two means instead)."""
    ws = _composition_weights()
    w = ws.w
    x = _composition_rows()
    xn = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + w.rms_eps)
    win_v = np.array([[[5.0, -3.0], [1.0, 8.0]], [[9.0, 1.0], [-6.0, 4.0]]])  # [W 2, Hkv 2, h 2]
    win_k = np.ones_like(win_v)
    out = model.canvas_layer(x, ws.layer(0), (win_k, win_v), 40, w)[0]
    keys = np.concatenate([win_v.reshape(2, 4), xn[:, 0:4]])
    np.testing.assert_allclose(out, _composition_expected(x, keys, w.rms_eps), rtol=1e-12,
                               atol=1e-12)
    two = 0.5 * (win_v.reshape(2, 4).mean(0) + xn[:, 0:4].mean(0))
    x1 = x + np.concatenate([two[0:2], two[0:2], two[2:4], two[2:4]])
    u = x1 / np.sqrt((x1 * x1).mean(1, keepdims=True) + w.rms_eps)
    assert np.abs(x1 + u * u / (1 + np.exp(-u)) - out).max() > 0.1


# --------------------------------------------------------------- metric formulas (pages' numbers)
def test_tps_formula_reproduces_pages():
    from masked_discrete_diffusion_b200 import metrics
    g = json.load(open(os.path.join(GOLDEN, "tps_h100_fp8.json")))
    tps = metrics.tokens_per_second(g["tpf"], g["t_fwd_ms"] / 1000.0)
    assert round(tps) == g["tps_reported"]
    # tokens per forward counts one extra forward between consecutive canvases
    assert metrics.tokens_per_forward([256, 256, 100], [12, 12, 5]) == 612 / (29 + 2)
    assert metrics.effective_steps([256, 100], [12, 4]) == (256 * 12 + 100 * 4) / 356


# --------------------------------------------------------------- entropy gain and bf16 storage
def test_entropy_sigma_two_point_and_first_order_gain():
    """sigma = std of the logits under p: two-point closed form |a - b| sqrt(p (1 - p)),
    zero for equal logits; and the entropy's first-order change is -Cov_p(l, dl)."""
    a, b = 1.7, -0.4
    st = model.entropy_stats(np.array([[a, b], [0.3, 0.3]]))
    p = 1.0 / (1.0 + math.exp(b - a))
    assert st["sigma"][0] == pytest.approx(abs(a - b) * math.sqrt(p * (1 - p)), rel=1e-12)
    assert st["sigma"][1] == pytest.approx(0.0, abs=1e-15)
    r = np.random.default_rng(5)
    lg = r.normal(0, 3, (4, 300))
    d = r.normal(0, 1, (4, 300))
    delta = 1e-6
    h0 = model.entropy_stats(lg)["H64"]
    h1 = model.entropy_stats(lg + delta * d)["H64"]
    p = scipy.special.softmax(lg, axis=1)
    cov = (p * lg * d).sum(1) - (p * lg).sum(1) * (p * d).sum(1)
    np.testing.assert_allclose((h1 - h0) / delta, -cov, rtol=1e-4, atol=1e-8)
    sig = model.entropy_stats(lg)["sigma"]
    assert np.all(np.abs(cov) <= sig * np.abs(d).max(1) * (1 + 1e-12))


def test_round_bf16_ties_and_library():
    """8 significant bits, ties to even; equals torch's fp32 -> bf16 rounding on fp32 values."""
    import torch
    f = model.round_bf16
    assert f(np.array([1 + 2.0 ** -8]))[0] == 1.0                      # tie -> even (1.0)
    assert f(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6        # tie -> even (up)
    assert f(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1 + 2.0 ** -7
    assert f(np.array([-3.0, 0.0, 255.5]))[:2].tolist() == [-3.0, 0.0]
    assert f(np.array([255.5]))[0] == 256.0                            # carry into the exponent
    x = np.random.default_rng(9).normal(0, 10, 20000).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(f(x.astype(np.float64)), ref)


def test_bf16_storage_variant():
    """storage="fp64" is the oracle itself; storage="bf16" keeps the cache keys/values
    and entropies within bf16 distance of it, with every cached value bf16-exact."""
    w = workloads.TINY_F32
    prompt = np.arange(w.prompt_len) % w.vocab
    c = np.full(w.canvas, w.mask_id)
    ref = model.Weights(w, keep_layers=True)
    same = model.Weights(w, keep_layers=True, storage="fp64")
    s16 = model.Weights(w, keep_layers=True, storage="bf16")
    kv_ref, kv_same, kv_16 = model.prefill(ref, prompt), model.prefill(same, prompt), model.prefill(s16, prompt)
    for (k0, v0), (k1, v1), (k2, v2) in zip(kv_ref, kv_same, kv_16):
        assert np.array_equal(k0, k1) and np.array_equal(v0, v1)
        assert np.array_equal(model.round_bf16(k2), k2) and np.array_equal(model.round_bf16(v2), v2)
        assert not np.array_equal(k0, k2)
        assert np.abs(k2 - k0).max() <= 2.0 ** -6 * np.abs(k0).max()
    h0 = model.denoise_forward(ref, kv_ref, c, w.T, w.T, w.prompt_len)["H64"]
    h2 = model.denoise_forward(s16, kv_16, c, w.T, w.T, w.prompt_len)["H64"]
    assert 0 < np.abs(h2 - h0).max() < 2e-2 * np.abs(h0).max()
    with pytest.raises(ValueError):
        model.Weights(w, storage="fp16")


def test_bf16_storage_rounds_dequantised_fp8_weights():
    """In the storage variant FP8 expert weights enter as bf16 values (code * scale
    rounded); the fp64 oracle keeps code * scale exactly."""
    w = workloads.SMALL_FP8
    exact = model.Weights(w, keep_layers=True).layer(0).expert(1)[0]
    s16 = model.Weights(w, keep_layers=True, storage="bf16").layer(0).expert(1)[0]
    assert np.array_equal(model.round_bf16(exact), s16)
    assert not np.array_equal(exact, s16)
    assert np.all(np.abs(s16 - exact) <= 2.0 ** -8 * np.abs(exact))   # unit roundoff, 8 bits
