"""Pins of oracle/anneal.py (the Report's default sampler) against values the
definitions fix: published generator outputs, closed-form moments and
distributions, brute force of the mutual-information bound, and fake forwards whose
whole trajectory is known in advance."""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import anneal as an


# --- SplitMix64 ------------------------------------------------------------------------
def test_splitmix64_published_outputs():
    # first outputs of SplitMix64 seeded with 0 (Steele, Lea and Flood's generator as
    # used to seed the xorshift/xoshiro family)
    got = [int(x) for x in an.splitmix_outputs(0, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_form_is_the_sequential_generator():
    for key in (0, 1, 0xDEADBEEF, (1 << 64) - 1):
        seq = an.splitmix_outputs(key, 40)
        assert np.array_equal(an.draw(key, np.arange(40)), seq)


def test_stream_keys_are_generator_outputs():
    seed = 987654321
    seq = an.splitmix_outputs(seed, 3)
    assert [an.stream_key(seed, j) for j in (1, 2, 3)] == [int(x) for x in seq]


def test_token_draw_range_ends_and_uniformity():
    V = 10
    top = np.array([0xFFFFFFFF << 32], dtype=np.uint64)
    assert an.token_from_bits(np.array([0], dtype=np.uint64), V)[0] == 0
    assert an.token_from_bits(top, V)[0] == V - 1
    z = an.draw(an.stream_key(7, 1), np.arange(200_000))
    t = an.token_from_bits(z, V)
    assert t.min() == 0 and t.max() == V - 1
    counts = np.bincount(t, minlength=V)
    chi2 = ((counts - 20_000) ** 2 / 20_000).sum()
    assert chi2 < 40.0                      # 9 degrees of freedom; p ~ 5e-6


def test_gumbel_moments():
    # Gumbel(0, 1): mean = Euler-Mascheroni constant, variance = pi^2 / 6, for the even
    # and the odd field alike, and the two fields of one output uncorrelated
    z = an.draw(an.stream_key(3, 2), np.arange(400_000))
    f = an.fields_of_bits(z)
    for h in (0, 1):
        g = an.gumbel_from_field(f[:, h])
        assert np.isfinite(g).all()
        assert abs(g.mean() - 0.5772156649015329) < 0.01
        assert abs(g.var() - math.pi ** 2 / 6) < 0.03
    assert abs(np.corrcoef(f[:, 0], f[:, 1])[0, 1]) < 0.01
    # u stays strictly inside (0, 1): the extreme codes give finite noise
    ext = an.gumbel_from_field(np.array([0, (1 << 23) - 1]))
    assert np.isfinite(ext).all() and ext[0] < ext[1]


def test_fields_are_the_stated_bits():
    z = np.array([(0b1011 << 60) | (0x7FFFFF << 41) | (0x1234 << 9) | 0x1FF], dtype=np.uint64)
    f = an.fields_of_bits(z)[0]
    assert int(f[0]) == ((0b1011 << 60) | (0x7FFFFF << 41)) >> 41
    assert int(f[1]) == 0x1234
    # odd vocabulary: the last token takes the even field of its own output
    g = an.gumbel_row(4, 1, 2, 3, 5)
    zz = an.draw(an.stream_key(4, 2), [(1 * 3 + 2) * 3 + 2])
    assert g[4] == an.gumbel_from_field(an.fields_of_bits(zz)[:, 0])[0]


# --- temperature, tempered statistics, Gumbel-max ---------------------------------------
def test_temperature_schedule():
    p = an.Params()
    assert an.temperature(0, p) == float(np.float32(0.8))           # t = 1
    assert abs(an.temperature(24, p) - 0.6) < 1e-7                  # t = 1/2
    assert abs(an.temperature(47, p) - (0.4 + 0.4 / 48)) < 1e-7      # t = 1/N
    taus = [an.temperature(k, p) for k in range(48)]
    steps = np.diff(taus)
    assert np.allclose(steps, steps[0]) and steps[0] < 0             # linear, decreasing
    assert [an.step_time(k, 48) for k in (0, 47)] == [1.0, 1.0 / 48]


def test_tempered_entropy_closed_forms():
    V = 7
    H = an.tempered_stats(np.zeros((1, V)), 0.3)["H64"][0]
    assert abs(H - math.log(V)) < 1e-12
    l = np.array([[1.3, -0.4]])
    for tau in (0.4, 0.8, 2.0):
        p = 1.0 / (1.0 + math.exp(-(1.3 + 0.4) / tau))
        ref = -p * math.log(p) - (1 - p) * math.log(1 - p)
        assert abs(an.tempered_stats(l, tau)["H64"][0] - ref) < 1e-14
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 50)) * 3
    a, b = an.tempered_stats(x, 0.5), an.tempered_stats(x / 0.5, 1.0)
    assert np.allclose(a["H64"], b["H64"], rtol=1e-13) and np.array_equal(a["argmax"], b["argmax"])
    assert (np.diff([an.tempered_stats(x, t)["H64"][0] for t in (0.2, 0.4, 0.8)]) > 0).all()


def test_gumbel_max_draws_follow_the_tempered_softmax():
    l = np.array([0.0, 1.0, -0.5, 2.0, 0.3, -2.0])
    tau, n = 0.7, 30_000
    p = np.exp(l / tau) / np.exp(l / tau).sum()
    counts = np.zeros(len(l))
    key = an.stream_key(11, 2)
    z = an.draw(key, np.arange(n * len(l) // 2))
    g = an.gumbel_from_field(an.fields_of_bits(z).reshape(n, len(l)))
    for r in range(n):
        counts[an.gumbel_max(l / tau, g[r])[0]] += 1
    sd = np.sqrt(n * p * (1 - p))
    assert (np.abs(counts - n * p) < 4.5 * sd).all()


def test_gumbel_max_low_temperature_is_the_argmax_and_ties_take_the_lowest_id():
    l = np.array([0.1, 0.9, 0.5])
    g = an.gumbel_row(5, 0, 0, 1, 3)
    assert an.gumbel_max(l / 1e-4, g)[0] == 1
    assert an.gumbel_max(np.zeros(4), np.zeros(4)) == (0, 0.0)


def test_sample_tokens_uses_the_per_position_stream():
    C, V, seed, k = 3, 20, 99, 5
    rng = np.random.default_rng(1)
    logits = rng.normal(size=(C, V))
    tok, gap = an.sample_tokens(logits, 0.6, seed, k)
    for i in range(C):
        y = logits[i] / 0.6 + an.gumbel_row(seed, k, i, C, V)
        assert tok[i] == int(np.argmax(y))
        s = np.sort(y)
        assert abs(gap[i] - (s[-1] - s[-2])) < 1e-12


# --- the mutual-information bound, re-noising, the stop test ----------------------------
def _accept_brute(H, b):
    """Longest prefix of the ascending (entropy, position) order with
    sum - max <= b, in exact rational arithmetic (at least one position)."""
    keys = sorted(range(len(H)), key=lambda i: (float(np.float32(H[i])), i))
    vals = [Fraction(float(np.float32(H[i]))) for i in keys]
    bb = Fraction(float(np.float32(b)))
    best = 0
    for n in range(1, len(H) + 1):
        pre = vals[:n]
        if sum(pre) - max(pre) <= bb:
            best = n
    return best


def test_mi_bound_example_where_the_largest_entropy_does_not_count():
    # 0.04 + 0.05 + 0.2 - 0.2 = 0.09 <= 0.1: all three; a plain sum bound would stop at 2
    assert an.accepted_count([0.05, 0.04, 0.2], 0.1) == 3
    assert an.accepted_count([0.05, 0.06, 0.2], 0.1) == 2          # 0.05 + 0.06 > 0.1
    assert an.accepted_count([5.0, 7.0], 0.1) == 1                 # the first always goes
    assert an.accepted_count(np.zeros(9), 0.1) == 9
    assert an.accepted_count([np.nan, 0.0, 0.01], 0.1) == 3          # NaN sorts last
    assert an.accepted_count([np.nan, 0.0, 0.2], 0.1) == 2
    assert an.accepted_count([0.3, 0.2, 0.1], 0.0) == 1
    assert an.accepted_count([0.0, 0.0, 0.1], 0.0) == 3


def test_mi_bound_matches_brute_force():
    rng = np.random.default_rng(2)
    for trial in range(300):
        C = int(rng.integers(1, 40))
        H = rng.exponential(0.02 if trial % 2 else 0.5, size=C).astype(np.float32)
        b = float(rng.choice([0.0, 0.05, 0.1, 0.3, 2.0]))
        # skip draws that sit within the fixed-point resolution of the bound
        srt = np.sort(H.astype(np.float64))
        if np.min(np.abs(np.cumsum(srt) - b)) < 1e-9:
            continue
        assert an.accepted_count(H, b) == _accept_brute(H, b)


def test_refine_keeps_the_prefix_and_renoises_the_rest():
    C, V, seed, k, b = 12, 50, 4, 3, 0.1
    H = np.array([0.5, 0.01, 0.02, 0.9, 0.03, 0.0, 0.07, 0.3, 0.2, 1.0, 0.045, 0.6], np.float32)
    sampled = np.arange(100, 100 + C)
    out, n = an.refine(H, sampled, seed, k, V, b)
    # ascending: 0.0 (5), 0.01 (1), 0.02 (2), 0.03 (4), 0.045 (10), 0.07 (6) ...
    # prefix of 5: 0.105 - 0.045 = 0.06 <= 0.1; prefix of 6: 0.175 - 0.07 = 0.105 > 0.1
    assert n == 5 == _accept_brute(H, b)
    acc = sorted(range(C), key=lambda i: (float(H[i]), i))[:n]
    noise = an.renoise_tokens(seed, k, C, V)
    for i in range(C):
        assert out[i] == (sampled[i] if i in acc else noise[i])
    assert ((noise >= 0) & (noise < V)).all()


def test_stop_test_cases():
    H_low = np.full(8, 0.004, np.float32)
    H_high = np.full(8, 0.006, np.float32)
    a = np.arange(8)
    assert an.stop_test(H_low, a, a.copy(), 0.005)
    assert not an.stop_test(H_low, a, None, 0.005)                 # first step
    assert not an.stop_test(H_high, a, a.copy(), 0.005)            # mean too high
    b = a.copy()
    b[3] += 1
    assert not an.stop_test(H_low, a, b, 0.005)                    # argmax changed
    mixed = np.array([0.0] * 7 + [0.039], np.float32)              # mean 0.004875
    assert an.stop_test(mixed, a, a.copy(), 0.005)
    mixed[7] = 0.041                                               # mean 0.005125
    assert not an.stop_test(mixed, a, a.copy(), 0.005)
    inf = np.array([np.inf] * 8, np.float32)
    assert not an.stop_test(inf, a, a.copy(), 16.0)
    with pytest.raises(ValueError):
        an.stop_test(H_low, a, a, 17.0)


# --- whole canvases with fake forwards --------------------------------------------------
def test_peaked_forward_converges_in_two_steps():
    C, V, seed = 16, 40, 21
    target = (np.arange(C) * 7 + 3) % V
    seen = []

    def forward(canvas, k):
        seen.append((k, canvas.copy()))
        l = np.zeros((C, V))
        l[np.arange(C), target] = 1e4
        return l

    p = an.Params()
    out, traj = an.generate_block(forward, C, V, seed, p)
    assert np.array_equal(out, target) and len(traj) == 2
    assert np.array_equal(seen[0][1], an.initial_canvas(seed, C, V))
    # step 0: every entropy is 0, so all positions are accepted with their drawn tokens
    assert traj[0]["n_accepted"] == C and not traj[0]["stop"]
    assert np.array_equal(traj[0]["sampled"], target)
    assert np.array_equal(seen[1][1], target)
    assert traj[1]["stop"] and [e["k"] for e in traj] == [0, 1]


def test_flat_forward_runs_all_steps_and_returns_the_last_argmax():
    C, V, seed = 6, 9, 5
    p = an.Params(N=7)
    out, traj = an.generate_block(lambda canvas, k: np.zeros((C, V)), C, V, seed, p)
    assert len(traj) == 7 and not any(e["stop"] for e in traj)
    assert np.array_equal(out, np.zeros(C))                       # ties -> lowest id
    for e in traj[:-1]:
        assert e["n_accepted"] == 1                               # log 9 > b
        H = e["H64"]
        assert np.allclose(H, math.log(V))
        # the accepted position (all entropies equal: position 0) keeps its draw
        noise = an.renoise_tokens(seed, e["k"], C, V)
        assert e["canvas"][0] == e["sampled"][0]
        assert np.array_equal(e["canvas"][1:], noise[1:])
    assert traj[-1]["n_accepted"] == C


def test_canvas_dependent_argmax_never_stops():
    C, V = 5, 11

    def forward(canvas, k):
        l = np.full((C, V), -50.0)
        l[np.arange(C), (canvas + 1) % V] = 50.0                 # H ~ 0, argmax moves
        return l

    out, traj = an.generate_block(forward, C, V, 8, an.Params(N=6))
    assert len(traj) == 6
    for prev, cur in zip(traj, traj[1:]):
        assert np.array_equal(cur["argmax"], (prev["canvas"] + 1) % V)


def test_model_level_block_is_consistent_with_its_steps():
    from oracle import model as om
    from synth import model_inputs, workloads
    w = workloads.TINY_F32
    ws = om.Weights(w, keep_layers=True)
    prompt = model_inputs.prompt(w, "cpu")[0].numpy()
    p = an.Params(tau_max=0.02, tau_min=0.02)
    out, traj = om.generate_block_annealed(ws, prompt, 1, p)
    assert traj[-1]["stop"] and len(traj) < p.N
    assert np.array_equal(out, traj[-1]["argmax"])
    prev = None
    for e in traj:
        assert an.stop_test(e["H"], e["argmax"], prev, p.e_stop) == e["stop"]
        if not e["stop"]:
            c, n = an.refine(e["H"], e["sampled"], 1, e["k"], w.vocab, p.b)
            assert np.array_equal(c, e["canvas"]) and n == e["n_accepted"]
        prev = e["argmax"]
