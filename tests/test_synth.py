"""The seeded generator shared by both sides follows SplitMix64's published definition."""
import numpy as np
import torch

from synth import gen, model_inputs, workloads


def test_splitmix64_published_vector():
    # SplitMix64 (Steele, Lea, Flood 2014) seeded with 1234567: its first five outputs,
    # as printed by the reference implementation's test.
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    s, M = 1234567, (1 << 64) - 1
    got = []
    for _ in range(5):
        s = (s + 0x9E3779B97F4A7C15) & M
        got.append(gen.mix64_int(s))
    assert got == want


def test_tensor_bits_follow_scalar_definition():
    z = gen.raw_bits(5, "l3.gate", 1000, 64)
    key = gen.tensor_key(5, "l3.gate")
    M = (1 << 64) - 1
    want = [gen.mix64_int(key + (1000 + i + 1) * 0x9E3779B97F4A7C15) for i in range(64)]
    assert [v & M for v in z.tolist()] == want


def test_normal_values_moments_and_slices():
    v = gen.normal_values(0, "w", 0, 1 << 20, 0.02)
    assert abs(v.mean().item()) < 1e-4 and abs(v.std().item() - 0.02) < 1e-4
    part = gen.normal_values(0, "w", 12345, 100, 0.02)
    assert torch.equal(part, v[12345:12445])


def test_weight_rows_and_prompt():
    w = workloads.TINY_F32
    full = model_inputs.weight(w, "l0.gate", (8, 128, 64))
    rows = model_inputs.weight(w, "l0.gate", (8, 128, 64), start_row=3, n_rows=2)
    assert torch.equal(full[3:5], rows)
    out = torch.empty(2, 128, 64)
    gen.fill_weight_(out, w.seed, "l0.gate", w.init_std, start_row=3)
    assert torch.equal(out, rows)
    p = model_inputs.prompt(w)
    assert p.shape == (1, 32) and p.dtype == torch.int32
    assert int(p.min()) >= 0 and int(p.max()) < w.vocab
    wb = workloads.LAYER1_BF16
    assert model_inputs.weight(wb, "l0.wo", (4, 2048), n_rows=4).dtype == torch.bfloat16
