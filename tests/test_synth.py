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


def test_e4m3_codes_roundtrip_and_rounding():
    from synth import fp8
    codes = torch.arange(256, dtype=torch.uint8)
    finite = codes[(codes & 0x7F) != 0x7F]
    vals = fp8.e4m3_decode(finite)
    # every finite code decodes to a value that encodes back to itself (0x80 is -0)
    back = fp8.e4m3_encode(vals)
    keep = finite != 0x80
    assert torch.equal(back[keep], finite[keep])
    assert float(vals.max()) == 448.0 and float(vals[vals > 0].min()) == 2.0 ** -9
    # known points of the format: 1.0 = 0x38, 448 = 0x7E, 2^-6 = 0x08, 2^-9 = 0x01
    for v, c in [(1.0, 0x38), (448.0, 0x7E), (2.0 ** -6, 0x08), (2.0 ** -9, 0x01), (-1.5, 0xBC)]:
        assert int(fp8.e4m3_encode(torch.tensor([v], dtype=torch.float64))[0]) == c
    # rounding is to the nearest representable value, ties to even, saturating
    x = torch.tensor([1.0625, 1.1875, 1.0624, 500.0, -3e-3, 2.0 ** -10], dtype=torch.float64)
    r = fp8.e4m3_round(x)
    assert r.tolist() == [1.0, 1.25, 1.0, 448.0, -2 * 2.0 ** -9, 0.0]
    # brute force: nearest of all finite values
    grid = torch.unique(torch.cat([vals, -vals]))
    xs = torch.linspace(-460, 460, 20001, dtype=torch.float64)
    rr = fp8.e4m3_round(xs)
    d = (xs[:, None] - grid[None, :]).abs()
    assert torch.all((rr - xs).abs() <= d.min(dim=1).values + 1e-12)


def test_fp8_block_scales():
    from synth import fp8
    w = gen.normal_values(4, "fp8test", 0, 4 * 256, 0.02).reshape(4, 256)
    codes, scales = fp8.quantize_rows(w)
    assert scales.shape == (4, 2) and codes.dtype == torch.uint8
    deq = fp8.e4m3_decode(codes).reshape(4, 2, 128) * scales.double()[..., None]
    blk = w.double().reshape(4, 2, 128)
    # the largest element of every block is represented (almost) exactly; error <= 1/16 relative
    assert torch.allclose(deq.abs().amax(2), blk.abs().amax(2), rtol=1e-6)
    assert float(((deq - blk).abs() / blk.abs().amax(2, keepdim=True)).max()) <= 2.0 ** -4
