"""Pins of the NVFP4 weight format (synth/nvfp4.py) against definitions written
independently of it: the E2M1 bit fields, brute-force nearest rounding, the error
bound of the two-level scaling, the nibble order and the tensor-scale rule."""
import math

import numpy as np
import torch

from synth import fp8, nvfp4, workloads


def _e2m1_from_bits(c: int) -> float:
    """E2M1 from its fields: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
    exponent 0 is subnormal (m * 2^-1), else (1 + m / 2) * 2^(e - 1)."""
    s, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_decode_matches_the_bit_fields():
    codes = torch.arange(16, dtype=torch.uint8)
    got = nvfp4.e2m1_decode(codes).tolist()
    want = [_e2m1_from_bits(c) for c in range(16)]
    assert got == want
    assert sorted({abs(v) for v in want}) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_encode_decode_round_trip():
    for c in list(range(8)) + list(range(9, 16)):  # code 8 is -0
        v = torch.tensor([_e2m1_from_bits(c)], dtype=torch.float64)
        assert int(nvfp4.e2m1_encode(v)[0]) == c


def test_rounding_is_nearest_with_ties_to_even_and_saturates():
    grid = np.array(sorted({_e2m1_from_bits(c) for c in range(16)}))
    rng = np.random.default_rng(7)
    x = rng.uniform(-7.5, 7.5, 20000)
    r = nvfp4.e2m1_round(torch.from_numpy(x)).numpy()
    d = np.abs(x[:, None] - grid[None, :])
    nearest = grid[d.argmin(axis=1)]
    tie = np.sort(d, axis=1)[:, 1] - np.sort(d, axis=1)[:, 0] < 1e-12
    assert np.array_equal(r[~tie], nearest[~tie])
    # midpoints go to the neighbour whose mantissa bit is 0
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, -5.0], dtype=torch.float64)
    assert nvfp4.e2m1_round(mids).tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -1.0, -4.0]
    assert nvfp4.e2m1_round(torch.tensor([6.9, -100.0], dtype=torch.float64)).tolist() == [6.0, -6.0]


def test_tensor_scale_rule():
    for sigma in (0.02, 0.003, 1.0, 4.0):
        s_t = nvfp4.tensor_scale(sigma)
        assert math.log2(s_t) == int(math.log2(s_t))
        assert 6 * 448 * s_t >= 8 * sigma > 6 * 448 * s_t / 2


def test_quantize_rows_scales_codes_and_error_bound():
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(6, 64, generator=g, dtype=torch.float64) * 0.02)
    w[0, :16] = 0.0                              # an all-zero block
    w[1, 0], w[1, 1] = 1e-9, -2e-9               # tiny values next to normal ones
    s_t = nvfp4.tensor_scale(0.02)
    packed, sb = nvfp4.quantize_rows(w, s_t)
    assert packed.shape == (6, 32) and sb.shape == (6, 4)
    blocks = w.reshape(6, 4, 16)
    want_sb = fp8.e4m3_round(blocks.abs().amax(dim=2) / (6 * s_t))
    want_sb = torch.where(want_sb > 0, want_sb, torch.full_like(want_sb, 2.0 ** -9))
    assert torch.equal(fp8.e4m3_decode(sb), want_sb)
    codes = nvfp4.unpack(packed)
    deq = (nvfp4.e2m1_decode(codes).reshape(6, 4, 16) * want_sb[..., None] * s_t)
    # each value is within half of its E2M1 quantum (times the block's scales) unless it
    # saturated at 6 because the block scale rounded down
    x = blocks / (want_sb[..., None] * s_t)
    ex = torch.frexp(x.abs().clamp(max=6.0))[1]
    quantum = torch.ldexp(torch.ones_like(x), (ex - 1).clamp(min=0) - 1)
    err = (deq - blocks).abs() / (want_sb[..., None] * s_t)
    sat = x.abs() > 6.0
    assert torch.all(err[~sat] <= quantum[~sat] / 2 + 1e-12)
    assert torch.all(deq[0, 0] == 0.0)


def test_nibble_order():
    s_t = 1.0
    w = torch.zeros(1, 32, dtype=torch.float64)
    w[0, 0], w[0, 1] = 1.0 * 448 / 448, 6.0      # block amax 6 -> s_b = 1
    w[0, 16] = 6.0
    packed, sb = nvfp4.quantize_rows(w, s_t)
    assert fp8.e4m3_decode(sb)[0, 0] == 1.0
    assert int(packed[0, 0]) == (7 << 4) | 2     # element 0 (1.0, code 2) in the low nibble


def test_dequantised_matches_the_stored_format():
    w = workloads.SMALL_FP4
    shape = (w.n_experts, w.expert_inter, w.d_model)
    q, s, st = nvfp4.quantised(w, "l0.gate", shape, w.init_std)
    deq = nvfp4.dequantised(w, "l0.gate", shape, w.init_std, start_row=2, n_rows=3)
    R, K = 3 * w.expert_inter, w.d_model
    codes = nvfp4.unpack(q[2:5].reshape(R, K // 2))
    vals = (nvfp4.e2m1_decode(codes).reshape(R, K // 16, 16)
            * fp8.e4m3_decode(s[2:5].reshape(R, K // 16))[..., None] * float(st[0]))
    assert np.array_equal(deq, vals.reshape(3, w.expert_inter, K).numpy())
    # the represented weights stay close to the drawn normal values
    ref = torch.from_numpy(deq).to(torch.float64)
    assert float(ref.abs().max()) < 6 * w.init_std
