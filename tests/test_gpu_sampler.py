"""EB sampler kernel vs the oracle sampler, bit-exact, on seeded synthetic statistics.

Both sides receive the same fp32 entropies, argmax ids, canvases and masks (drawn
by the shared seeded generator); the committed sets, canvases, masks and counts
must be identical.
"""
import numpy as np
import pytest
import torch

from oracle import sampler as osamp
from synth import gen

pytestmark = pytest.mark.gpu


def _case(seed, B, C, tie_levels=None, special=False):
    u = gen.uniform_u16(seed, "sampler.case", 4 * B * C).numpy().reshape(4, B, C)
    H = (u[0] / 65536.0 * 3.0).astype(np.float32)
    if tie_levels:
        H = (np.floor(H * tie_levels) / tie_levels).astype(np.float32)
    if special:
        H[:, ::7] = 0.0
        H[:, 3::11] = -0.25
        H[:, 5::13] = np.nan
        H[:, 6::17] = np.inf
    am = (u[1] % 1000).astype(np.int32)
    mask = (u[2] % 10 < 7).astype(np.uint8)
    canvas = np.where(mask == 1, 1000, u[3] % 1000).astype(np.int32)
    return H, am, canvas, mask


@pytest.mark.parametrize("B,C", [(1, 1), (1, 32), (3, 256), (2, 200), (1, 1024), (4, 33)])
@pytest.mark.parametrize("s,gamma", [(1, 1.0), (4, 1.0), (12, 0.0), (3, 2.5), (2, float("inf"))])
@pytest.mark.parametrize("kind", ["plain", "ties", "special"])
def test_sampler_bit_exact(B, C, s, gamma, kind):
    from masked_discrete_diffusion_b200 import binding
    H, am, canvas, mask = _case(B * 1000 + C + s, B, C, tie_levels=4 if kind == "ties" else None,
                                special=kind == "special")
    dH = torch.from_numpy(H).cuda()
    dA = torch.from_numpy(am).cuda()
    dC = torch.from_numpy(canvas).cuda()
    dM = torch.from_numpy(mask).cuda()
    n = binding.dg_eb_sample(dH, dA, dC, dM, s, gamma)
    torch.cuda.synchronize()
    for b in range(B):
        c2, m2, n2, _ = osamp.eb_step(H[b], am[b], canvas[b], mask[b], s, gamma)
        assert int(n[b]) == n2
        assert np.array_equal(dC[b].cpu().numpy(), c2)
        assert np.array_equal(dM[b].cpu().numpy(), m2)


def test_sampler_nothing_masked_is_noop():
    from masked_discrete_diffusion_b200 import binding
    H, am, canvas, _ = _case(5, 2, 64)
    mask = np.zeros_like(canvas, dtype=np.uint8)
    dC = torch.from_numpy(canvas).cuda()
    n = binding.dg_eb_sample(torch.from_numpy(H).cuda(), torch.from_numpy(am).cuda(), dC,
                             torch.from_numpy(mask).cuda(), 3, 1.0)
    assert n.cpu().tolist() == [0, 0] and np.array_equal(dC.cpu().numpy(), canvas)


@pytest.mark.parametrize("C,s", [(1024, 64), (512, 8), (1024, 1)])
def test_sampler_saturated_prefix_sums(C, s):
    """Every position masked with a NaN entropy (fixed point 2^54 each) and gamma = inf
    (bound 2^62): the prefix sums pass 2^63 past position 511; the count within the bound
    must still be exactly 256 (the oracle's unbounded integers)."""
    from masked_discrete_diffusion_b200 import binding
    H = np.full((1, C), np.nan, np.float32)
    am = (np.arange(C, dtype=np.int32) * 7 % 1000).reshape(1, C)
    canvas = np.full((1, C), 1000, np.int32)
    mask = np.ones((1, C), np.uint8)
    dC = torch.from_numpy(canvas).cuda()
    dM = torch.from_numpy(mask).cuda()
    n = binding.dg_eb_sample(torch.from_numpy(H).cuda(), torch.from_numpy(am).cuda(), dC, dM, s,
                             float("inf"))
    c2, m2, n2, kg = osamp.eb_step(H[0], am[0], canvas[0], mask[0], s, float("inf"))
    assert kg == 256
    assert int(n[0]) == n2 == max(256, -(-C // s))
    assert np.array_equal(dC[0].cpu().numpy(), c2) and np.array_equal(dM[0].cpu().numpy(), m2)
