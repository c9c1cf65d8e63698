"""Tiny fp32 model (2 layers, d 64, vocab 512, canvas 32, T 4): the whole path vs the oracle.

The CUDA path for fp32 weights carries activations and sums in fp64, so the
entropies agree to ~1e-12 and the committed-token trajectory is compared exactly.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import sampler as osamp
from synth import model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel

pytestmark = pytest.mark.gpu
W = workloads.TINY_F32
TOL = 1e-4  # fp32 bound of the workload; observed error is far below it


@pytest.fixture(scope="module")
def setup():
    from masked_discrete_diffusion_b200 import binding
    model = make_model(W)
    prompt = model_inputs.prompt(W, "cuda")
    kv = binding.dg_prefill(model, prompt)
    ws = om.Weights(W, keep_layers=True)
    okv = om.prefill(ws, prompt[0].cpu().numpy())
    yield binding, model, kv, ws, okv
    kv.close()
    model.close()


def test_prefill_kv_matches_oracle(setup):
    binding, model, kv, ws, okv = setup
    k, v = binding.dg_kv_read(kv)
    binding.dg_sync_status(model)
    for l in range(W.n_layers):
        ok = np.transpose(okv[l][0], (1, 0, 2))   # [Hkv, W, h]
        ovv = np.transpose(okv[l][1], (1, 0, 2))
        assert max_abs_rel(k[l, 0].cpu().numpy(), ok) < 1e-9
        assert max_abs_rel(v[l, 0].cpu().numpy(), ovv) < 1e-9


@pytest.mark.parametrize("s", [4, 1])
def test_forward_logits_entropy_match(setup, s):
    binding, model, kv, ws, okv = setup
    canvas = np.full(W.canvas, W.mask_id)
    canvas[::3] = np.arange(0, W.canvas, 3) * 13 % W.vocab
    dc = torch.from_numpy(canvas.astype(np.int32)).cuda()[None]
    ent, am, lg, hd = binding.dg_debug_forward(model, kv, dc, s, W.T, logits=True, hidden=True)
    binding.dg_sync_status(model)
    st = om.denoise_forward(ws, okv, canvas, s, W.T, W.prompt_len, want_logits=True,
                            want_hidden=True)
    assert max_abs_rel(lg.cpu().numpy(), st["logits"]) < TOL
    assert max_abs_rel(hd.cpu().numpy(), st["hidden"]) < TOL
    H = ent[0].cpu().numpy()
    assert np.all(np.abs(H - st["H"]) <= TOL * np.abs(st["H"]))
    assert np.array_equal(am[0].cpu().numpy(), st["argmax"])
    assert np.all(H >= 0) and np.all(H <= np.log(W.vocab) + 1e-6)


def test_block_trajectory_exact(setup):
    """dg_denoise_step x T from all [MASK] equals the oracle's trajectory step by step."""
    binding, model, kv, ws, okv = setup

    def fwd(canvas, s):
        st = om.denoise_forward(ws, okv, canvas, s, W.T, W.prompt_len)
        return st["H"], st["argmax"]

    ocanvas, traj = osamp.generate_block(fwd, W.canvas, W.mask_id, W.T, W.gamma)
    dc = torch.full((1, W.canvas), W.mask_id, dtype=torch.int32, device="cuda")
    dm = torch.ones((1, W.canvas), dtype=torch.uint8, device="cuda")
    for (s, H, am, c_after, m_after, n) in traj:
        ent, amax, ncom = binding.dg_denoise_step(model, kv, dc, dm, s, W.T, W.gamma)
        torch.cuda.synchronize()
        assert np.array_equal(ent[0].cpu().numpy(), H), f"entropies differ at s={s}"
        assert np.array_equal(amax[0].cpu().numpy(), am)
        assert int(ncom[0]) == n
        assert np.array_equal(dc[0].cpu().numpy(), c_after)
        assert np.array_equal(dm[0].cpu().numpy(), m_after)
    binding.dg_sync_status(model)
    # the device-side block loop gives the same final canvas
    out = binding.dg_generate_block(model, kv, W.T, W.gamma,
                                    n_forwards=torch.zeros(1, dtype=torch.int32, device="cuda"))
    binding.dg_sync_status(model)
    assert np.array_equal(out[0].cpu().numpy(), ocanvas)
    assert not (out == W.mask_id).any()


def test_bad_token_reported(setup):
    binding, model, kv, ws, okv = setup
    dc = torch.full((1, W.canvas), W.vocab + 5, dtype=torch.int32, device="cuda")
    binding.dg_debug_forward(model, kv, dc, 2, W.T)
    with pytest.raises(binding.DGError) as e:
        binding.dg_sync_status(model)
    assert e.value.status == 1


def test_kv_outlives_model():
    """Destroying the model first leaves its caches destroyable, and unusable."""
    from masked_discrete_diffusion_b200 import binding
    model = make_model(W)
    kv = binding.dg_prefill(model, model_inputs.prompt(W, "cuda"))
    binding.dg_sync_status(model)
    h = kv.handle
    binding._check(binding.lib().dg_model_destroy(model.handle))
    model.handle = None
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = binding.lib().dg_kv_read(h, n.data_ptr(), n.data_ptr(), None)
    assert st == 1                                        # DG_ERR_INVALID_ARG
    assert binding.lib().dg_kv_destroy(h) == 0
    kv.handle = None
