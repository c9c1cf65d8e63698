"""One Gemma-4-26B-A4B-shaped layer + 262,144-token LM head (bf16): CUDA path vs oracle.

Expected values come from tests/golden/layer1-bf16.npz, written by
tests/golden/make_golden.py from the oracle alone.  Tolerance 2e-2 max-abs
relative to the oracle for logits and entropies (bf16 workload bound).
"""
import math
import os

import numpy as np
import pytest
import torch

from synth import model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel

pytestmark = pytest.mark.gpu
W = workloads.LAYER1_BF16
TOL = 2e-2
GOLD = os.path.join(os.path.dirname(__file__), "golden", "layer1-bf16.npz")


@pytest.fixture(scope="module")
def run():
    from masked_discrete_diffusion_b200 import binding
    g = np.load(GOLD)
    model = make_model(W)
    kv = binding.dg_prefill(model, model_inputs.prompt(W, "cuda"))
    canvas = torch.full((1, W.canvas), W.mask_id, dtype=torch.int32, device="cuda")
    ent, am, lg, _ = binding.dg_debug_forward(model, kv, canvas, W.T, W.T, logits=True)
    ent2, am2, _, _ = binding.dg_debug_forward(model, kv, canvas, W.T, W.T)
    k, v = binding.dg_kv_read(kv)
    binding.dg_sync_status(model)
    rows = torch.as_tensor(g["logit_rows"]).cuda()
    cols = torch.as_tensor(g["logit_cols"]).cuda()
    out = dict(g=g, ent=ent[0].cpu().numpy(), am=am[0].cpu().numpy(),
               ent2=ent2[0].cpu().numpy(), am2=am2[0].cpu().numpy(),
               lg=lg[rows][:, cols].cpu().numpy(), lmax=float(lg.abs().max()),
               k=k.float().cpu().numpy(), v=v.float().cpu().numpy(), binding=binding,
               model=model, kv=kv)
    del lg
    yield out
    kv.close()
    model.close()


def test_prefill_window_kv(run):
    g = run["g"]
    kl = g["kv_last"][0]                        # layer 0: [2, Hkv, 8, h]
    assert max_abs_rel(run["k"][0, 0, :, -8:], kl[0]) < TOL
    assert max_abs_rel(run["v"][0, 0, :, -8:], kl[1]) < TOL


def test_logits_sampled(run):
    assert max_abs_rel(run["lg"], run["g"]["logits"]) < TOL


def test_entropies(run):
    g = run["g"]
    for ent in (run["ent"], run["ent2"]):          # CUDA-core and tensor-core LM heads
        assert max_abs_rel(ent, g["H"]) < TOL
        assert np.all(ent >= 0) and np.all(ent <= math.log(W.vocab) + 1e-3)


def test_argmax_where_decided(run):
    g = run["g"]
    eps = float(np.abs(run["lg"] - g["logits"]).max())
    decided = g["margin"] > 2 * eps + 1e-3
    assert decided.mean() > 0.5
    for am in (run["am"], run["am2"]):
        assert np.array_equal(am[decided], g["argmax"][decided])


def test_sampler_step_valid(run):
    """The device sampler's commit on its own entropies is the rule's unique result."""
    b = run["binding"]
    H = torch.from_numpy(run["ent2"]).cuda()[None]
    am = torch.from_numpy(run["am2"]).cuda()[None]
    canvas = torch.full((1, W.canvas), W.mask_id, dtype=torch.int32, device="cuda")
    mask = torch.ones_like(canvas, dtype=torch.uint8)
    n = int(b.dg_eb_sample(H, am, canvas, mask, W.T, W.gamma)[0])
    Hn = run["ent2"]
    order = sorted(range(W.canvas), key=lambda i: (Hn[i], i))
    acc, kg = 0.0, 0
    for i in order:
        if acc + Hn[i] > W.gamma:
            break
        acc += Hn[i]
        kg += 1
    assert n == max(kg, math.ceil(W.canvas / W.T)) == int(run["g"]["step_n"])
    committed = set(np.nonzero(mask[0].cpu().numpy() == 0)[0])
    assert committed == set(order[:n])
    assert np.array_equal(canvas[0].cpu().numpy()[order[:n]], run["am2"][order[:n]])
