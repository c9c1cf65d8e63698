"""Small bf16 model through the whole tensor-core path vs the oracle.

Covers what the full-size workloads do not: a prompt longer than the attention
window (160 > 128, sliding-window causal prefill), a canvas that is not a multiple
of the 128-row tile (C = 96), batch 3, experts receiving more than 256 rows.
Tolerance 2e-2 max-abs relative (bf16 bound).
"""
import math

import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import sampler as osamp
from synth import model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel

pytestmark = pytest.mark.gpu
W = workloads.SMALL_BF16
TOL = 2e-2


@pytest.fixture(scope="module")
def setup():
    from masked_discrete_diffusion_b200 import binding
    model = make_model(W)
    prompt = model_inputs.prompt(W, "cuda")
    kv = binding.dg_prefill(model, prompt)
    binding.dg_sync_status(model)
    ws = om.Weights(W, keep_layers=True)
    okv = [om.prefill(ws, prompt[b].cpu().numpy()) for b in range(W.batch)]
    yield binding, model, kv, ws, okv
    kv.close()
    model.close()


def test_prefill_window(setup):
    binding, model, kv, ws, okv = setup
    assert kv.W == W.window
    k, v = binding.dg_kv_read(kv)
    binding.dg_sync_status(model)
    for b in range(W.batch):
        for l in range(W.n_layers):
            assert max_abs_rel(k[l, b].float().cpu().numpy(), okv[b][l][0].transpose(1, 0, 2)) < TOL
            assert max_abs_rel(v[l, b].float().cpu().numpy(), okv[b][l][1].transpose(1, 0, 2)) < TOL


@pytest.mark.parametrize("s", [6, 2])
def test_forward(setup, s):
    binding, model, kv, ws, okv = setup
    canvas = np.full((W.batch, W.canvas), W.mask_id)
    canvas[:, ::5] = (np.arange(0, W.canvas, 5)[None, :] * 7 + np.arange(W.batch)[:, None] * 3) % W.vocab
    dc = torch.from_numpy(canvas.astype(np.int32)).cuda()
    ent, am, lg, hd = binding.dg_debug_forward(model, kv, dc, s, W.T, logits=True, hidden=True)
    ent2, am2, _, _ = binding.dg_debug_forward(model, kv, dc, s, W.T)
    binding.dg_sync_status(model)
    lg = lg.cpu().numpy().reshape(W.batch, W.canvas, W.vocab)
    for b in range(W.batch):
        st = om.denoise_forward(ws, okv[b], canvas[b], s, W.T, W.prompt_len, want_logits=True,
                                want_hidden=True)
        assert max_abs_rel(lg[b], st["logits"]) < TOL
        for e, a in ((ent, am), (ent2, am2)):
            assert max_abs_rel(e[b].cpu().numpy(), st["H"]) < TOL
            eps = float(np.abs(lg[b] - st["logits"]).max())
            decided = st["margin"] > 2 * eps + 1e-3
            assert np.array_equal(a[b].cpu().numpy()[decided], st["argmax"][decided])
        assert np.all(ent2[b].cpu().numpy() <= math.log(W.vocab) + 1e-3)


def test_block_invariants(setup):
    binding, model, kv, ws, okv = setup
    nf = torch.zeros(W.batch, dtype=torch.int32, device="cuda")
    load = torch.zeros(W.n_layers, W.n_experts, dtype=torch.int32, device="cuda")
    out = binding.dg_generate_block(model, kv, W.T, W.gamma, n_forwards=nf, router_load=load)
    binding.dg_sync_status(model)
    assert not (out == W.mask_id).any()
    assert int(out.min()) >= 0 and int(out.max()) < W.vocab
    assert nf.cpu().tolist() == [W.T] * W.batch          # the ceil(m/s) minimum ends at step T
    # every (token, forward) routes to top_k experts in each layer
    assert load.sum(dim=1).cpu().tolist() == [W.batch * W.canvas * W.top_k * W.T] * W.n_layers
    # the same block through dg_denoise_step, step by step: identical canvases
    dc = torch.full((W.batch, W.canvas), W.mask_id, dtype=torch.int32, device="cuda")
    dm = torch.ones_like(dc, dtype=torch.uint8)
    prev = dm.clone()
    for k in range(W.T):
        s = W.T - k
        ent, am, n = binding.dg_denoise_step(model, kv, dc, dm, s, W.T, W.gamma)
        assert bool((dm <= prev).all())
        assert int(dm.sum(dim=1).max()) <= W.canvas * (s - 1) // W.T
        prev = dm.clone()
    binding.dg_sync_status(model)
    assert torch.equal(dc, out)


def test_block_graph_replay_is_deterministic(setup):
    """The captured block replays to bit-identical canvases and routing counts."""
    binding, model, kv, ws, okv = setup
    outs = []
    for _ in range(3):
        load = torch.zeros(W.n_layers, W.n_experts, dtype=torch.int32, device="cuda")
        out = torch.empty(W.batch, W.canvas, dtype=torch.int32, device="cuda")
        binding.dg_generate_block(model, kv, W.T, W.gamma, canvas_out=out, router_load=load)
        outs.append((out.clone(), load.clone()))
    binding.dg_sync_status(model)
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


def test_prefill_into_reuses_the_handle(setup):
    """Refilling a handle in place gives the cache a fresh dg_prefill of the same prompt
    gives, and the block graph captured for the handle then denoises the new prompt
    exactly as a fresh handle would."""
    binding, model, kv, ws, okv = setup
    other = model_inputs.prompt(W, "cuda", first=W.batch)            # canvases 3..5
    fresh = binding.dg_prefill(model, other)
    slot = binding.dg_prefill(model, model_inputs.prompt(W, "cuda"))
    a = binding.dg_generate_block(model, slot, W.T, W.gamma)          # graph for the slot
    binding.dg_prefill_into(model, other, slot)
    k1, v1 = binding.dg_kv_read(slot)
    k2, v2 = binding.dg_kv_read(fresh)
    assert torch.equal(k1, k2) and torch.equal(v1, v2)
    b = binding.dg_generate_block(model, slot, W.T, W.gamma)          # same graph, new cache
    c = binding.dg_generate_block(model, fresh, W.T, W.gamma)
    binding.dg_sync_status(model)
    assert torch.equal(b, c) and not torch.equal(a, b)
    with pytest.raises(binding.DGError):                              # batch must match
        binding.dg_prefill_into(model, other[:2].contiguous(), slot)
    slot.close()
    fresh.close()
