"""NVFP4 routed-expert weights (E2M1 codes, an E4M3 scale per 16 input columns, a
power-of-two scale per tensor), bf16 elsewhere.

A represented weight e2m1(code) * block scale * 2^k has at most 6 significant bits,
so the bf16 tile the converter warps write holds it exactly: the CUDA path and the
oracle (which uses the represented weights in fp64) see the same expert weights, and
only the activations' bf16 storage separates them.  Tolerance: the stated bf16 bound
2e-2 max-abs relative (the pages state none for NVFP4), with the storage rule of the
deep workloads where the oracle's own bf16-storage run moves further.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import model as om
from synth import gen, model_inputs, nvfp4, workloads

from gpu_helpers import make_model, max_abs_rel, storage_tol

pytestmark = pytest.mark.gpu
TOL = 2e-2
W = workloads.SMALL_FP4


@pytest.fixture(scope="module")
def small():
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


def test_fp4_weights_are_stored_packed(small):
    binding, model, kv, ws, okv = small
    t = model.tensors
    assert t["l0.gate"].dtype == torch.uint8
    assert t["l0.gate"].shape == (W.n_experts, W.expert_inter, W.d_model // 2)
    assert t["l0.down"].shape == (W.n_experts, W.d_model, W.expert_inter // 2)
    assert t["l0.gate_scale"].dtype == torch.uint8
    assert t["l0.gate_scale"].shape == (W.n_experts, W.expert_inter, W.d_model // 16)
    assert t["l0.down_tscale"].dtype == torch.float32 and t["l0.down_tscale"].numel() == 1
    # every represented weight is a bf16 value (the exactness the parity relies on)
    deq = nvfp4.dequantised(W, "l0.gate", (W.n_experts, W.expert_inter, W.d_model),
                            W.init_std, 0, 2)
    t64 = torch.from_numpy(deq)
    assert torch.equal(t64.to(torch.bfloat16).to(torch.float64), t64)


def test_fp4_moe_block(small):
    binding, model, kv, ws, okv = small
    n = 288
    x = gen.normal_values(9, "x4", 0, n * W.d_model, 1.0, "cuda").reshape(n, W.d_model)
    out = binding.dg_op_moe(model, 1, x)
    binding.dg_sync_status(model)
    xd = x.double().cpu().numpy()
    y, idx, g, logits = om.moe(om.rmsnorm(xd, W.rms_eps), ws.layer(1), W.top_k)
    srt = np.sort(logits, axis=1)[:, ::-1]
    decided = (srt[:, W.top_k - 1] - srt[:, W.top_k]) > 1e-3
    assert decided.mean() > 0.8
    assert max_abs_rel(out.cpu().numpy()[decided] - xd[decided], y[decided]) < TOL


def test_fp4_prefill_and_forward(small):
    binding, model, kv, ws, okv = small
    k, v = binding.dg_kv_read(kv)
    canvas = np.full((W.batch, W.canvas), W.mask_id)
    canvas[:, 1::4] = 17
    dc = torch.from_numpy(canvas.astype(np.int32)).cuda()
    ent, am, lg, _ = binding.dg_debug_forward(model, kv, dc, 4, W.T, logits=True)
    ent2, am2, _, _ = binding.dg_debug_forward(model, kv, dc, 4, W.T)
    binding.dg_sync_status(model)
    lg = lg.cpu().numpy().reshape(W.batch, W.canvas, W.vocab)
    for b in range(W.batch):
        for l in range(W.n_layers):
            assert max_abs_rel(k[l, b].float().cpu().numpy(), okv[b][l][0].transpose(1, 0, 2)) < TOL
        st = om.denoise_forward(ws, okv[b], canvas[b], 4, W.T, W.prompt_len, want_logits=True)
        assert max_abs_rel(lg[b], st["logits"]) < TOL
        for e in (ent, ent2):
            assert max_abs_rel(e[b].cpu().numpy(), st["H"]) < TOL
        eps = float(np.abs(lg[b] - st["logits"]).max())
        decided = st["margin"] > 2 * eps + 1e-3
        assert np.array_equal(am2[b].cpu().numpy()[decided], st["argmax"][decided])


def test_fp4_block(small):
    binding, model, kv, ws, okv = small
    nf = torch.zeros(W.batch, dtype=torch.int32, device="cuda")
    out = binding.dg_generate_block(model, kv, W.T, W.gamma, n_forwards=nf)
    binding.dg_sync_status(model)
    assert not (out == W.mask_id).any() and ((nf >= 1) & (nf <= W.T)).all()


def test_fp4_needs_its_scales():
    from masked_discrete_diffusion_b200 import binding
    w = W.with_(n_layers=1)
    t = model_inputs.weight_set(w, "cuda")
    up_ts = t.pop("l0.up_tscale")
    with pytest.raises(binding.DGError) as e:
        binding.Model(binding.make_config(w), t)
    assert "NVFP4 scale" in str(e.value)
    # a tensor scale that is not a power of two would make the widened weights inexact
    t["l0.up_tscale"] = up_ts * 3
    with pytest.raises(binding.DGError) as e:
        binding.Model(binding.make_config(w), t)
    assert "power of two" in str(e.value)


GOLD = os.path.join(os.path.dirname(__file__), "golden", "layer1-fp4exp.npz")


@pytest.mark.skipif(not os.path.exists(GOLD), reason="golden file missing")
def test_fp4_full_size_layer():
    """One full-size layer (d 2048, 128 experts top-8, I 768) with NVFP4 experts."""
    from masked_discrete_diffusion_b200 import binding
    w = workloads.LAYER1_FP4
    g = np.load(GOLD)
    model = make_model(w)
    try:
        kv = binding.dg_prefill(model, model_inputs.prompt(w, "cuda"))
        canvas = torch.full((1, w.canvas), w.mask_id, dtype=torch.int32, device="cuda")
        ent, am, lg, _ = binding.dg_debug_forward(model, kv, canvas, w.T, w.T, logits=True)
        ent2, am2, _, _ = binding.dg_debug_forward(model, kv, canvas, w.T, w.T)
        k, v = binding.dg_kv_read(kv)
        binding.dg_sync_status(model)
        rows = torch.as_tensor(g["logit_rows"]).cuda()
        cols = torch.as_tensor(g["logit_cols"]).cuda()
        lgs = lg[rows][:, cols].cpu().numpy()
        assert max_abs_rel(lgs, g["logits"]) < storage_tol(g, "logits", TOL)
        tol_h = storage_tol(g, "H", TOL)
        assert max_abs_rel(ent2[0].cpu().numpy(), g["H"]) < tol_h
        assert max_abs_rel(ent[0].cpu().numpy(), g["H"]) < tol_h
        assert max_abs_rel(k[0, 0, :, -8:].float().cpu().numpy(), g["kv_last"][0, 0]) < TOL
        eps = float(np.abs(lgs - g["logits"]).max())
        decided = g["margin"] > 2 * eps + 1e-3
        assert np.array_equal(am2[0].cpu().numpy()[decided], g["argmax"][decided])
        assert np.all(ent2[0].cpu().numpy() <= math.log(w.vocab) + 1e-3)
        kv.close()
    finally:
        model.close()
