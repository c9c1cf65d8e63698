"""FP8 E4M3 routed-expert weights (per-row, per-128-column fp32 scales), bf16 elsewhere.

The oracle uses the represented weights code * scale in fp64; the CUDA path
converts the FP8 tiles to bf16 in shared memory before the tensor-core MMA.
Tolerance 3e-2 max-abs relative (the FP8 workload's bound).
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import model as om
from synth import gen, model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel, storage_tol

pytestmark = pytest.mark.gpu
TOL = 3e-2
W = workloads.SMALL_FP8


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


def test_fp8_weights_are_stored_as_bytes(small):
    binding, model, kv, ws, okv = small
    t = model.tensors
    assert t["l0.gate"].dtype == torch.uint8 and t["l0.gate_scale"].dtype == torch.float32
    assert t["l0.gate_scale"].shape == (W.n_experts, W.expert_inter, W.d_model // 128)
    assert t["l0.down_scale"].shape == (W.n_experts, W.d_model, W.expert_inter // 128)


def test_fp8_moe_block(small):
    binding, model, kv, ws, okv = small
    n = 288
    x = gen.normal_values(9, "x8", 0, n * W.d_model, 1.0, "cuda").reshape(n, W.d_model)
    out = binding.dg_op_moe(model, 1, x)
    binding.dg_sync_status(model)
    xd = x.double().cpu().numpy()
    y, idx, g, logits = om.moe(om.rmsnorm(xd, W.rms_eps), ws.layer(1), W.top_k)
    srt = np.sort(logits, axis=1)[:, ::-1]
    decided = (srt[:, W.top_k - 1] - srt[:, W.top_k]) > 1e-3
    assert max_abs_rel(out.cpu().numpy()[decided] - xd[decided], y[decided]) < TOL


def test_fp8_prefill_and_forward(small):
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


def test_fp8_block(small):
    binding, model, kv, ws, okv = small
    nf = torch.zeros(W.batch, dtype=torch.int32, device="cuda")
    out = binding.dg_generate_block(model, kv, W.T, W.gamma, n_forwards=nf)
    binding.dg_sync_status(model)
    assert not (out == W.mask_id).any() and nf.cpu().tolist() == [W.T] * W.batch


GOLD = os.path.join(os.path.dirname(__file__), "golden", "layer1-fp8exp-p4096.npz")


@pytest.mark.skipif(not os.path.exists(GOLD), reason="golden file missing")
def test_fp8_full_size_layer():
    """One full-size layer with FP8 experts and the FP8 workload's 4096-token prompt."""
    from masked_discrete_diffusion_b200 import binding
    w = workloads.LAYER1_FP8
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
        assert max_abs_rel(lgs, g["logits"]) < TOL
        # entropies: no stated tolerance; twice the oracle's bf16-storage distance
        # (bf16 activations and the FP8 weights dequantised to bf16), at least TOL
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
