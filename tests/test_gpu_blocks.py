"""Block-autoregressive continuation: a finished block joins the context through the
causal pass (dg_append_block), and blocks follow one another (dg_generate_blocks).

The oracle's reference for appending is the causal pass over the whole sequence
(prompt followed by the block): the cache after an append must hold the keys and
values that pass gives to the last min(P + C, window) positions.
  * tiny fp32 model (fp64 activations on the device): three blocks generated one after
    the other must reproduce oracle.model.generate_blocks token for token, with the
    same number of forwards per block, and the cache after two appends must match the
    causal pass over prompt + two blocks (1e-9);
  * small bf16 model: the window (128) is full before the append, so part of it shifts
    out; three canvases at once; 2e-2 max-abs relative;
  * one full-size layer: prompt 1024 + a 256-token block through the tensor-core
    attention in causal mode over the cached window and the block
    (tests/golden/layer1-bf16-append.npz); 2e-2 max-abs relative.
"""
import os

import numpy as np
import pytest
import torch

from oracle import model as om
from synth import model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_tiny_blocks_exact():
    from masked_discrete_diffusion_b200 import binding
    w = workloads.TINY_F32
    n_blocks = 3
    model = make_model(w, max_prompt=w.prompt_len + (n_blocks - 1) * w.canvas)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        out, nf = binding.dg_generate_blocks(model, kv, n_blocks, w.T, w.gamma)
        binding.dg_sync_status(model)
        assert kv.P == w.prompt_len + (n_blocks - 1) * w.canvas
        ws = om.Weights(w, keep_layers=True)
        blocks, trajs = om.generate_blocks(ws, prompt[0].cpu().numpy(), n_blocks, w.T, w.gamma)
        assert np.array_equal(out[0].cpu().numpy(), blocks.reshape(-1))
        assert nf[:, 0].cpu().tolist() == [len(t) for t in trajs]
        k, v = binding.dg_kv_read(kv)
        seq = np.concatenate([prompt[0].cpu().numpy(), blocks[:-1].reshape(-1)])
        okv = om.prefill(ws, seq)
        for l in range(w.n_layers):
            ok, ov = okv[l]
            assert max_abs_rel(k[l, 0].cpu().numpy(), ok.transpose(1, 0, 2)) < 1e-9
            assert max_abs_rel(v[l, 0].cpu().numpy(), ov.transpose(1, 0, 2)) < 1e-9
        kv.close()
    finally:
        model.close()


def test_small_append_shifts_the_window():
    from masked_discrete_diffusion_b200 import binding
    w = workloads.SMALL_BF16
    model = make_model(w, max_prompt=w.prompt_len + w.canvas)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        block = model_inputs.block_tokens(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        assert kv.W == w.window                     # 160 > 128: the window is full
        binding.dg_append_block(model, kv, block)
        binding.dg_sync_status(model)
        assert kv.P == w.prompt_len + w.canvas and kv.W == w.window
        k, v = binding.dg_kv_read(kv)
        ws = om.Weights(w, keep_layers=True)
        for b in range(w.batch):
            seq = np.concatenate([prompt[b].cpu().numpy(), block[b].cpu().numpy()])
            okv = om.prefill(ws, seq)
            for l in range(w.n_layers):
                ok, ov = okv[l]
                assert max_abs_rel(k[l, b].float().cpu().numpy(), ok.transpose(1, 0, 2)) < 2e-2
                assert max_abs_rel(v[l, b].float().cpu().numpy(), ov.transpose(1, 0, 2)) < 2e-2
        # a block denoised on the extended cache is complete and the cache keeps its size
        out = binding.dg_generate_block(model, kv, w.T, w.gamma)
        binding.dg_sync_status(model)
        assert not (out == w.mask_id).any()
        kv.close()
    finally:
        model.close()


def test_full_size_layer_append():
    path = os.path.join(GOLDEN, "layer1-bf16-append.npz")
    if not os.path.exists(path):
        pytest.skip("golden file missing")
    from masked_discrete_diffusion_b200 import binding
    w = workloads.LAYER1_BF16
    g = np.load(path)
    model = make_model(w, max_prompt=w.prompt_len + w.canvas)
    try:
        kv = binding.dg_prefill(model, model_inputs.prompt(w, "cuda"))
        binding.dg_append_block(model, kv, model_inputs.block_tokens(w, "cuda"))
        k, v = binding.dg_kv_read(kv)
        binding.dg_sync_status(model)
        assert kv.W == int(g["window"])
        sel = torch.as_tensor(g["positions"]).cuda()
        kk = k[0, 0][:, sel].float().cpu().numpy()   # [Hkv, positions, h]
        vv = v[0, 0][:, sel].float().cpu().numpy()
        assert max_abs_rel(kk, g["k"]) < 2e-2
        assert max_abs_rel(vv, g["v"]) < 2e-2
        kv.close()
    finally:
        model.close()


@pytest.mark.parametrize("name", ["tiny-f32", "tiny-f32-sc"])
def test_tiny_annealed_blocks_with_append_exact(name):
    """Block-autoregressive generation with the Report's sampler: an annealed block, its
    causal append, a second annealed block conditioned on prompt + first block; both
    blocks token for token against the oracle's annealed blocks over the same contexts
    (with self-conditioning: z starts from 0 again in the second block)."""
    from masked_discrete_diffusion_b200 import binding
    from oracle import anneal as an
    w = workloads.get(name)
    p = an.Params(tau_max=0.02, tau_min=0.02)      # canvas 0 of this prompt stops early
    model = make_model(w, max_prompt=w.prompt_len + w.canvas)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        b1, nf1 = binding.dg_generate_block_annealed(model, kv, [7], p)
        binding.dg_append_block(model, kv, b1)
        b2, nf2 = binding.dg_generate_block_annealed(model, kv, [8], p)
        binding.dg_sync_status(model)
        ws = om.Weights(w, keep_layers=True)
        ctx = prompt[0].cpu().numpy()
        r1, t1 = om.generate_block_annealed(ws, ctx, 7, p)
        r2, t2 = om.generate_block_annealed(ws, np.concatenate([ctx, r1]), 8, p)
        assert np.array_equal(b1[0].cpu().numpy(), r1) and int(nf1[0]) == len(t1)
        assert np.array_equal(b2[0].cpu().numpy(), r2) and int(nf2[0]) == len(t2)
        kv.close()
    finally:
        model.close()
