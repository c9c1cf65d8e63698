"""Self-conditioning on the device (models with sc_inter > 0) against the oracle's
oracle.model.selfcond / CanvasForwards.

  * tiny fp32 model (fp64 activations on the device): one forward's entropies (1e-6)
    and the z it hands on (1e-9), a second forward fed the device's own z; whole
    Entropy-Bound and annealed blocks token for token with the oracle's forward counts
    (the FFW's weights are drawn large enough that z changes 13 of the 32 tokens);
  * small bf16 model (tensor-core p0 E^T GEMM, K-sliced): z within 2e-2 max-abs
    relative, the next forward's entropies with the oracle's z fed in; the block as a
    loop graph equals the plain launches; switched off, the block equals that of the
    same weights without the FFW;
  * the annealed forward with self-conditioning (tempered statistics and draws, p0 at
    temperature 1): tiny exact, small bf16 within 2e-2 and on decided draws;
  * one full-size layer (V = 262,144: p0 over the whole vocabulary, 16 K slices):
    the entropies and z against the golden file (2e-2, or 1.5x the oracle's
    bf16-storage distance where that exceeds 1e-2).
"""
import os

import numpy as np
import pytest
import torch

from oracle import anneal as an
from oracle import model as om
from synth import model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel, storage_tol

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_tiny_forward_and_z():
    from masked_discrete_diffusion_b200 import binding
    w = workloads.TINY_F32_SC
    model = make_model(w)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        ws = om.Weights(w, keep_layers=True)
        okv = om.prefill(ws, prompt[0].cpu().numpy())
        canvas = np.full(w.canvas, w.mask_id)
        dcanvas = torch.from_numpy(canvas.astype(np.int32)).reshape(1, -1).cuda()
        H, am, z = binding.dg_selfcond_forward(model, kv, dcanvas, w.T, w.T)
        binding.dg_sync_status(model)
        st = om.denoise_forward(ws, okv, canvas, w.T, w.T, w.prompt_len, want_logits=True)
        oz = om.selfcond(ws, st["logits"])
        assert max_abs_rel(H[0].cpu().numpy(), st["H64"]) < 1e-6
        assert np.array_equal(am[0].cpu().numpy(), st["argmax"])
        assert max_abs_rel(z[0].cpu().numpy(), oz) < 1e-9
        # the next forward, fed the device's z (and the oracle's own on its side)
        H2, am2, z2 = binding.dg_selfcond_forward(model, kv, dcanvas, w.T - 1, w.T, z_in=z)
        binding.dg_sync_status(model)
        st2 = om.denoise_forward(ws, okv, canvas, w.T - 1, w.T, w.prompt_len, want_logits=True,
                                 z=oz)
        assert max_abs_rel(H2[0].cpu().numpy(), st2["H64"]) < 1e-6
        assert np.array_equal(am2[0].cpu().numpy(), st2["argmax"])
        assert max_abs_rel(z2[0].cpu().numpy(), om.selfcond(ws, st2["logits"])) < 1e-9
        # z matters: the second forward differs from one without it
        plain = om.denoise_forward(ws, okv, canvas, w.T - 1, w.T, w.prompt_len)
        assert np.abs(plain["H64"] - st2["H64"]).max() > 1e-3
        kv.close()
    finally:
        model.close()


def test_tiny_entropy_bound_block_token_for_token():
    from masked_discrete_diffusion_b200 import binding
    w = workloads.TINY_F32_SC
    model = make_model(w)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        nf = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = binding.dg_generate_block(model, kv, w.T, w.gamma, n_forwards=nf)
        binding.dg_sync_status(model)
        ws = om.Weights(w, keep_layers=True)
        canvas, traj = om.generate_block(ws, prompt[0].cpu().numpy(), w.T, w.gamma)
        assert np.array_equal(out[0].cpu().numpy(), canvas)
        assert int(nf[0]) == len(traj)
        # the same weights without self-conditioning give another block
        binding.dg_set_selfcond(model, False)
        out0 = binding.dg_generate_block(model, kv, w.T, w.gamma)
        binding.dg_sync_status(model)
        ref0, _ = om.generate_block(om.Weights(workloads.TINY_F32, keep_layers=True),
                                    prompt[0].cpu().numpy(), w.T, w.gamma)
        assert np.array_equal(out0[0].cpu().numpy(), ref0)
        assert not np.array_equal(canvas, ref0)
        kv.close()
    finally:
        model.close()


@pytest.mark.parametrize("tau", [None, 0.02])
def test_tiny_annealed_block_token_for_token(tau):
    from masked_discrete_diffusion_b200 import binding
    w = workloads.TINY_F32_SC.with_(batch=2)
    p = an.Params() if tau is None else an.Params(tau_max=tau, tau_min=tau)
    seeds = [71, 72]
    model = make_model(w)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        out, nf = binding.dg_generate_block_annealed(model, kv, seeds, p)
        binding.dg_sync_status(model)
        ws = om.Weights(w, keep_layers=True)
        for b in range(2):
            res, traj = om.generate_block_annealed(ws, prompt[b].cpu().numpy(), seeds[b], p)
            assert np.array_equal(out[b].cpu().numpy(), res), b
            assert int(nf[b]) == len(traj), b
        kv.close()
    finally:
        model.close()


@pytest.mark.parametrize("vocab", [1024, 1000])
def test_small_bf16_z_and_next_forward(vocab):
    """V = 1000: p0's last vocabulary tile is partial."""
    from masked_discrete_diffusion_b200 import binding
    w = workloads.SMALL_BF16_SC.with_(vocab=vocab)
    model = make_model(w)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        ws = om.Weights(w, keep_layers=True)
        canvas = np.full((w.batch, w.canvas), w.mask_id)
        dcanvas = torch.from_numpy(canvas.astype(np.int32)).cuda()
        H, am, z = binding.dg_selfcond_forward(model, kv, dcanvas, w.T, w.T)
        binding.dg_sync_status(model)
        ozs = []
        for b in range(w.batch):
            st = om.prefill_then_forward(ws, prompt[b].cpu().numpy(), canvas[b], w.T, w.T,
                                         want_logits=True)
            oz = om.selfcond(ws, st["logits"])
            ozs.append(oz)
            assert max_abs_rel(H[b].cpu().numpy(), st["H64"]) < 2e-2
            assert max_abs_rel(z[b].cpu().numpy(), oz) < 2e-2
        # the next forward with the oracle's z fed to both sides
        zin = torch.from_numpy(np.stack(ozs).astype(np.float32)).cuda()
        H2, _, _ = binding.dg_selfcond_forward(model, kv, dcanvas, w.T - 1, w.T, z_in=zin)
        binding.dg_sync_status(model)
        for b in range(w.batch):
            st2 = om.prefill_then_forward(ws, prompt[b].cpu().numpy(), canvas[b], w.T - 1, w.T,
                                          z=ozs[b])
            plain = om.prefill_then_forward(ws, prompt[b].cpu().numpy(), canvas[b], w.T - 1,
                                            w.T)
            assert max_abs_rel(H2[b].cpu().numpy(), st2["H64"]) < 2e-2
            assert max_abs_rel(plain["H64"], st2["H64"]) > 2e-2      # z matters (3-5 %)
        kv.close()
    finally:
        model.close()


def test_small_bf16_block_graph_plain_and_switch(monkeypatch):
    from masked_discrete_diffusion_b200 import binding
    w = workloads.SMALL_BF16_SC
    outs = {}
    for no_graphs in ("0", "1"):
        monkeypatch.setenv("DG_NO_GRAPHS", no_graphs)
        model = make_model(w)
        try:
            kv = binding.dg_prefill(model, model_inputs.prompt(w, "cuda"))
            nf = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
            out = binding.dg_generate_block(model, kv, w.T, w.gamma, n_forwards=nf)
            binding.dg_set_selfcond(model, False)
            off = binding.dg_generate_block(model, kv, w.T, w.gamma)
            binding.dg_set_selfcond(model, True)
            again = binding.dg_generate_block(model, kv, w.T, w.gamma)
            binding.dg_sync_status(model)
            assert torch.equal(again, out)
            assert not (out == w.mask_id).any()
            outs[no_graphs] = (out.cpu(), off.cpu(), nf.cpu())
            kv.close()
        finally:
            model.close()
    assert all(torch.equal(a, b) for a, b in zip(outs["0"], outs["1"]))
    # switched off, the block is that of the same weights without the FFW
    monkeypatch.setenv("DG_NO_GRAPHS", "0")
    plain = make_model(workloads.SMALL_BF16)
    try:
        kv = binding.dg_prefill(plain, model_inputs.prompt(w, "cuda"))
        ref = binding.dg_generate_block(plain, kv, w.T, w.gamma)
        binding.dg_sync_status(plain)
        assert torch.equal(ref.cpu(), outs["0"][1])
        kv.close()
    finally:
        plain.close()


def test_set_selfcond_needs_the_ffw():
    from masked_discrete_diffusion_b200 import binding
    model = make_model(workloads.TINY_F32)
    try:
        with pytest.raises(binding.DGError) as e:
            binding.dg_set_selfcond(model, True)
        assert e.value.status == 1
        binding.dg_set_selfcond(model, False)
    finally:
        model.close()


def test_full_size_layer_z():
    path = os.path.join(GOLDEN, "layer1-bf16-sc-selfcond.npz")
    if not os.path.exists(path):
        pytest.skip("golden file missing")
    from masked_discrete_diffusion_b200 import binding
    w = workloads.LAYER1_BF16_SC
    g = np.load(path)
    model = make_model(w)
    try:
        kv = binding.dg_prefill(model, model_inputs.prompt(w, "cuda"))
        canvas = torch.full((1, w.canvas), w.mask_id, dtype=torch.int32, device="cuda")
        H, am, z = binding.dg_selfcond_forward(model, kv, canvas, w.T, w.T)
        binding.dg_sync_status(model)
        assert max_abs_rel(H[0].cpu().numpy(), g["H64"]) < storage_tol(g, "H64", 2e-2)
        # z ends a chain of bf16 stores (p0, y = p0 E, the FFW's hidden rows) and a
        # cancelling sum over d: the storage-noise rule of the deep tests applies
        assert max_abs_rel(z[0].cpu().numpy(), g["z"]) < storage_tol(g, "z", 2e-2)
        kv.close()
    finally:
        model.close()


# --- self-conditioning inside the annealed forward (p0 at temperature 1 while the
# statistics and the draw are tempered) ---------------------------------------------------
def _anneal_sc_oracle(ws, okv_or_prompt, canvas, k, seed, p, z, w, prefilled):
    if prefilled:
        st = om.denoise_forward(ws, okv_or_prompt, canvas, p.N - k, p.N, w.prompt_len,
                                want_logits=True, z=z)
    else:
        st = om.prefill_then_forward(ws, okv_or_prompt, canvas, p.N - k, p.N,
                                     want_logits=True, z=z)
    tau = an.temperature(k, p)
    ts = an.tempered_stats(st["logits"], tau)
    drawn, gap = an.sample_tokens(st["logits"], tau, seed, k)
    return ts, drawn, gap, om.selfcond(ws, st["logits"])


def test_tiny_annealed_forward_with_selfcond():
    from masked_discrete_diffusion_b200 import binding
    w = workloads.TINY_F32_SC
    model = make_model(w)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        ws = om.Weights(w, keep_layers=True)
        okv = om.prefill(ws, prompt[0].cpu().numpy())
        p, seed, k = an.Params(), 5, 3
        canvas = an.initial_canvas(seed, w.canvas, w.vocab)
        z0 = om.selfcond(ws, om.denoise_forward(ws, okv, canvas, p.N, p.N, w.prompt_len,
                                                want_logits=True)["logits"])
        H, am, smp, z = binding.dg_anneal_forward(
            model, kv, torch.from_numpy(canvas.astype(np.int32)).reshape(1, -1).cuda(), k, [seed],
            p, z_in=torch.from_numpy(z0).reshape(1, w.canvas, w.d_model).cuda(), want_z=True)
        binding.dg_sync_status(model)
        ts, drawn, _, oz = _anneal_sc_oracle(ws, okv, canvas, k, seed, p, z0, w, True)
        assert max_abs_rel(H[0].cpu().numpy(), ts["H64"]) < 1e-6
        assert np.array_equal(am[0].cpu().numpy(), ts["argmax"])
        assert np.array_equal(smp[0].cpu().numpy(), drawn)
        assert max_abs_rel(z[0].cpu().numpy(), oz) < 1e-9
        kv.close()
    finally:
        model.close()


def test_small_bf16_annealed_forward_with_selfcond():
    """The tensor-core epilogue that both draws (tempered) and stores p0 (temperature
    1): entropies and z within 2e-2, draws equal where the race is decided."""
    from masked_discrete_diffusion_b200 import binding
    w = workloads.SMALL_BF16_SC
    model = make_model(w)
    try:
        prompt = model_inputs.prompt(w, "cuda")
        kv = binding.dg_prefill(model, prompt)
        ws = om.Weights(w, keep_layers=True)
        p, k = an.Params(), 4
        seeds = [41 + b for b in range(w.batch)]
        canvas = np.stack([an.initial_canvas(s, w.canvas, w.vocab) for s in seeds])
        z0 = [om.selfcond(ws, om.prefill_then_forward(ws, prompt[b].cpu().numpy(), canvas[b],
                                                      p.N, p.N, want_logits=True)["logits"])
              for b in range(w.batch)]
        H, am, smp, z = binding.dg_anneal_forward(
            model, kv, torch.from_numpy(canvas.astype(np.int32)).cuda(), k, seeds, p,
            z_in=torch.from_numpy(np.stack(z0).astype(np.float32)).cuda(), want_z=True)
        binding.dg_sync_status(model)
        decided = total = 0
        for b in range(w.batch):
            ts, drawn, gap, oz = _anneal_sc_oracle(ws, prompt[b].cpu().numpy(), canvas[b], k,
                                                   seeds[b], p, z0[b], w, False)
            assert max_abs_rel(H[b].cpu().numpy(), ts["H64"]) < 2e-2
            assert max_abs_rel(z[b].cpu().numpy(), oz) < 2e-2
            ok = gap > 0.05
            assert np.array_equal(smp[b].cpu().numpy()[ok], drawn[ok])
            decided += int(ok.sum())
            total += len(ok)
        assert decided >= 0.9 * total
        kv.close()
    finally:
        model.close()
