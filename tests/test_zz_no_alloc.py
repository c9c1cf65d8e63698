"""The allocation-free LM-head entropy entry point agrees with the regular path.

Some callers cannot allocate device memory (their allocator belongs to another
runtime, or their device memory is fixed before they start), so the library
offers dg_lmhead_entropy_noalloc, which keeps its scratch in a static device
array instead of a workspace.  This test runs the regular forward
(dg_debug_forward, whose LM head uses the model's allocated workspace), takes
the final residual rows it reports, and feeds them to the allocation-free entry
point twice in a row; both calls must reproduce the regular entropies and argmax.
It is also checked against the oracle's LM-head statistics on seeded rows, over
shapes that exercise fewer than 128 rows, a single row, the full 256 rows, a
vocabulary smaller than one 256-column tile and one with a ragged last tile.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from synth import gen, model_inputs, workloads

from gpu_helpers import make_model, max_abs_rel

pytestmark = pytest.mark.gpu
W = workloads.SMALL_BF16
TOL = 2e-2   # the bf16 tolerance used by the parity tests


def test_noalloc_entropy_matches_regular_path():
    from masked_discrete_diffusion_b200 import binding
    model = make_model(W)
    try:
        prompt = model_inputs.prompt(W, "cuda")[:2].contiguous()   # 2 canvases: M = 192 rows
        kv = binding.dg_prefill(model, prompt)
        canvas = torch.full((2, W.canvas), W.mask_id, dtype=torch.int32, device="cuda")
        canvas[:, ::7] = 11
        ent, am, _, hidden = binding.dg_debug_forward(model, kv, canvas, 3, W.T, hidden=True)
        binding.dg_sync_status(model)
        ref_e = ent.reshape(-1).cpu().numpy()
        ref_a = am.reshape(-1).cpu().numpy()
        lm = model.tensors["lm_head"]
        for _ in range(2):
            e, a = binding.dg_lmhead_entropy_noalloc(hidden, lm, W.rms_eps, W.logit_scale)
            torch.cuda.synchronize()
            e, a = e.cpu().numpy(), a.cpu().numpy()
            assert np.all(np.isfinite(e)) and np.all(a >= 0)
            assert max_abs_rel(e, ref_e) < TOL
            assert np.array_equal(a, ref_a)
        kv.close()
    finally:
        model.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from masked_discrete_diffusion_b200 import binding
    h = torch.zeros(257, 64, dtype=torch.float32, device="cuda")
    lm = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.DGError) as e:
        binding.dg_lmhead_entropy_noalloc(h, lm, 1e-6, 8.0)
    assert e.value.status == 1
    with pytest.raises(binding.DGError):
        binding.dg_lmhead_entropy_noalloc(h[:8], torch.zeros(262145, 64, dtype=torch.bfloat16,
                                                             device="cuda"), 1e-6, 8.0)


@pytest.mark.parametrize("M,V,d", [(1, 1000, 64), (100, 200, 256), (256, 1000, 256),
                                   (100, 1000, 64)])
def test_noalloc_matches_oracle(M, V, d):
    from masked_discrete_diffusion_b200 import binding
    w = W.with_(name=f"noalloc-{M}-{V}-{d}", vocab=V, d_model=d)
    hidden = gen.normal_values(w.seed, "noalloc.hidden", 0, M * d, 1.0).reshape(M, d)
    lm = model_inputs.weight(w, "lm_head", (V, d)).cuda()
    ref = om.lm_head_stats(om.Weights(w), hidden.double().numpy())
    # bf16 rounding of the normalised rows moves logit j of a row by at most
    # scale * 2^-8 * sum_k |xn_k W_jk| (half an ulp of bf16 is 2^-9 relative; doubled
    # for the fp32 accumulation); argmax is compared where the top-2 gap exceeds twice that
    xn = om.rmsnorm(hidden.double().numpy(), w.rms_eps)
    wabs = np.abs(lm.float().cpu().double().numpy())
    bound = w.logit_scale * 2.0 ** -8 * (np.abs(xn) @ wabs.T).max(axis=1)
    decided = ref["margin"] > 2 * bound
    for _ in range(2):
        e, a = binding.dg_lmhead_entropy_noalloc(hidden.cuda(), lm, w.rms_eps, w.logit_scale)
        torch.cuda.synchronize()
        e, a = e.cpu().numpy(), a.cpu().numpy()
        assert max_abs_rel(e, ref["H"]) < TOL
        assert np.all(e >= 0) and np.all(e <= np.log(V) + 1e-3)
        assert np.array_equal(a[decided], ref["argmax"][decided])
        assert np.all((a >= 0) & (a < V))
