"""The allocation-free LM-head entropy entry point agrees with the regular path.

Some callers cannot allocate device memory (their allocator belongs to another
runtime, or their device memory is fixed before they start), so the library
offers dg_lmhead_entropy_noalloc, which keeps its scratch in a static device
array instead of a workspace.  This test runs the regular forward
(dg_debug_forward, whose LM head uses the model's allocated workspace), takes
the final residual rows it reports, and feeds them to the allocation-free entry
point twice in a row; both calls must reproduce the regular entropies and argmax.
"""
import numpy as np
import pytest
import torch

from synth import model_inputs, workloads

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
