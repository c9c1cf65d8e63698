"""A device-side bounded wait that runs out is reported, and the model stays usable.

Every wait inside the library's kernels gives up after a time limit, records
DG_ERR_TIMEOUT in the model's device error word and unwinds instead of spinning
forever.  dg_debug_stall_experts makes the next routed-expert launch wait for a
gate/up unit that never comes (a chunk counter that can never reach its target) with
every wait of that launch limited to a few milliseconds: the launch must end, the next
dg_sync_status must return DG_ERR_TIMEOUT, and the following calls must run normally
and reproduce the result of a call made before the stall, bit for bit.  No GPU fault
is involved: the kernel only stops waiting.
"""
import pytest
import torch

from synth import gen, workloads

from gpu_helpers import make_model

pytestmark = pytest.mark.gpu
W = workloads.SMALL_BF16
DG_ERR_TIMEOUT = 5


def test_expert_wait_runs_out_and_is_reported():
    from masked_discrete_diffusion_b200 import binding
    model = make_model(W)
    try:
        n = 96
        x = gen.normal_values(3, "timeout.x", 0, n * W.d_model, 1.0, "cuda").reshape(n, W.d_model)
        ref = binding.dg_op_moe(model, 0, x)
        binding.dg_sync_status(model)
        binding.dg_debug_stall_experts(model, 5_000_000)      # 5 ms per wait
        binding.dg_op_moe(model, 0, x)
        with pytest.raises(binding.DGError) as e:
            binding.dg_sync_status(model)
        assert e.value.status == DG_ERR_TIMEOUT
        # the error word was cleared by the report; the next calls are normal
        out = binding.dg_op_moe(model, 0, x)
        binding.dg_sync_status(model)
        assert torch.equal(out, ref)
        out = binding.dg_op_moe(model, 1, x)
        binding.dg_sync_status(model)
        assert torch.isfinite(out).all()
    finally:
        model.close()


def test_stall_hook_rejects_bad_limits_and_other_models():
    from masked_discrete_diffusion_b200 import binding
    model = make_model(W)
    try:
        for bad in (0, 99_999, 2_000_000_000):
            with pytest.raises(binding.DGError) as e:
                binding.dg_debug_stall_experts(model, bad)
            assert e.value.status == 1
    finally:
        model.close()
    tiny = make_model(workloads.TINY_F32)
    try:
        with pytest.raises(binding.DGError) as e:
            binding.dg_debug_stall_experts(tiny, 1_000_000)
        assert e.value.status == 2
    finally:
        tiny.close()
