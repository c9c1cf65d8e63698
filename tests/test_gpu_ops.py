"""Single kernel groups of the bf16 path vs the oracle's definition of the step.

* the tcgen05 dense GEMM vs an fp64 matrix product of the same bf16 operands,
  on shapes spanning several tiles with ragged row tails;
* the MoE block (router, permutation, grouped tcgen05 expert GEMMs, shared
  expert, combine) vs oracle.model.moe on the same fp32 rows.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from synth import gen, workloads

from gpu_helpers import make_model, max_abs_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def small():
    m = make_model(workloads.SMALL_BF16)
    yield m
    m.close()


# (256, 2048, 2048), (256, 4096, 2048) and (100, 1024, 512) run as clusters that split K
# (4, 2 and 4 ways) and reduce the partial tiles through distributed shared memory.
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (200, 192, 128), (300, 64, 64), (1, 64, 64),
                                   (520, 4096, 2048), (256, 2048, 2048), (256, 4096, 2048),
                                   (100, 1024, 512)])
def test_tc_gemm_matches_fp64(small, M, N, K):
    from masked_discrete_diffusion_b200 import binding
    A = gen.normal_values(1, f"A{M}", 0, M * K, 1.0, "cuda").reshape(M, K).to(torch.bfloat16)
    W = gen.normal_values(1, f"W{N}", 0, N * K, 0.05, "cuda").reshape(N, K).to(torch.bfloat16)
    out = binding.dg_op_gemm(small, A, W)
    binding.dg_sync_status(small)
    ref = A.double().cpu().numpy() @ W.double().cpu().numpy().T
    assert max_abs_rel(out.cpu().numpy(), ref) < 1e-4


@pytest.mark.parametrize("wname,n", [("small-bf16", 288), ("small-bf16", 7), ("layer1-bf16", 256)])
def test_moe_block_matches_oracle(wname, n, small):
    from masked_discrete_diffusion_b200 import binding
    w = workloads.get(wname)
    model = small if wname == "small-bf16" else make_model(w)
    x = gen.normal_values(2, f"x{n}", 0, n * w.d_model, 1.0, "cuda").reshape(n, w.d_model)
    out = binding.dg_op_moe(model, 0, x)
    binding.dg_sync_status(model)
    ws = om.Weights(w, keep_layers=False)
    xd = x.double().cpu().numpy()
    y, idx, g, logits = om.moe(om.rmsnorm(xd, w.rms_eps), ws.layer(0), w.top_k)
    want = xd + y
    got = out.cpu().numpy()
    # rows whose top-k set is decided well above the rounding of the bf16 path
    srt = np.sort(logits, axis=1)[:, ::-1]
    decided = (srt[:, w.top_k - 1] - srt[:, w.top_k]) > 1e-3
    assert decided.mean() > 0.9
    assert max_abs_rel(got[decided] - xd[decided], y[decided]) < 2e-2
    if model is not small:
        model.close()
