"""The binding's checks on caller tensors, which run before any library call (no GPU).

Every C entry point takes bare device pointers and reads or writes as many elements of
one type as the model, the KV handle or the sizes it is given imply; a tensor of
another dtype or shape, or on the host, must be refused in Python, before a kernel
could read or write outside it."""
import pytest
import torch

from masked_discrete_diffusion_b200 import binding


def test_arg_rejects_wrong_dtype_shape_and_device():
    ok = torch.zeros(2, 8, dtype=torch.int32)
    assert binding._arg(None, "x", torch.int32, (2, 8)) is None
    with pytest.raises(ValueError, match="int32 of shape"):
        binding._arg(ok.to(torch.int64), "x", torch.int32, (2, 8))
    with pytest.raises(ValueError, match="of shape"):
        binding._arg(ok[:, :4], "x", torch.int32, (2, 8))
    with pytest.raises(ValueError, match="of shape"):
        binding._arg(ok.reshape(16), "x", torch.int32, (2, 8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding._arg(ok, "x", torch.int32, (2, 8))
    with pytest.raises(ValueError, match="must be a tensor"):
        binding._arg([[0] * 8] * 2, "x", torch.int32, (2, 8))


def test_eb_sample_checks_before_any_launch():
    H = torch.zeros(1, 8)
    a = torch.zeros(1, 8, dtype=torch.int32)
    m = torch.ones(1, 8, dtype=torch.uint8)
    with pytest.raises(ValueError, match="entropy"):
        binding.dg_eb_sample(H.double(), a, a, m, 1, 1.0)
    with pytest.raises(ValueError, match="entropy must be a 2-D"):
        binding.dg_eb_sample(H[0], a, a, m, 1, 1.0)
    with pytest.raises(ValueError, match="entropy"):  # host tensors are refused too
        binding.dg_eb_sample(H, a, a, m, 1, 1.0)


def test_anneal_sample_requires_every_tensor():
    H = torch.zeros(1, 8)
    with pytest.raises(ValueError):
        binding.dg_anneal_sample(H, None, None, None, None, None, 0, 10, [1])
    with pytest.raises(ValueError, match="entropy must be a 2-D"):
        binding.dg_anneal_sample(H[0], None, None, None, None, None, 0, 10, [1])


def test_z_type_follows_the_model_precision():
    class M:  # the attribute the helper reads
        def __init__(self, dt):
            self.cfg = type("C", (), {"dtype": dt})()
    assert binding._z_type(M(binding.DG_F32)) == torch.float64
    assert binding._z_type(M(binding.DG_BF16)) == torch.float32
    assert binding._z_type(M(binding.DG_BF16_FP8EXP)) == torch.float32
