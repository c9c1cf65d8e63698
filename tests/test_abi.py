"""The C-ABI library builds, loads and exports every entry point include/*.h declares;
host-side argument validation rejects bad calls before touching the device."""
import ctypes
import glob
import os
import re

import pytest
import torch

from masked_discrete_diffusion_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(dg_\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lib.dg_status_str(0) == b"DG_OK"
    assert lib.dg_status_str(1) == b"DG_ERR_INVALID_ARG"
    assert lib.dg_status_str(5) == b"DG_ERR_TIMEOUT"


def test_host_validation_without_device(lib):
    vp = ctypes.c_void_p
    # null pointers and bad scalars are rejected before any CUDA call
    assert lib.dg_eb_sample(None, None, None, None, 1, 8, 1, 1.0, None, None) == 1
    fake = vp(16)
    assert lib.dg_eb_sample(fake, fake, fake, fake, 1, 8, 0, 1.0, None, None) == 1   # steps 0
    assert lib.dg_eb_sample(fake, fake, fake, fake, 1, 2048, 1, 1.0, None, None) == 1
    assert lib.dg_eb_sample(fake, fake, fake, fake, 1, 8, 1, float("nan"), None, None) == 1
    assert lib.dg_eb_sample(fake, fake, fake, fake, 1, 8, 1, -0.5, None, None) == 1
    assert b"gamma" in lib.dg_last_error()
    out = vp()
    assert lib.dg_model_create(None, None, ctypes.byref(out)) == 1
    cfg = binding.dg_config(n_layers=1, d_model=64, n_q_heads=3, n_kv_heads=2, head_dim=16,
                            n_experts=8, top_k=2, expert_inter=8, shared_inter=8, vocab=16,
                            window=4, canvas=8, rope_base=1e4, rms_eps=1e-6, logit_scale=8,
                            dtype=0, max_batch=1, max_prompt=8)
    w = binding.dg_weights()
    assert lib.dg_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(out)) == 1
    assert b"multiple" in lib.dg_last_error()
    # NVFP4 expert weights: d and I multiples of 32 and at most 2048 (a unit's block scales
    # are staged in shared memory), checked before any weight pointer or device call
    for d, inter in ((2048 + 32, 768), (2048, 48), (2056, 768)):
        cfg4 = binding.dg_config(n_layers=1, d_model=d, n_q_heads=16, n_kv_heads=8,
                                 head_dim=128, n_experts=8, top_k=2, expert_inter=inter,
                                 shared_inter=64, vocab=16, window=4, canvas=8,
                                 rope_base=1e4, rms_eps=1e-6, logit_scale=8,
                                 dtype=binding.DG_BF16_FP4EXP, max_batch=1, max_prompt=8)
        assert lib.dg_model_create(ctypes.byref(cfg4), ctypes.byref(w), ctypes.byref(out)) == 1
        assert b"NVFP4" in lib.dg_last_error(), (d, inter, lib.dg_last_error())
    cfg5 = binding.dg_config(n_layers=1, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16,
                             n_experts=8, top_k=2, expert_inter=64, shared_inter=64, vocab=16,
                             window=4, canvas=8, rope_base=1e4, rms_eps=1e-6, logit_scale=8,
                             dtype=4, max_batch=1, max_prompt=8)
    assert lib.dg_model_create(ctypes.byref(cfg5), ctypes.byref(w), ctypes.byref(out)) == 1
    assert b"dtype" in lib.dg_last_error()
    assert lib.dg_model_destroy(None) == 0 and lib.dg_kv_destroy(None) == 0


def test_kv_destroy_after_model_destroy_is_safe_without_device(lib):
    # only null handles can be exercised without a GPU; the ordering itself is
    # covered on the GPU by the model/KV lifetime test
    assert lib.dg_kv_destroy(None) == 0 and lib.dg_model_destroy(None) == 0


def test_null_handles_and_bad_sizes_rejected_without_device(lib):
    """Every entry point that takes a handle or buffers checks them before any CUDA call
    (DG_ERR_INVALID_ARG = 1), so these run on a machine without a GPU."""
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    fake = vp(256)
    n = i64()
    calls = {
        "dg_sync_status": (None, None),
        "dg_prefill": (None, fake, 1, 8, ctypes.byref(vp()), None),
        "dg_kv_info": (None, None, None, None),
        "dg_kv_read": (None, fake, fake, None),
        "dg_denoise_step": (None, None, fake, fake, 1, 4, 1.0, fake, fake, fake, None),
        "dg_generate_block": (None, None, 4, 1.0, fake, None, None, None),
        "dg_debug_forward": (None, None, fake, 1, 4, fake, fake, None, None, None),
        "dg_profile_start": (None, 0),
        "dg_profile_stop": (None, None, None),
        "dg_launch_count": (None, ctypes.byref(n)),
        "dg_expert_units": (None, ctypes.byref(n)),
        "dg_block_loop_launches": (None, ctypes.byref(n)),
        "dg_op_gemm": (None, fake, fake, fake, 1, 64, 64, None),
        "dg_op_moe": (None, 0, fake, fake, 1, None),
        "dg_debug_stall_experts": (None, 1000000),
        "dg_prefill_into": (None, fake, 1, 1, fake, None),
        "dg_append_block": (None, fake, fake, None),
        "dg_generate_blocks": (None, fake, 1, 1, 1.0, fake, None, None),
    }
    for name, args in calls.items():
        assert getattr(lib, name)(*args) == 1, name
        assert lib.dg_last_error(), name
    # the allocation-free LM head: pointers, ranges and alignment
    na = lib.dg_lmhead_entropy_noalloc
    ok = dict(h=fake, w=fake, M=256, V=262144, d=2048, eps=1e-6, s=8.0, e=fake, a=fake)

    def call(**kw):
        a = dict(ok, **kw)
        return na(a["h"], a["w"], a["M"], a["V"], a["d"], a["eps"], a["s"], a["e"], a["a"], None)

    for bad in (dict(h=None), dict(w=None), dict(e=None), dict(a=None), dict(M=0),
                dict(M=257), dict(V=0), dict(V=262145), dict(d=32), dict(d=100),
                dict(d=4160), dict(w=vp(264)), dict(eps=-1.0), dict(s=float("inf")),
                dict(s=float("nan"))):
        assert call(**bad) == 1, bad


def test_noalloc_binding_rejects_bad_tensors_before_any_launch():
    """The Python wrapper of the allocation-free entry point checks dtype, rank, the
    shared width and the device before calling into the library (CPU tensors here:
    no call can reach the GPU)."""
    from masked_discrete_diffusion_b200 import binding
    f32 = torch.zeros(4, 64, dtype=torch.float32)
    b16 = torch.zeros(8, 64, dtype=torch.bfloat16)
    bad = [
        (f32.to(torch.bfloat16), b16, "hidden"),                         # hidden not fp32
        (f32.reshape(-1), b16, "hidden"),                                # hidden not 2-D
        (f32, b16.float(), "lm_head"),                                   # lm_head not bf16
        (f32, b16.reshape(8, 8, 8), "lm_head"),                          # lm_head not 2-D
        (f32, torch.zeros(8, 128, dtype=torch.bfloat16), "columns"),     # widths differ
        (f32, b16, "CUDA"),                                              # not on a GPU
    ]
    for h, w, what in bad:
        with pytest.raises(ValueError, match=what):
            binding.dg_lmhead_entropy_noalloc(h, w, 1e-6, 8.0)


def _header_struct_types(name: str) -> list[str]:
    """The C type of each field of `name`, in order (as _header_struct_fields)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "include", "dg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct %s \{(.*?)\} %s;" % (name, name), src, flags=re.S).group(1)
    types = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        first, *others = [p.strip() for p in decl.split(",")]
        words = first.split()
        t = " ".join(words[:-1]) + ("*" if words[-1].startswith("*") else "")
        types += [t] * (1 + len(others))
    return types


def _header_struct_fields(name: str) -> list[str]:
    """Field names, in order, of `typedef struct name { ... } name;` in include/dg.h
    (comments stripped; one declaration per field, several names per line allowed)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "include", "dg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct %s \{(.*?)\} %s;" % (name, name), src, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        # "int32_t a, b, c", "const void* p" or "float x": the first name ends the type
        first, *others = [p.strip() for p in decl.split(",")]
        fields += [first.split()[-1].lstrip("*")] + [o.lstrip("*") for o in others]
    return fields


def test_binding_structs_match_the_header():
    """The ctypes structs pass field offsets by declaration order: a field out of order
    or missing would hand the library a wrong pointer or size."""
    from masked_discrete_diffusion_b200 import binding
    assert [f for f, _ in binding.dg_config._fields_] == _header_struct_fields("dg_config")
    assert list(binding._LAYER_FIELDS) == _header_struct_fields("dg_layer_weights")
    assert [f for f, _ in binding.dg_weights._fields_] == _header_struct_fields("dg_weights")
    assert [f for f, _ in binding.dg_anneal_params._fields_] == \
        _header_struct_fields("dg_anneal_params")
    # and the scalar structs' field types
    import ctypes
    ctype_of = {"int32_t": ctypes.c_int32, "float": ctypes.c_float}
    for st, name in ((binding.dg_config, "dg_config"),
                     (binding.dg_anneal_params, "dg_anneal_params")):
        want = [ctype_of[t] for t in _header_struct_types(name)]
        assert [t for _, t in st._fields_] == want, name
