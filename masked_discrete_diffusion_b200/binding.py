"""ctypes binding of libdg (include/dg.h): argument marshalling only.

Every function below forwards to the C entry point of the same name; device
buffers are passed as torch CUDA tensors (PyTorch supplies device memory and
streams).  There is no fallback: if libdg.so is missing or a call fails, an
exception is raised.

The calls come in four groups: model and batch set-up; one denoising forward
with the entropy-bounded (EB) draw and the whole EB generation loop, for one
block or with block appends; the annealed sampler (tempered Gumbel-max draws,
acceptance of the lowest-entropy prefix, re-noising of the rest), as one forward
or as the whole loop; and self-conditioning, where the tensor z that a forward
leaves behind is fed into the canvas input of the next one.  Tensors for z hold
the model's accumulate type: fp64 for the f32 model, fp32 for the bf16 ones.
"""
from __future__ import annotations

import ctypes
import os
import weakref

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_F32, DG_BF16, DG_BF16_FP8EXP, DG_BF16_FP4EXP = 0, 1, 2, 3
_DTYPES = {"f32": DG_F32, "bf16": DG_BF16, "bf16_fp8exp": DG_BF16_FP8EXP,
           "bf16_fp4exp": DG_BF16_FP4EXP}


class DGError(RuntimeError):
    def __init__(self, status: int, name: str, detail: str):
        super().__init__(f"{name}: {detail}")
        self.status = status
        self.name = name


class dg_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_layers", "d_model", "n_q_heads", "n_kv_heads", "head_dim", "n_experts", "top_k",
        "expert_inter", "shared_inter", "vocab", "window", "canvas")] + [
        ("rope_base", ctypes.c_float), ("rms_eps", ctypes.c_float),
        ("logit_scale", ctypes.c_float), ("dtype", ctypes.c_int32),
        ("max_batch", ctypes.c_int32), ("max_prompt", ctypes.c_int32),
        ("sc_inter", ctypes.c_int32)]


_LAYER_FIELDS = ("wqkv", "wo", "router", "gate", "up", "down", "gate_scale", "up_scale",
                 "down_scale", "sgate", "sup", "sdown", "gate_tscale", "up_tscale",
                 "down_tscale")


class dg_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _LAYER_FIELDS]


class dg_weights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("layers", ctypes.POINTER(dg_layer_weights)), ("sc_gate", ctypes.c_void_p),
                ("sc_up", ctypes.c_void_p), ("sc_down", ctypes.c_void_p)]


_lib = None


class dg_anneal_params(ctypes.Structure):
    """Constants of the annealed entropy-bounded sampler (defaults: the Report's)."""
    _fields_ = [("N", ctypes.c_int32), ("b", ctypes.c_float), ("tau_max", ctypes.c_float),
                ("tau_min", ctypes.c_float), ("e_stop", ctypes.c_float)]


def anneal_params(N: int = 48, b: float = 0.1, tau_max: float = 0.8, tau_min: float = 0.4,
                  e_stop: float = 0.005) -> dg_anneal_params:
    return dg_anneal_params(N, b, tau_max, tau_min, e_stop)


def _params(p) -> dg_anneal_params:
    if p is None:
        return anneal_params()
    if isinstance(p, dg_anneal_params):
        return p
    return anneal_params(p.N, p.b, p.tau_max, p.tau_min, p.e_stop)   # any object with the fields


def _seeds(seeds, B: int) -> torch.Tensor:
    """[B] uint64 seeds on the device (int64 storage); ints or a tensor."""
    if not torch.is_tensor(seeds):
        seeds = torch.tensor([int(x) - (1 << 64) if int(x) >= (1 << 63) else int(x)
                              for x in seeds], dtype=torch.int64)
    if seeds.dtype not in (torch.int64, torch.uint64) or seeds.numel() != B:
        raise ValueError(f"expected {B} 64-bit seeds")
    return seeds.reshape(B).to("cuda").contiguous()


def lib() -> ctypes.CDLL:
    """Load libdg.so (built in-tree by build.py); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdg.so not built ({LIB_PATH}); run "
                               "`python -m masked_discrete_diffusion_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        L.dg_status_str.restype = ctypes.c_char_p
        L.dg_status_str.argtypes = [ctypes.c_int]
        L.dg_last_error.restype = ctypes.c_char_p
        L.dg_last_error.argtypes = []
        sigs = {
            "dg_model_create": [ctypes.POINTER(dg_config), ctypes.POINTER(dg_weights),
                                ctypes.POINTER(vp)],
            "dg_model_destroy": [vp],
            "dg_sync_status": [vp, vp],
            "dg_prefill": [vp, vp, i32, i32, ctypes.POINTER(vp), vp],
            "dg_prefill_into": [vp, vp, i32, i32, vp, vp],
            "dg_append_block": [vp, vp, vp, vp],
            "dg_generate_blocks": [vp, vp, i32, i32, f32, vp, vp, vp],
            "dg_kv_destroy": [vp],
            "dg_kv_info": [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)],
            "dg_kv_read": [vp, vp, vp, vp],
            "dg_denoise_step": [vp, vp, vp, vp, i32, i32, f32, vp, vp, vp, vp],
            "dg_generate_block": [vp, vp, i32, f32, vp, vp, vp, vp],
            "dg_eb_sample": [vp, vp, vp, vp, i32, i32, i32, f32, vp, vp],
            "dg_debug_forward": [vp, vp, vp, i32, i32, vp, vp, vp, vp, vp],
            "dg_profile_start": [vp, i32],
            "dg_profile_stop": [vp, vp, vp],
            "dg_launch_count": [vp, ctypes.POINTER(ctypes.c_int64)],
            "dg_expert_units": [vp, ctypes.POINTER(ctypes.c_int64)],
            "dg_block_loop_launches": [vp, ctypes.POINTER(ctypes.c_int64)],
            "dg_lmhead_entropy_noalloc": [vp, vp, i32, i32, i32, f32, f32, vp, vp, vp],
            "dg_op_gemm": [vp, vp, vp, vp, i32, i32, i32, vp],
            "dg_op_moe": [vp, i32, vp, vp, i32, vp],
            "dg_debug_stall_experts": [vp, ctypes.c_int64],
            "dg_generate_block_annealed": [vp, vp, ctypes.POINTER(dg_anneal_params), vp, vp,
                                           vp, vp],
            "dg_anneal_forward": [vp, vp, vp, i32, ctypes.POINTER(dg_anneal_params), vp, vp,
                                  vp, vp, vp, vp, vp],
            "dg_anneal_sample": [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                 ctypes.POINTER(dg_anneal_params), vp, vp],
            "dg_anneal_init": [vp, vp, vp, i32, i32, i32, vp, vp],
            "dg_set_selfcond": [vp, i32],
            "dg_selfcond_forward": [vp, vp, vp, i32, i32, vp, vp, vp, vp, vp],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        _lib = L
    return _lib


def exported_symbols():
    return [n for n in ("dg_status_str", "dg_last_error", "dg_model_create", "dg_model_destroy",
                        "dg_sync_status", "dg_prefill", "dg_kv_destroy", "dg_kv_info",
                        "dg_kv_read", "dg_denoise_step", "dg_generate_block", "dg_eb_sample",
                        "dg_debug_forward", "dg_profile_start", "dg_profile_stop",
                        "dg_launch_count", "dg_op_gemm", "dg_op_moe", "dg_expert_units",
                        "dg_lmhead_entropy_noalloc", "dg_block_loop_launches",
                        "dg_debug_stall_experts", "dg_prefill_into", "dg_append_block",
                        "dg_generate_blocks", "dg_generate_block_annealed",
                        "dg_anneal_forward", "dg_anneal_sample", "dg_anneal_init",
                        "dg_set_selfcond", "dg_selfcond_forward")
            if hasattr(lib(), n)]


def _check(status: int):
    if status != 0:
        L = lib()
        raise DGError(status, L.dg_status_str(status).decode(), L.dg_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _arg(t, name: str, dtype, shape):
    """Device pointer of a caller tensor after checking what the C entry point assumes
    about it: a contiguous CUDA tensor on the current device with exactly this dtype and
    shape (the library reads or writes that many elements of that type, so anything
    else would be read or written out of bounds, or misread).  None stays None."""
    if t is None:
        return None
    if not torch.is_tensor(t):
        raise ValueError(f"{name} must be a tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {dtype} of shape {tuple(shape)}, got {t.dtype} "
                         f"{tuple(t.shape)}")
    if not t.is_cuda or t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} must be a CUDA tensor on the current device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _z_type(model) -> torch.dtype:
    """Accumulate type of a model: that of its self-conditioning signal z."""
    return torch.float64 if model.cfg.dtype == DG_F32 else torch.float32


def _stream(stream=None) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def make_config(w, max_batch: int | None = None, max_prompt: int | None = None) -> dg_config:
    """dg_config from a workload description (any object with the workload fields)."""
    return dg_config(
        n_layers=w.n_layers, d_model=w.d_model, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
        head_dim=w.head_dim, n_experts=w.n_experts, top_k=w.top_k, expert_inter=w.expert_inter,
        shared_inter=w.shared_inter, vocab=w.vocab, window=w.window, canvas=w.canvas,
        rope_base=w.rope_base, rms_eps=w.rms_eps, logit_scale=w.logit_scale,
        dtype=_DTYPES[w.dtype], max_batch=max_batch or w.batch,
        max_prompt=max_prompt or w.prompt_len, sc_inter=getattr(w, "sc_inter", 0))


class Model:
    """A dg_model handle; `tensors` maps weight names (see include/dg.h) to CUDA tensors
    and must stay alive as long as the model (the library borrows them)."""

    def __init__(self, cfg: dg_config, tensors: dict):
        self.cfg = cfg
        self.tensors = tensors
        n = cfg.n_layers
        self._layers = (dg_layer_weights * n)()
        for l in range(n):
            for f in _LAYER_FIELDS:
                setattr(self._layers[l], f, _ptr(tensors.get(f"l{l}.{f}")))
        self._w = dg_weights(tok_emb=_ptr(tensors["tok_emb"]), lm_head=_ptr(tensors["lm_head"]),
                             layers=self._layers, sc_gate=_ptr(tensors.get("sc.gate")),
                             sc_up=_ptr(tensors.get("sc.up")), sc_down=_ptr(tensors.get("sc.down")))
        h = ctypes.c_void_p()
        _check(lib().dg_model_create(ctypes.byref(cfg), ctypes.byref(self._w), ctypes.byref(h)))
        self.handle = h
        self._kvs = weakref.WeakSet()

    def close(self):
        """Destroys the model after every KV cache created from it."""
        for kv in list(getattr(self, "_kvs", ())):
            kv.close()
        if getattr(self, "handle", None):
            _check(lib().dg_model_destroy(self.handle))
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


class KV:
    def __init__(self, model: Model, handle):
        self.model = model
        self.handle = handle
        model._kvs.add(self)
        B, P, W = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().dg_kv_info(handle, ctypes.byref(B), ctypes.byref(P), ctypes.byref(W)))
        self.B, self.P, self.W = B.value, P.value, W.value

    def refresh(self):
        """Re-reads B, P and W (they change when blocks are appended)."""
        B, P, W = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().dg_kv_info(self.handle, ctypes.byref(B), ctypes.byref(P), ctypes.byref(W)))
        self.B, self.P, self.W = B.value, P.value, W.value

    def close(self):
        if getattr(self, "handle", None):
            _check(lib().dg_kv_destroy(self.handle))
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


def dg_sync_status(model: Model, stream=None):
    _check(lib().dg_sync_status(model.handle, _stream(stream)))


def dg_prefill(model: Model, prompt: torch.Tensor, stream=None) -> KV:
    if not torch.is_tensor(prompt) or prompt.dim() != 2:
        raise ValueError("prompt must be a 2-D int32 tensor")
    pp = _arg(prompt, "prompt", torch.int32, prompt.shape)
    h = ctypes.c_void_p()
    _check(lib().dg_prefill(model.handle, pp, prompt.shape[0], prompt.shape[1],
                            ctypes.byref(h), _stream(stream)))
    return KV(model, h)


def dg_prefill_into(model: Model, prompt: torch.Tensor, kv: KV, stream=None) -> KV:
    """Causal pass of prompt [B, P] into an existing handle of the same B."""
    if not torch.is_tensor(prompt) or prompt.dim() != 2:
        raise ValueError("prompt must be a 2-D int32 tensor")
    B, P = prompt.shape
    pp = _arg(prompt, "prompt", torch.int32, (B, P))
    _check(lib().dg_prefill_into(model.handle, pp, B, P, kv.handle, _stream(stream)))
    kv.refresh()
    return kv


def dg_append_block(model: Model, kv: KV, tokens: torch.Tensor, stream=None) -> KV:
    """Causal pass of the finished blocks tokens [B, C] into kv (the context grows by C)."""
    tp = _arg(tokens, "tokens", torch.int32, (kv.B, model.cfg.canvas))
    _check(lib().dg_append_block(model.handle, kv.handle, tp, _stream(stream)))
    kv.refresh()
    return kv


def dg_generate_blocks(model: Model, kv: KV, n_blocks: int, T: int, gamma: float,
                       stream=None):
    """n_blocks blocks one after the other; returns (tokens [B, n_blocks C],
    forwards [n_blocks, B]); kv ends extended by n_blocks - 1 blocks."""
    c = model.cfg
    out = torch.empty(kv.B, n_blocks * c.canvas, dtype=torch.int32, device="cuda")
    nf = torch.zeros(n_blocks, kv.B, dtype=torch.int32, device="cuda")
    _check(lib().dg_generate_blocks(model.handle, kv.handle, n_blocks, T, gamma, _ptr(out),
                                    _ptr(nf), _stream(stream)))
    kv.refresh()
    return out, nf


def dg_kv_read(kv: KV, stream=None):
    c = kv.model.cfg
    dt = torch.float64 if c.dtype == DG_F32 else torch.bfloat16
    shape = (c.n_layers, kv.B, c.n_kv_heads, kv.W, c.head_dim)
    k = torch.empty(shape, dtype=dt, device="cuda")
    v = torch.empty(shape, dtype=dt, device="cuda")
    _check(lib().dg_kv_read(kv.handle, _ptr(k), _ptr(v), _stream(stream)))
    return k, v


def dg_denoise_step(model: Model, kv: KV, canvas, mask, steps_left: int, T: int, gamma: float,
                    entropy=None, argmax=None, n_committed=None, stream=None):
    B, C = kv.B, model.cfg.canvas
    cp = _arg(canvas, "canvas", torch.int32, (B, C))
    mp = _arg(mask, "mask", torch.uint8, (B, C))
    entropy = entropy if entropy is not None else torch.empty(B, C, dtype=torch.float32, device="cuda")
    argmax = argmax if argmax is not None else torch.empty(B, C, dtype=torch.int32, device="cuda")
    n_committed = (n_committed if n_committed is not None
                   else torch.empty(B, dtype=torch.int32, device="cuda"))
    _check(lib().dg_denoise_step(model.handle, kv.handle, cp, mp, steps_left, T, gamma,
                                 _arg(entropy, "entropy", torch.float32, (B, C)),
                                 _arg(argmax, "argmax", torch.int32, (B, C)),
                                 _arg(n_committed, "n_committed", torch.int32, (B,)),
                                 _stream(stream)))
    return entropy, argmax, n_committed


def dg_generate_block(model: Model, kv: KV, T: int, gamma: float, canvas_out=None,
                      n_forwards=None, router_load=None, stream=None):
    c = model.cfg
    canvas_out = (canvas_out if canvas_out is not None
                  else torch.empty(kv.B, c.canvas, dtype=torch.int32, device="cuda"))
    _check(lib().dg_generate_block(model.handle, kv.handle, T, gamma,
                                   _arg(canvas_out, "canvas_out", torch.int32, (kv.B, c.canvas)),
                                   _arg(n_forwards, "n_forwards", torch.int32, (kv.B,)),
                                   _arg(router_load, "router_load", torch.int32,
                                        (c.n_layers, c.n_experts)),
                                   _stream(stream)))
    return canvas_out


def dg_eb_sample(entropy, argmax, canvas, mask, steps_left: int, gamma: float,
                 n_committed=None, stream=None):
    if not torch.is_tensor(entropy) or entropy.dim() != 2:
        raise ValueError("entropy must be a 2-D float32 tensor")
    B, C = entropy.shape
    ep = _arg(entropy, "entropy", torch.float32, (B, C))
    ap = _arg(argmax, "argmax", torch.int32, (B, C))
    cp = _arg(canvas, "canvas", torch.int32, (B, C))
    mp = _arg(mask, "mask", torch.uint8, (B, C))
    n_committed = (n_committed if n_committed is not None
                   else torch.empty(B, dtype=torch.int32, device="cuda"))
    _arg(n_committed, "n_committed", torch.int32, (B,))
    _check(lib().dg_eb_sample(ep, ap, cp, mp, B, C,
                              steps_left, gamma, _ptr(n_committed), _stream(stream)))
    return n_committed


def dg_generate_block_annealed(model: Model, kv: KV, seeds, params=None, canvas_out=None,
                               n_forwards=None, stream=None):
    """The annealed block; returns (canvas [B, C] int32, n_forwards [B] int32)."""
    c = model.cfg
    p = _params(params)
    sd = _seeds(seeds, kv.B)
    canvas_out = (canvas_out if canvas_out is not None
                  else torch.empty(kv.B, c.canvas, dtype=torch.int32, device="cuda"))
    n_forwards = (n_forwards if n_forwards is not None
                  else torch.empty(kv.B, dtype=torch.int32, device="cuda"))
    _check(lib().dg_generate_block_annealed(
        model.handle, kv.handle, ctypes.byref(p), _ptr(sd),
        _arg(canvas_out, "canvas_out", torch.int32, (kv.B, c.canvas)),
        _arg(n_forwards, "n_forwards", torch.int32, (kv.B,)), _stream(stream)))
    return canvas_out, n_forwards


def dg_anneal_forward(model: Model, kv: KV, canvas, k: int, seeds, params=None, z_in=None,
                      want_z=False, stream=None):
    """Step k's forward: (tempered entropy [B, C], argmax [B, C], Gumbel-max draw [B, C]),
    and with want_z the self-conditioning signal it hands on [B, C, d] (z_in: the one
    it receives, in the model's accumulate type)."""
    c = model.cfg
    B, C = kv.B, c.canvas
    zt = _z_type(model)
    cp = _arg(canvas, "canvas", torch.int32, (B, C))
    zp = _arg(z_in, "z_in", zt, (B, C, c.d_model))
    p = _params(params)
    sd = _seeds(seeds, kv.B)
    H = torch.empty(B, C, dtype=torch.float32, device="cuda")
    am = torch.empty(B, C, dtype=torch.int32, device="cuda")
    smp = torch.empty(B, C, dtype=torch.int32, device="cuda")
    z_out = torch.empty(B, C, c.d_model, dtype=zt, device="cuda") if want_z else None
    _check(lib().dg_anneal_forward(model.handle, kv.handle, cp, k, ctypes.byref(p),
                                   _ptr(sd), _ptr(H), _ptr(am), _ptr(smp), zp,
                                   _ptr(z_out), _stream(stream)))
    return (H, am, smp, z_out) if want_z else (H, am, smp)


def dg_anneal_sample(entropy, argmax, sampled, canvas, prev_argmax, state, k: int, V: int,
                     seeds, params=None, stream=None):
    """Step k's refinement in place (canvas, prev_argmax, state); returns n_accepted [B]."""
    if not torch.is_tensor(entropy) or entropy.dim() != 2:
        raise ValueError("entropy must be a 2-D float32 tensor")
    B, C = entropy.shape
    ptrs = [_arg(entropy, "entropy", torch.float32, (B, C))]
    for name, t in (("argmax", argmax), ("sampled", sampled), ("canvas", canvas),
                    ("prev_argmax", prev_argmax)):
        if t is None:
            raise ValueError(f"{name} is required")
        ptrs.append(_arg(t, name, torch.int32, (B, C)))
    if state is None:
        raise ValueError("state is required")
    ptrs.append(_arg(state, "state", torch.int32, (B,)))
    p = _params(params)
    sd = _seeds(seeds, B)
    nacc = torch.empty(B, dtype=torch.int32, device="cuda")
    _check(lib().dg_anneal_sample(*ptrs[:6], _ptr(nacc), B, C, V, k,
                                  ctypes.byref(p), _ptr(sd), _stream(stream)))
    return nacc


def dg_anneal_init(B: int, C: int, V: int, seeds, stream=None):
    """(x_1 [B, C] int32, prev_argmax [B, C] = -1, state [B] = 0)."""
    sd = _seeds(seeds, B)
    canvas = torch.empty(B, C, dtype=torch.int32, device="cuda")
    prev = torch.empty(B, C, dtype=torch.int32, device="cuda")
    state = torch.empty(B, dtype=torch.int32, device="cuda")
    _check(lib().dg_anneal_init(_ptr(canvas), _ptr(prev), _ptr(state), B, C, V, _ptr(sd),
                                _stream(stream)))
    return canvas, prev, state


def dg_set_selfcond(model: Model, on: bool):
    _check(lib().dg_set_selfcond(model.handle, 1 if on else 0))


def dg_selfcond_forward(model: Model, kv: KV, canvas, steps_left: int, T: int, z_in=None,
                        stream=None):
    """(entropy [B, C], argmax [B, C], z_out [B, C, d]); z in the model's accumulate type
    (float64 for the fp32 model, float32 otherwise)."""
    c = model.cfg
    B, C = kv.B, c.canvas
    zt = _z_type(model)
    cp = _arg(canvas, "canvas", torch.int32, (B, C))
    zp = _arg(z_in, "z_in", zt, (B, C, c.d_model))
    H = torch.empty(B, C, dtype=torch.float32, device="cuda")
    am = torch.empty(B, C, dtype=torch.int32, device="cuda")
    z_out = torch.empty(B, C, c.d_model, dtype=zt, device="cuda")
    _check(lib().dg_selfcond_forward(model.handle, kv.handle, cp, steps_left, T,
                                     zp, _ptr(H), _ptr(am), _ptr(z_out), _stream(stream)))
    return H, am, z_out


def dg_debug_forward(model: Model, kv: KV, canvas, steps_left: int, T: int, logits=False,
                     hidden=False, stream=None):
    c = model.cfg
    B, C = kv.B, c.canvas
    cp = _arg(canvas, "canvas", torch.int32, (B, C))
    n = B * C
    ent = torch.empty(B, C, dtype=torch.float32, device="cuda")
    am = torch.empty(B, C, dtype=torch.int32, device="cuda")
    lg = torch.empty(n, c.vocab, dtype=torch.float32, device="cuda") if logits else None
    hd = torch.empty(n, c.d_model, dtype=torch.float32, device="cuda") if hidden else None
    _check(lib().dg_debug_forward(model.handle, kv.handle, cp, steps_left, T,
                                  _ptr(ent), _ptr(am), _ptr(lg), _ptr(hd), _stream(stream)))
    return ent, am, lg, hd


KINDS = ("experts", "lmhead", "attention", "dense", "shared", "routing", "glue")


def dg_profile_start(model: Model, max_forwards: int = 0):
    """Event records around every launch group from now on; a profiled block runs at
    most max_forwards forwards (0: T), unrolled."""
    _check(lib().dg_profile_start(model.handle, max_forwards))


def dg_profile_stop(model: Model) -> dict:
    """{kind: (device ms summed, launch groups)} since dg_profile_start."""
    ms = (ctypes.c_float * len(KINDS))()
    groups = (ctypes.c_int64 * len(KINDS))()
    _check(lib().dg_profile_stop(model.handle, ms, groups))
    return {k: (float(ms[i]), int(groups[i])) for i, k in enumerate(KINDS)}


def dg_launch_count(model: Model) -> int:
    out = ctypes.c_int64()
    _check(lib().dg_launch_count(model.handle, ctypes.byref(out)))
    return out.value


def dg_op_gemm(model: Model, A, W, stream=None):
    """out[M, N] = A[M, K] W[N, K]^T (fp32) on the path's GEMM kernel."""
    M, K = A.shape
    N = W.shape[0]
    out = torch.empty(M, N, dtype=torch.float32, device="cuda")
    _check(lib().dg_op_gemm(model.handle, _ptr(A), _ptr(W), _ptr(out), M, N, K, _stream(stream)))
    return out


def dg_op_moe(model: Model, layer: int, x, stream=None):
    """x + MoE_layer(RMSNorm(x)) for fp32 rows x [n, d]."""
    out = torch.empty_like(x)
    _check(lib().dg_op_moe(model.handle, layer, _ptr(x), _ptr(out), x.shape[0], _stream(stream)))
    return out


def dg_expert_units(model: Model) -> int:
    out = ctypes.c_int64()
    _check(lib().dg_expert_units(model.handle, ctypes.byref(out)))
    return out.value


def _check_noalloc_args(hidden, lm_head):
    """The C entry point reads hidden as fp32 [M, d] and lm_head as bf16 [V, d] on the
    current device; anything else would be read out of bounds or misinterpreted, so it
    is rejected here, before any launch."""
    if hidden.dim() != 2 or hidden.dtype != torch.float32:
        raise ValueError(f"hidden must be a 2-D float32 tensor, got {hidden.dtype} "
                         f"{tuple(hidden.shape)}")
    if lm_head.dim() != 2 or lm_head.dtype != torch.bfloat16:
        raise ValueError(f"lm_head must be a 2-D bfloat16 tensor, got {lm_head.dtype} "
                         f"{tuple(lm_head.shape)}")
    if lm_head.shape[1] != hidden.shape[1]:
        raise ValueError(f"lm_head has {lm_head.shape[1]} columns, hidden has "
                         f"{hidden.shape[1]}")
    for name, t in (("hidden", hidden), ("lm_head", lm_head)):
        if not t.is_cuda or t.device.index != torch.cuda.current_device():
            raise ValueError(f"{name} must be a CUDA tensor on the current device")


def dg_lmhead_entropy_noalloc(hidden, lm_head, rms_eps: float, logit_scale: float, stream=None):
    """Entropy [M] and argmax [M] of logit_scale * RMSNorm(hidden) lm_head^T, computed
    without any device allocation by the library (static scratch)."""
    _check_noalloc_args(hidden, lm_head)
    M, d = hidden.shape
    V = lm_head.shape[0]
    ent = torch.empty(M, dtype=torch.float32, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    _check(lib().dg_lmhead_entropy_noalloc(_ptr(hidden), _ptr(lm_head), M, V, d, rms_eps,
                                           logit_scale, _ptr(ent), _ptr(am), _stream(stream)))
    return ent, am


def dg_block_loop_launches(model: Model) -> int:
    out = ctypes.c_int64()
    _check(lib().dg_block_loop_launches(model.handle, ctypes.byref(out)))
    return out.value


def dg_debug_stall_experts(model: Model, limit_ns: int):
    """Test hook: the next routed-expert launch runs its waits out after limit_ns."""
    _check(lib().dg_debug_stall_experts(model.handle, limit_ns))
