"""Pins of the oracle's self-conditioning signal (oracle.model.selfcond_mix, selfcond,
CanvasForwards): closed forms of p0 E for peaked, uniform and shifted logits, a
brute force on a tiny vocabulary, the FFW's closed form with identity weights, the
[MASK] row left out, and the way the block loop carries z from forward to forward."""
import math

import numpy as np

from oracle import model as om
from synth import model_inputs, workloads


class _Given(om.Weights):
    """Weights whose tensors are given by hand."""

    def __init__(self, w, tensors):
        super().__init__(w, keep_layers=True)
        self.t = tensors

    def get(self, name, shape):
        assert self.t[name].shape == tuple(shape), name
        return self.t[name]


def _tiny(V=5, d=3, I=3):
    w = workloads.TINY_F32.with_(name="sc-pin", vocab=V, d_model=d, sc_inter=I)
    rng = np.random.default_rng(7)
    E = rng.normal(size=(V + 1, d))
    return w, E


def test_peaked_logits_give_the_embedding_row():
    w, E = _tiny()
    ws = _Given(w, {"tok_emb": E})
    l = np.zeros((3, w.vocab))
    for r, t in enumerate((4, 0, 2)):
        l[r, t] = 1e4
    y = om.selfcond_mix(ws, l)
    assert np.allclose(y, E[[4, 0, 2]], rtol=0, atol=1e-12)


def test_uniform_and_shifted_logits():
    w, E = _tiny()
    ws = _Given(w, {"tok_emb": E})
    y = om.selfcond_mix(ws, np.full((2, w.vocab), 3.5))
    assert np.allclose(y, E[:w.vocab].mean(axis=0)[None, :], atol=1e-14)
    rng = np.random.default_rng(1)
    l = rng.normal(size=(4, w.vocab)) * 3
    assert np.allclose(om.selfcond_mix(ws, l), om.selfcond_mix(ws, l + 123.0), atol=1e-13)


def test_brute_force_mixture_and_the_mask_row():
    w, E = _tiny()
    rng = np.random.default_rng(2)
    l = rng.normal(size=(2, w.vocab)) * 2
    E[w.vocab] = 1e9                    # the [MASK] row is not a class of p0
    ws = _Given(w, {"tok_emb": E})
    y = om.selfcond_mix(ws, l)
    for r in range(2):
        ex = [math.exp(v) for v in l[r]]
        Z = sum(ex)
        for j in range(w.d_model):
            ref = sum(ex[v] / Z * E[v, j] for v in range(w.vocab))
            assert abs(y[r, j] - ref) < 1e-12


def test_ffw_closed_form_with_identity_weights():
    w, E = _tiny()
    I3 = np.eye(3)
    ws = _Given(w, {"tok_emb": E, "sc.gate": I3, "sc.up": I3, "sc.down": I3})
    rng = np.random.default_rng(3)
    l = rng.normal(size=(2, w.vocab))
    y = om.selfcond_mix(ws, l)
    z = om.selfcond(ws, l)
    assert np.allclose(z, y * y / (1.0 + np.exp(-y)), atol=1e-15)


def test_canvas_input_adds_z_and_the_loop_carries_it():
    w = workloads.TINY_F32_SC
    ws = om.Weights(w, keep_layers=True)
    prompt = model_inputs.prompt(w, "cpu")[0].numpy()
    canvas = np.full(w.canvas, w.mask_id)
    z = np.random.default_rng(4).normal(size=(w.canvas, w.d_model))
    assert np.array_equal(om.canvas_input(ws, canvas, 3, 4, z),
                          om.canvas_input(ws, canvas, 3, 4) + z)
    kv = om.prefill(ws, prompt)
    fw = om.CanvasForwards(ws, kv, len(prompt))
    st0 = fw.logits(canvas, 4, 4)
    z1 = fw.z
    assert np.array_equal(z1, om.selfcond(ws, st0["logits"]))
    st1 = fw.logits(canvas, 3, 4)
    ref = om.denoise_forward(ws, kv, canvas, 3, 4, len(prompt), want_logits=True, z=z1)
    assert np.array_equal(st1["logits"], ref["logits"])
    assert fw.zs[0] is None and fw.zs[1] is z1
    # without the FFW weights' signal (z = 0) the forward is the plain one
    plain = om.denoise_forward(ws, kv, canvas, 3, 4, len(prompt), want_logits=True)
    zero = om.denoise_forward(ws, kv, canvas, 3, 4, len(prompt), want_logits=True,
                              z=np.zeros_like(z1))
    assert np.array_equal(plain["logits"], zero["logits"])
    # a model without self-conditioning never carries z
    w0 = workloads.TINY_F32
    f0 = om.CanvasForwards(om.Weights(w0, keep_layers=True), om.prefill(
        om.Weights(w0, keep_layers=True), prompt), len(prompt))
    f0.logits(canvas, 4, 4)
    f0.logits(canvas, 3, 4)
    assert f0.zs == [None, None] and f0.z is None
