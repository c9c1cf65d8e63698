"""The golden files (written from the oracle alone by tests/golden/make_golden.py) on
CPU: the fields the GPU parity tests read are present and consistent, and the
distances between the oracle's bf16-storage run and its fp64 run behave as the
tolerance reading for the deep workloads assumes — small after one layer, amplified
through thirty."""
import glob
import os

import numpy as np
import pytest

from gpu_helpers import max_abs_rel, storage_tol

HERE = os.path.join(os.path.dirname(__file__), "golden")
# first-forward files (the depth sweep and the whole block have their own layouts)
FILES = sorted(f for f in glob.glob(os.path.join(HERE, "*.npz"))
               if not f.endswith(("-depths.npz", "-block.npz", "-append.npz", "-anneal.npz",
                                   "-selfcond.npz")))
STATED = 2e-2


def _load(name):
    path = os.path.join(HERE, name)
    if not os.path.exists(path):
        pytest.skip(f"{name} missing")
    return np.load(path)


@pytest.mark.parametrize("path", FILES, ids=[os.path.basename(f) for f in FILES])
def test_fields_and_shapes(path):
    g = np.load(path)
    for k in ("H", "argmax", "logits", "logit_rows", "logit_cols", "margin", "kv_last",
              "H_s16", "logits_s16", "kv_last_s16"):
        assert k in g.files, k
    C = g["H"].shape[0]
    assert g["argmax"].shape == (C,) and g["margin"].shape == (C,)
    assert g["logits"].shape == (len(g["logit_rows"]), len(g["logit_cols"]))
    assert g["logits_s16"].shape == g["logits"].shape
    assert g["kv_last_s16"].shape == g["kv_last"].shape and g["H_s16"].shape == g["H"].shape
    assert np.all(g["H"] >= 0) and np.all(np.isfinite(g["logits"]))
    assert np.all(g["margin"] >= 0)
    # the sampled logit rows and columns index real canvas rows and vocabulary entries
    assert g["logit_rows"].min() >= 0 and g["logit_rows"].max() < C
    assert g["logit_cols"].min() >= 0


def test_one_layer_storage_distance_within_stated_tolerance():
    for name in ("layer1-bf16.npz", "layer1-fp8exp-p4096.npz"):
        g = _load(name)
        assert max_abs_rel(g["logits_s16"], g["logits"]) < STATED / 2
        assert max_abs_rel(g["H_s16"], g["H"]) < STATED
        for j in range(2):  # layer 0's keys and values
            assert max_abs_rel(g["kv_last_s16"][0, j], g["kv_last"][0, j]) < STATED / 2


def test_thirty_layers_amplify_storage_noise():
    one, deep = _load("layer1-bf16.npz"), _load("full30-bf16.npz")
    # same first layer: layer 0's K/V see the same storage noise in both workloads
    for j in range(2):
        a = max_abs_rel(one["kv_last_s16"][0, j], one["kv_last"][0, j])
        b = max_abs_rel(deep["kv_last_s16"][0, j], deep["kv_last"][0, j])
        assert 0.5 < b / a < 2.0
    # the last layer's K/V, the logits and the entropies move several times further
    assert max_abs_rel(deep["kv_last_s16"][1, 0], deep["kv_last"][1, 0]) > \
        3 * max_abs_rel(deep["kv_last_s16"][0, 0], deep["kv_last"][0, 0])
    assert max_abs_rel(deep["logits_s16"], deep["logits"]) > \
        3 * max_abs_rel(one["logits_s16"], one["logits"])
    assert max_abs_rel(deep["H_s16"], deep["H"]) > 3 * max_abs_rel(one["H_s16"], one["H"])
    # so the deep tolerances come from the storage run, the shallow ones stay stated
    assert storage_tol(deep, "H", STATED) > STATED
    assert storage_tol(deep, "logits", STATED) > STATED
    assert storage_tol(deep, "kv_last", STATED, (0, 0)) == STATED


def test_depth_sweep_file_matches_the_single_depth_files():
    """Depth 1 of the sweep is the one-layer workload and depth 30 the 30-layer one
    (weights seeded per layer name; the sweep runs the same oracle layer by layer), so
    their fp64 and bf16-storage outputs are identical."""
    d = _load("full30-bf16-depths.npz")
    assert list(d["depths"]) == [1, 2, 4, 8, 16, 30]
    for k, name in ((1, "layer1-bf16.npz"), (30, "full30-bf16.npz")):
        g = _load(name)
        for key in ("H", "argmax", "logits", "H_s16", "logits_s16"):
            sweep_key = key.replace("_s16", "") + ("_s16" if key.endswith("_s16") else "")
            np.testing.assert_array_equal(d[f"{sweep_key}_d{k}"], g[key], err_msg=f"{k} {key}")
        # layer k-1's keys/values: the single-depth files keep layers 0 and L-1
        np.testing.assert_array_equal(d[f"kv_last_d{k}"], g["kv_last"][-1])
    # storage noise grows with depth on the logits (1 layer -> 30 layers)
    assert max_abs_rel(d["logits_s16_d30"], d["logits_d30"]) > \
        3 * max_abs_rel(d["logits_s16_d1"], d["logits_d1"])


def test_whole_block_file_is_a_valid_trajectory():
    """The oracle's block: steps left T, T-1, ...; each input canvas is the previous one
    with exactly the committed positions set to their argmax; the committed counts obey
    the rule's minimum ceil(masked / steps_left); the block ends with no [MASK]."""
    import math
    from synth import workloads
    w = workloads.FULL30_BF16
    b = _load("full30-bf16-block.npz")
    n = int(b["n_forwards"])
    assert 1 <= n <= w.T and list(b["s"]) == [w.T - i for i in range(n)]
    assert np.all(b["canvas_in"][0] == w.mask_id)
    assert int(b["n_committed"].sum()) == w.canvas
    for i in range(n):
        m = int((b["canvas_in"][i] == w.mask_id).sum())
        assert int(b["n_committed"][i]) >= math.ceil(m / int(b["s"][i]))
        assert np.all((b["H"][i] >= 0) & (b["H"][i] <= math.log(w.vocab) + 1e-3))
        nxt = b["canvas_in"][i + 1] if i + 1 < n else b["final_canvas"]
        changed = nxt != b["canvas_in"][i]
        assert int(changed.sum()) == int(b["n_committed"][i])
        assert np.all(b["canvas_in"][i][changed] == w.mask_id)
        assert np.array_equal(nxt[changed], b["argmax"][i][changed])
        assert np.array_equal(b["mask_after"][i] == 1, nxt == w.mask_id)
    assert not np.any(b["final_canvas"] == w.mask_id)


def test_anneal_file_is_consistent():
    """The annealed forward file: its canvas is the seed's x_1, the draws are tokens, the
    gaps are non-negative, the argmax and draw agree where the noise cannot move them."""
    from oracle import anneal as an
    g = _load("layer1-bf16-anneal.npz")
    C, V = 256, 262144
    assert np.array_equal(g["canvas"], an.initial_canvas(int(g["seed"]), C, V))
    assert ((g["sampled"] >= 0) & (g["sampled"] < V)).all() and (g["gap"] >= 0).all()
    assert abs(float(g["tau"]) - an.temperature(int(g["k"]), an.Params(N=int(g["N"])))) < 1e-15
    assert np.allclose(g["H"], g["H64"], rtol=1e-6)
    assert 0.9 < (g["gap"] > 0.05).mean() <= 1.0
