"""Writes the oracle's expected outputs for the full-size workloads to tests/golden/.

Calls only `oracle/` and `synth/` (never the CUDA path).  Usage:
    python tests/golden/make_golden.py layer1-bf16 [full30-bf16+s16 full30-b8-p8192:7 ...]
Each file <workload>[-c<canvas>].npz holds, for one canvas of the workload's first forward
(all [MASK], steps_left = T):
  H [C] fp32 entropies, H64 [C], argmax [C], margin [C] (top-1 minus top-2 logit),
  lse [C], sigma [C] (std of the logits under the row's softmax); logit_rows [R] row
  ids and logit_cols [Vs] vocab ids with
  logits [R, Vs]; kv_last [L?, 2, Hkv, 8, h] post-RoPE keys / values of the last 8
  prompt positions of layers 0 and L-1; router margins per layer (min over rows of
  the gap between the k-th and (k+1)-th router logits); the sampler step's canvas,
  mask and count on these entropies.
With the suffix "+s16" the file also holds the same outputs of the oracle's bf16
storage variant (H_s16, argmax_s16, logits_s16, kv_last_s16): the sensitivity of the
workload to bf16 activation storage, from which the deep workloads' tolerances follow.
The suffix "+s16only" adds those fields to an existing file (the fp64 run is not
repeated).  Files also hold router_margin_rows [C]: per row, the smallest gap over the
layers between the top_k-th and (top_k+1)-th router logit ("+rmonly" adds it to an
existing file).

Two further modes on a deep workload:
  <name>@depths  -> <name>-depths.npz: the first forward of the models made of the
     first k layers of the workload (k in DEPTHS; the weights are seeded per layer
     name, so these are the same layers the full model holds), fp64 and bf16-storage
     runs, at every k: H, argmax, margin, sampled logits and layer k-1's last keys and
     values.  One pass through the layers serves every depth (the prompt pass and the
     canvas pass interleave layer by layer, so the canvas state after layer k-1 is the
     k-layer model's final residual).
  <name>@append  -> <name>-append.npz: canvas 0's prompt and a block of seeded tokens
     as one causal pass, layer 0's window keys / values at a few positions (the
     reference for appending a finished block to the cache).
  <name>@anneal  -> <name>-anneal.npz: one forward of the annealed sampler (the Report's
     default) for canvas 0 at step ANNEAL_K of N = 48 with seed ANNEAL_SEED, on the
     uniform initial canvas x_1: tempered entropies H/H64, argmax, the Gumbel-max draw
     `sampled` and its gap to the runner-up, the router margins of the rows, and the
     bf16-storage run's H_s16 and sampled_s16.
  <name>@selfcond -> <name>-selfcond.npz (a self-conditioned workload): canvas 0's first
     forward (all [MASK], steps_left = T), its entropies and the self-conditioning signal
     z = FFW(p0 E) it hands to the next forward, with y = p0 E; and the bf16-storage
     run's H64_s16 and z_s16.
  <name>@block   -> <name>-block.npz: the oracle's whole block (all [MASK], up to T
     forwards, the entropy-bound sampler after each): per step the input canvas, the
     steps left, H, argmax, margin and the number committed; the number of forwards.
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import model as om  # noqa: E402
from oracle import sampler as osamp  # noqa: E402
from synth import model_inputs, workloads  # noqa: E402

LOGIT_ROWS = [0, 1, 77, 128, 255]


def _kv_last(w, st):
    return np.stack([np.stack([st["kv"][l][0][-8:].transpose(1, 0, 2),
                               st["kv"][l][1][-8:].transpose(1, 0, 2)])
                     for l in sorted({0, w.n_layers - 1})])


def add_storage_variant(name: str, canvas_index: int = 0):
    """Adds the bf16-storage run's fields to an existing golden file."""
    w = workloads.get(name)
    t0 = time.time()
    suffix = f"-c{canvas_index}" if canvas_index else ""
    path = os.path.join(HERE, f"{name}{suffix}.npz")
    old = dict(np.load(path))
    prompt = model_inputs.prompt(w.with_(batch=1), first=canvas_index)[0].numpy()
    canvas = np.full(w.canvas, w.mask_id)
    ws16 = om.Weights(w, keep_layers=False, storage="bf16")
    s16 = om.prefill_then_forward(ws16, prompt, canvas, w.T, w.T, want_logits=True)
    rows, cols = old["logit_rows"], old["logit_cols"]
    old.update(H_s16=s16["H"], argmax_s16=s16["argmax"], kv_last_s16=_kv_last(w, s16),
               logits_s16=s16["logits"][rows][:, cols].astype(np.float64))
    np.savez_compressed(path, **old)
    print(f"{name}{suffix}: added the bf16-storage run in {time.time() - t0:.0f} s")


def _router_margin_rows(w, routes):
    """Per canvas row, the smallest gap over the layers between the top_k-th and the
    (top_k+1)-th router logit: a row whose gap is small may be routed differently by
    any path that perturbs the router's input (bf16 storage included)."""
    gaps = []
    for _, _, rl in routes:
        srt = np.sort(rl, axis=1)[:, ::-1]
        gaps.append(srt[:, w.top_k - 1] - srt[:, w.top_k])
    return np.min(np.stack(gaps), axis=0)


def add_router_margins(name: str, canvas_index: int = 0):
    """Adds router_margin_rows to an existing golden file (reruns the fp64 forward)."""
    w = workloads.get(name)
    t0 = time.time()
    suffix = f"-c{canvas_index}" if canvas_index else ""
    path = os.path.join(HERE, f"{name}{suffix}.npz")
    old = dict(np.load(path))
    prompt = model_inputs.prompt(w.with_(batch=1), first=canvas_index)[0].numpy()
    canvas = np.full(w.canvas, w.mask_id)
    st = om.prefill_then_forward(om.Weights(w, keep_layers=False), prompt, canvas, w.T, w.T)
    assert np.array_equal(st["H"], old["H"]), "the oracle no longer reproduces this file"
    old["router_margin_rows"] = _router_margin_rows(w, st["routes"])
    np.savez_compressed(path, **old)
    print(f"{name}{suffix}: added per-row router margins in {time.time() - t0:.0f} s; "
          f"rows with margin < 1e-2: {(old['router_margin_rows'] < 1e-2).sum()}", flush=True)


def make(name: str, canvas_index: int = 0, storage_variant: bool = False):
    """Oracle outputs of the first forward of canvas `canvas_index` of the workload."""
    w = workloads.get(name)
    t0 = time.time()
    ws = om.Weights(w, keep_layers=False)
    prompt = model_inputs.prompt(w.with_(batch=1), first=canvas_index)[0].numpy()
    canvas = np.full(w.canvas, w.mask_id)
    st = om.prefill_then_forward(ws, prompt, canvas, w.T, w.T, want_logits=True)
    cols = np.arange(0, w.vocab, max(1, w.vocab // 4096))
    rows = [r for r in LOGIT_ROWS if r < w.canvas]
    kv_last = _kv_last(w, st)
    extra = {}
    if storage_variant:
        ws16 = om.Weights(w, keep_layers=False, storage="bf16")
        s16 = om.prefill_then_forward(ws16, prompt, canvas, w.T, w.T, want_logits=True)
        extra = dict(H_s16=s16["H"], argmax_s16=s16["argmax"], kv_last_s16=_kv_last(w, s16),
                     logits_s16=s16["logits"][rows][:, cols].astype(np.float64))
    rmarg = []
    for idx, g, rl in st["routes"]:
        srt = np.sort(rl, axis=1)[:, ::-1]
        rmarg.append((srt[:, w.top_k - 1] - srt[:, w.top_k]).min())
    c2, m2, n2, kg = osamp.eb_step(st["H"], st["argmax"], canvas, np.ones(w.canvas, np.uint8),
                                   w.T, w.gamma)
    suffix = f"-c{canvas_index}" if canvas_index else ""
    out = os.path.join(HERE, f"{name}{suffix}.npz")
    np.savez_compressed(out, H=st["H"], H64=st["H64"], argmax=st["argmax"], margin=st["margin"],
                        lse=st["lse"], sigma=st["sigma"], logit_rows=np.array(rows),
                        logit_cols=cols,
                        logits=st["logits"][rows][:, cols].astype(np.float64), kv_last=kv_last,
                        router_margin=np.array(rmarg),
                        router_margin_rows=_router_margin_rows(w, st["routes"]),
                        step_canvas=c2, step_mask=m2,
                        step_n=np.array(n2), step=np.array(w.T), **extra)
    print(f"{name}: wrote {out} in {time.time() - t0:.0f} s; H range "
          f"[{st['H'].min():.4f}, {st['H'].max():.4f}], min margin {st['margin'].min():.4g}, "
          f"min router gap {min(rmarg):.3g}, sampler n {n2}")


APPEND_POS = (0, 8, 760, 776, 1016, 1024)   # window offsets: 8 positions from each


def append_case(name: str):
    """<name>-append.npz: canvas 0's prompt followed by a block of seeded tokens
    (synth.model_inputs.block_tokens), as one causal pass: layer 0's keys and values
    of 8 consecutive window positions from each offset in APPEND_POS (the window is
    the last min(P + C, window) positions of the whole sequence)."""
    w = workloads.get(name)
    t0 = time.time()
    prompt = model_inputs.prompt(w.with_(batch=1))[0].numpy()
    block = model_inputs.block_tokens(w.with_(batch=1))[0].numpy()
    seq = np.concatenate([prompt, block])
    ws = om.Weights(w.with_(n_layers=1), keep_layers=False)
    K, V = om.prefill(ws, seq)[0]                       # [W, Hkv, h]
    Wn = K.shape[0]
    sel = [o + i for o in APPEND_POS for i in range(8) if o + i < Wn]
    out = dict(window=np.array(Wn), positions=np.array(sel),
               k=K[sel].transpose(1, 0, 2), v=V[sel].transpose(1, 0, 2))
    path = os.path.join(HERE, f"{name}-append.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s (window {Wn})")


ANNEAL_SEED, ANNEAL_K = 1234567, 5


def anneal_case(name: str):
    """<name>-anneal.npz: step ANNEAL_K's forward of the annealed sampler on canvas 0."""
    from oracle import anneal
    w = workloads.get(name)
    t0 = time.time()
    p = anneal.Params()
    prompt = model_inputs.prompt(w.with_(batch=1))[0].numpy()
    canvas = anneal.initial_canvas(ANNEAL_SEED, w.canvas, w.vocab)
    ws = om.Weights(w, keep_layers=False)
    st = om.prefill_then_forward(ws, prompt, canvas, p.N - ANNEAL_K, p.N, want_logits=True)
    tau = anneal.temperature(ANNEAL_K, p)
    ts = anneal.tempered_stats(st["logits"], tau)
    sampled, gap = anneal.sample_tokens(st["logits"], tau, ANNEAL_SEED, ANNEAL_K)
    ws16 = om.Weights(w, keep_layers=False, storage="bf16")
    s16 = om.prefill_then_forward(ws16, prompt, canvas, p.N - ANNEAL_K, p.N, want_logits=True)
    ts16 = anneal.tempered_stats(s16["logits"], tau)
    out = dict(seed=np.array(ANNEAL_SEED, dtype=np.uint64), k=np.array(ANNEAL_K),
               N=np.array(p.N), tau=np.array(tau), canvas=canvas, H=ts["H"], H64=ts["H64"],
               argmax=ts["argmax"], sampled=sampled, gap=gap,
               router_margin_rows=_router_margin_rows(w, st["routes"]), H_s16=ts16["H64"],
               sampled_s16=anneal.sample_tokens(s16["logits"], tau, ANNEAL_SEED, ANNEAL_K)[0])
    path = os.path.join(HERE, f"{name}-anneal.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s; tau {tau:.4f}, H range "
          f"[{ts['H'].min():.3f}, {ts['H'].max():.3f}], gaps > 0.05: {(gap > 0.05).mean():.3f}")


def selfcond_case(name: str):
    """<name>-selfcond.npz: canvas 0's first forward and the z it produces."""
    w = workloads.get(name)
    t0 = time.time()
    prompt = model_inputs.prompt(w.with_(batch=1))[0].numpy()
    canvas = np.full(w.canvas, w.mask_id)
    ws = om.Weights(w, keep_layers=False)
    st = om.prefill_then_forward(ws, prompt, canvas, w.T, w.T, want_logits=True)
    y = om.selfcond_mix(ws, st["logits"])
    z = om.selfcond(ws, st["logits"])
    ws16 = om.Weights(w, keep_layers=False, storage="bf16")
    s16 = om.prefill_then_forward(ws16, prompt, canvas, w.T, w.T, want_logits=True)
    out = dict(H=st["H"], H64=st["H64"], y=y, z=z, H64_s16=s16["H64"],
               z_s16=om.selfcond(ws16, s16["logits"]))
    path = os.path.join(HERE, f"{name}-selfcond.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s; |y| rms {np.sqrt((y * y).mean()):.3g},"
          f" |z| rms {np.sqrt((z * z).mean()):.3g}")


DEPTHS = (1, 2, 4, 8, 16, 30)


def depth_sweep(name: str, depths=DEPTHS):
    """Oracle outputs of the first forward of the k-layer prefixes of the workload."""
    w = workloads.get(name)
    t0 = time.time()
    prompt = model_inputs.prompt(w.with_(batch=1))[0].numpy()
    canvas = np.full(w.canvas, w.mask_id)
    P = prompt.shape[0]
    cols = np.arange(0, w.vocab, max(1, w.vocab // 4096))
    rows = [r for r in LOGIT_ROWS if r < w.canvas]
    out = dict(depths=np.array([k for k in depths if k <= w.n_layers]),
               logit_rows=np.array(rows), logit_cols=cols)
    for storage, tag in (("fp64", ""), ("bf16", "_s16")):
        ws = om.Weights(w, keep_layers=False, storage=storage)
        x = om.canvas_input(ws, canvas, w.T, w.T)
        for l, kw, vw, lw in om.prefill_layer_by_layer(ws, prompt):
            x, _, _, _ = om.canvas_layer(x, lw, (kw, vw), P, w)
            k = l + 1
            if k not in depths:
                continue
            st = om.lm_head_stats(ws, x, want_logits=True)
            kvl = np.stack([kw[-8:].transpose(1, 0, 2), vw[-8:].transpose(1, 0, 2)])
            out.update({f"H{tag}_d{k}": st["H"], f"H64{tag}_d{k}": st["H64"],
                        f"argmax{tag}_d{k}": st["argmax"], f"margin{tag}_d{k}": st["margin"],
                        f"sigma{tag}_d{k}": st["sigma"],
                        f"logits{tag}_d{k}": st["logits"][rows][:, cols].astype(np.float64),
                        f"kv_last{tag}_d{k}": kvl})
            print(f"{name} depth {k} ({storage}): H [{st['H'].min():.4f}, "
                  f"{st['H'].max():.4f}] at {time.time() - t0:.0f} s", flush=True)
            if k == max(depths):
                break
    path = os.path.join(HERE, f"{name}-depths.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s")


def whole_block(name: str):
    """The oracle's whole block on canvas 0 of the workload (steps as the sampler takes them)."""
    w = workloads.get(name)
    t0 = time.time()
    ws = om.Weights(w, keep_layers=True)
    prompt = model_inputs.prompt(w.with_(batch=1))[0].numpy()
    P = prompt.shape[0]
    kv = om.prefill(ws, prompt)
    print(f"{name}: prefill done at {time.time() - t0:.0f} s", flush=True)
    rec = []

    def forward(canvas, s):
        st = om.denoise_forward(ws, kv, canvas, s, w.T, P)
        rec.append(dict(canvas=np.array(canvas, dtype=np.int64), s=s, H=st["H"],
                        argmax=st["argmax"], margin=st["margin"], sigma=st["sigma"]))
        print(f"{name}: forward s={s} at {time.time() - t0:.0f} s; H [{st['H'].min():.4f}, "
              f"{st['H'].max():.4f}]", flush=True)
        return st["H"], st["argmax"]

    canvas, traj = osamp.generate_block(forward, w.canvas, w.mask_id, w.T, w.gamma)
    n = len(traj)
    out = dict(n_forwards=np.array(n), final_canvas=canvas,
               s=np.array([r["s"] for r in rec]),
               canvas_in=np.stack([r["canvas"] for r in rec]),
               H=np.stack([r["H"] for r in rec]), argmax=np.stack([r["argmax"] for r in rec]),
               margin=np.stack([r["margin"] for r in rec]),
               sigma=np.stack([r["sigma"] for r in rec]),
               n_committed=np.array([t[5] for t in traj]),
               mask_after=np.stack([t[4] for t in traj]))
    path = os.path.join(HERE, f"{name}-block.npz")
    np.savez_compressed(path, **out)
    print(f"{name}: wrote {path} in {time.time() - t0:.0f} s; {n} forwards, commits "
          f"{[int(t[5]) for t in traj]}")


if __name__ == "__main__":
    # arguments: workload names, optionally "name:canvas" to pick a canvas of the batch
    # and the suffix "+s16" for the bf16 storage variant as well ("+s16only": that alone)
    for arg in sys.argv[1:] or ["layer1-bf16"]:
        if arg.endswith("@append"):
            append_case(arg.removesuffix("@append"))
            continue
        if arg.endswith("@depths"):
            depth_sweep(arg.removesuffix("@depths"))
            continue
        if arg.endswith("@block"):
            whole_block(arg.removesuffix("@block"))
            continue
        if arg.endswith("@anneal"):
            anneal_case(arg.removesuffix("@anneal"))
            continue
        if arg.endswith("@selfcond"):
            selfcond_case(arg.removesuffix("@selfcond"))
            continue
        if arg.endswith("+rmonly"):
            name, _, c = arg.removesuffix("+rmonly").partition(":")
            add_router_margins(name, int(c) if c else 0)
            continue
        if arg.endswith("+s16only"):
            name, _, c = arg.removesuffix("+s16only").partition(":")
            add_storage_variant(name, int(c) if c else 0)
            continue
        s16 = arg.endswith("+s16")
        name, _, c = arg.removesuffix("+s16").partition(":")
        make(name, int(c) if c else 0, storage_variant=s16)
