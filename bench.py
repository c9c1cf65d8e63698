#!/usr/bin/env python
"""Throughput of block-parallel canvas denoising on B200.

One step = one 256-token block per canvas: `dg_generate_block` runs T denoise
forwards (all layers, LM head with online entropy, EB sampler) from an all
[MASK] canvas.  Metric: canvas tokens per second = canvases x 256 / block time.
Default workload: the 30-layer stand-in, batch 1, prompt 1024 (prefilled once),
T = 12, gamma = 1.0.  Weights (40 GB) exceed L2, so no flush is needed.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: one process per GPU (torchrun); every rank denoises its own canvases
(weak scaling, no collective on the data path); time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per routed expert streamed
# by the routed-expert kernel as it now stands (sixteen epilogue warps): one ncu capture
# of the 12 launches of a one-layer block (layer1-bf16, same kernel shapes as one layer
# of the 30-layer workload; profiles/tc_moe_kernel_layer1-bf16.md): 1,272.8 MB over 123
# streamed experts = 10,347,882 B each, 1.10x the 9,437,184 B of weights (the rest:
# gathered and hidden rows, which ncu's cold cache sends to DRAM).
DRAM_BYTES_PER_EXPERT = 10347882


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}",
                                       f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup(backend: str | None = None):
    """One process per GPU: RANK / LOCAL_RANK / WORLD_SIZE from the launcher, NCCL
    between the ranks (gloo when no GPU is visible, for the host-side tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_throughput(world: int, units_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job units per second: every rank processes units_per_rank per step (weak
    scaling), timed as the slowest rank's device time over the steps."""
    return world * units_per_rank * steps / (ms_max / 1e3)


def build_once(world: int, local: int):
    """The node's local rank 0 builds the library (if out of date); the others wait."""
    from masked_discrete_diffusion_b200 import build
    if local == 0:
        build.build()
    barrier(world)


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample of the workload
# ---------------------------------------------------------------------------
class OracleSample:
    """The oracle's canvas forward on layer 0 and on 1/vocab_frac of the LM head, one
    canvas, scaled to a block (T forwards of all layers); weights generated once."""

    def __init__(self, w, vocab_frac: int = 16):
        import numpy as np

        from oracle import model as om
        from synth import model_inputs
        self.om, self.w, self.vf = om, w, vocab_frac
        self.ws = om.Weights(w, keep_layers=True)
        self.lw = self.ws.layer(0)
        prompt = model_inputs.prompt(w.with_(batch=1))[0].numpy()
        P = len(prompt)
        empty = np.zeros((0, w.n_kv_heads, w.head_dim))
        _, k, v, _ = om.decoder_layer(om.embed(self.ws, prompt), np.arange(P), self.lw,
                                      (empty, empty), om.causal_window_mask(P, w.window), w)
        W = min(P, w.window)
        self.kv = (k[P - W:], v[P - W:])
        self.x = om.canvas_input(self.ws, np.full(w.canvas, w.mask_id), w.T, w.T)
        self.Wl = self.ws.rows("lm_head", (w.vocab, w.d_model), 0, w.vocab // vocab_frac)

    def run(self):
        from threadpoolctl import threadpool_info
        om, w = self.om, self.w
        t0 = time.perf_counter()
        x1, _, _, _ = om.canvas_layer(self.x, self.lw, self.kv, w.prompt_len, w)
        t_layer = time.perf_counter() - t0
        t0 = time.perf_counter()
        om.entropy_stats(w.logit_scale * (om.rmsnorm(x1, w.rms_eps) @ self.Wl.T))
        t_lm = time.perf_counter() - t0
        fwd = w.n_layers * t_layer + self.vf * t_lm
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        desc = (f"oracle canvas forward of layer 0 ({t_layer:.2f} s, x{w.n_layers} layers) and "
                f"LM head over 1/{self.vf} of the vocabulary ({t_lm:.2f} s, x{self.vf}), "
                f"one canvas, scaled to a block of {w.T} forwards x {w.batch} canvases; "
                f"weight generation excluded")
        return fwd * w.T * w.batch, desc, threads


def run_reference(args, w, world, rank):
    if rank != 0:
        return
    times = []
    desc, threads = "", 1
    smp = OracleSample(w)
    for _ in range(args.warmup):
        smp.run()
    for _ in range(args.steps):
        t, desc, threads = smp.run()
        times.append(t)
    block = statistics.mean(times)
    val = w.batch * w.canvas / block
    line = {"impl": "reference", "metric": "canvas tokens/sec at 1 B200 (256-tok block)",
            "value": val, "unit": "canvas tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": block * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "canvas": w.canvas,
                       "prompt": w.prompt_len, "layers": w.n_layers, "T": w.T},
            "cpu_baseline": {"value": val, "unit": "canvas tokens/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": val, "unit": "canvas tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our path
# ---------------------------------------------------------------------------
def run_e2e(args, w, world, model, prompt, canvas, stream):
    """Canvas tokens/s through the public API with host buffers, as a serving loop runs
    it: every step uploads the prompt from pinned host memory, refills the slot's KV
    handle (dg_prefill_into), denoises the block (dg_generate_block) and reads the
    canvas back.  The handle is made once, before the timed steps."""
    import torch

    from masked_discrete_diffusion_b200 import binding
    B, C, T = w.batch, w.canvas, w.T
    h_prompt = prompt.cpu().pin_memory()
    h_canvas = torch.empty(B, C, dtype=torch.int32).pin_memory()
    d_prompt = torch.empty_like(prompt)
    kv2 = binding.dg_prefill(model, prompt)
    for _ in range(max(args.warmup, 1)):
        binding.dg_prefill_into(model, prompt, kv2)
        binding.dg_generate_block(model, kv2, T, w.gamma, canvas)
    torch.cuda.synchronize()
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        d_prompt.copy_(h_prompt, non_blocking=True)
        binding.dg_prefill_into(model, d_prompt, kv2)
        binding.dg_generate_block(model, kv2, T, w.gamma, canvas)
        h_canvas.copy_(canvas, non_blocking=True)
        f1.record(stream)
        f1.synchronize()
    kv2.close()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    e2e_val = job_throughput(world, B * C, args.steps, e2e_ms)

    return e2e_val


def run_blocks(args, w, world, model, prompt):
    """Block-autoregressive generation of args.blocks blocks per canvas (each finished
    block joins the context through the causal pass before the next is denoised),
    device-timed from the first block to the last, prompt pass excluded; tokens per
    forward counts the K - 1 append passes of K blocks."""
    import torch

    from masked_discrete_diffusion_b200 import binding, metrics
    K, B, C = args.blocks, w.batch, w.canvas
    kv = binding.dg_prefill(model, prompt)
    for _ in range(max(args.warmup, 1)):
        binding.dg_prefill_into(model, prompt, kv)
        binding.dg_generate_blocks(model, kv, K, w.T, w.gamma)
    torch.cuda.synchronize()
    barrier(world)
    ms = 0.0
    nf = None
    for _ in range(args.steps):
        binding.dg_prefill_into(model, prompt, kv)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        _, nf = binding.dg_generate_blocks(model, kv, K, w.T, w.gamma)
        e1.record()
        e1.synchronize()
        ms += e0.elapsed_time(e1)
    binding.dg_sync_status(model)
    kv.close()
    ms_max = max_over_ranks(ms, world)
    per_block = nf.max(dim=1).values.cpu().tolist()
    return {"n_blocks": K,
            "canvas_tokens_per_s": job_throughput(world, B * K * C, args.steps, ms_max),
            "ms_per_step": ms_max / args.steps,
            "forwards_per_block": per_block,
            "tokens_per_forward_eq10": metrics.tokens_per_forward([C] * K, per_block),
            "includes": "dg_generate_blocks: K blocks, K - 1 dg_append_block causal passes"}


def run_annealed(args, w, world, model, prompt, eb_lmhead_ms):
    """The Report's default sampler (annealed entropy-bounded refinement over a uniform
    canvas, N = 48, b = 0.1, tau 0.8 -> 0.4, e_stop = 0.005): device-timed blocks of
    dg_generate_block_annealed (graph replays), then a profiled pass of its first
    forwards for the LM head's cost with the tempered statistics and the Gumbel-max race
    against the Entropy-Bound block's LM head."""
    import torch

    from masked_discrete_diffusion_b200 import binding
    B, C = w.batch, w.canvas
    p = binding.anneal_params()
    seeds = torch.tensor([0x5EED + 977 * b for b in range(B)], dtype=torch.int64,
                         device="cuda")
    out = torch.empty(B, C, dtype=torch.int32, device="cuda")
    nf = torch.empty(B, dtype=torch.int32, device="cuda")
    kv = binding.dg_prefill(model, prompt)
    binding.dg_generate_block_annealed(model, kv, seeds, p, out, nf)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("annealed")
    e0.record()
    for _ in range(args.annealed):
        binding.dg_generate_block_annealed(model, kv, seeds, p, out, nf)
    e1.record()
    e1.synchronize()
    torch.cuda.nvtx.range_pop()
    ms_max = max_over_ranks(e0.elapsed_time(e1), world)
    fwd = int(nf.max().item())
    binding.dg_profile_start(model, 3)
    binding.dg_generate_block_annealed(model, kv, seeds, p, out, nf)
    torch.cuda.synchronize()
    prof = binding.dg_profile_stop(model)
    units = binding.dg_expert_units(model)
    binding.dg_sync_status(model)
    kv.close()
    lm_ms, lm_n = prof["lmhead"]
    lm = lm_ms / max(lm_n, 1)
    n_prof = min(3, p.N)
    kinds = {k: round(v[0] / n_prof, 4) for k, v in prof.items()}
    return {"N": p.N, "b": round(p.b, 6), "tau_max": round(p.tau_max, 6),
            "tau_min": round(p.tau_min, 6), "e_stop": round(p.e_stop, 6),
            "steps": args.annealed,
            "canvas_tokens_per_s": job_throughput(world, B * C, args.annealed, ms_max),
            "ms_per_block": ms_max / args.annealed, "forwards_per_block": fwd,
            "ms_per_forward": ms_max / args.annealed / max(fwd, 1),
            "lmhead_ms_per_forward": lm,
            "lmhead_ms_per_forward_entropy_bound": eb_lmhead_ms,
            "kernel_groups_ms_per_forward": kinds,
            "experts_streamed_per_layer_forward": units / (n_prof * w.n_layers),
            "note": ("random-init weights keep the tempered entropies high, so the adaptive "
                     "stop does not fire and every block runs N forwards")}


def run_selfcond(args, w, world, tensors, prompt, eb):
    """The same blocks with self-conditioning (the Report's decoder input z = FFW(p0 E),
    p0 over the whole vocabulary): a second handle on the same weights plus the FFW's
    three tensors (sc_inter = 2048, init std 0.02), device-timed graph replays of
    dg_generate_block, then a profiled pass for the LM head's share (the p0 store, the
    rescale, the K-sliced p0 E^T GEMM and the FFW run inside that group)."""
    import torch

    from masked_discrete_diffusion_b200 import binding
    from synth import gen, model_inputs, workloads
    ws = w.with_(name=w.name + "-sc", sc_inter=2048)
    sc = {}
    for name, shape in model_inputs.global_specs(ws):
        if name.startswith("sc."):
            t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
            gen.fill_weight_(t, ws.seed, name, model_inputs.std_of(ws, name))
            sc[name] = t
    model = binding.Model(binding.make_config(ws, max_prompt=w.prompt_len), dict(tensors, **sc))
    try:
        B, C = w.batch, w.canvas
        kv = binding.dg_prefill(model, prompt)
        out = torch.empty(B, C, dtype=torch.int32, device="cuda")
        nf = torch.zeros(B, dtype=torch.int32, device="cuda")
        for _ in range(max(args.warmup, 1)):
            binding.dg_generate_block(model, kv, w.T, w.gamma, out, nf)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("selfcond")
        e0.record()
        for _ in range(args.steps):
            binding.dg_generate_block(model, kv, w.T, w.gamma, out, nf)
        e1.record()
        e1.synchronize()
        torch.cuda.nvtx.range_pop()
        ms_max = max_over_ranks(e0.elapsed_time(e1), world)
        fwd = int(nf.max().item())
        binding.dg_profile_start(model, fwd)
        binding.dg_generate_block(model, kv, w.T, w.gamma, out, nf)
        torch.cuda.synchronize()
        prof = binding.dg_profile_stop(model)
        binding.dg_sync_status(model)
        assert not bool((out == w.mask_id).any()), "a [MASK] survived the block"
        kv.close()
    finally:
        model.close()
    lm_ms, lm_n = prof["lmhead"]
    return {"sc_inter": 2048, "steps": args.steps,
            "canvas_tokens_per_s": job_throughput(world, B * C, args.steps, ms_max),
            "ms_per_block": ms_max / args.steps, "forwards_per_block": fwd,
            "ms_per_forward": ms_max / args.steps / max(fwd, 1),
            "lmhead_with_selfcond_ms_per_forward": lm_ms / max(lm_n, 1),
            "lmhead_ms_per_forward_without": eb,
            "note": "the LM-head group also holds the p0 store and rescale, the p0 E^T GEMM "
                    "(16 K slices) and the SwiGLU FFW of z"}


def run_ours(args, w, world, rank, local):
    import numpy as np
    import torch

    from masked_discrete_diffusion_b200 import binding, metrics
    from synth import model_inputs

    build_once(world, local)
    peaks, peak_src = load_peaks()
    tensors = model_inputs.weight_set(w, "cuda")
    # the context may grow by the appended blocks of the multi-block measurement
    max_prompt = w.prompt_len + max(args.blocks - 1, 0) * w.canvas
    model = binding.Model(binding.make_config(w, max_prompt=max_prompt), tensors)
    prompt = model_inputs.prompt(w, "cuda", first=rank * w.batch)
    kv = binding.dg_prefill(model, prompt)
    binding.dg_sync_status(model)
    B, C, T = w.batch, w.canvas, w.T
    canvas = torch.empty(B, C, dtype=torch.int32, device="cuda")
    nfwd = torch.zeros(B, dtype=torch.int32, device="cuda")
    load = torch.zeros(w.n_layers, w.n_experts, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        binding.dg_generate_block(model, kv, T, w.gamma, canvas, nfwd, load)
    binding.dg_sync_status(model)

    # nvidia-smi needs a moment before its first sample: the same blocks keep the GPU
    # under the timed load meanwhile, so that the clock samples are taken under load
    clocks = ClockSampler(local)
    clocks.start()
    t_end = time.time() + 0.3
    while time.time() < t_end:
        binding.dg_generate_block(model, kv, T, w.gamma, canvas, nfwd, load)
        torch.cuda.synchronize()
    # timed region: graph replays only (no instrumentation)
    barrier(world)
    torch.cuda.synchronize()
    n0 = binding.dg_launch_count(model)
    torch.cuda.nvtx.range_push("timed")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        binding.dg_generate_block(model, kv, T, w.gamma, canvas, nfwd, load)
    e1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    clk = clocks.stop()
    # the block's device-side loop runs as many forwards as needed (at most T)
    fwd_per_block = int(nfwd.max().item())
    launches = args.steps * (1 + binding.dg_block_loop_launches(model) * fwd_per_block)
    if binding.dg_block_loop_launches(model) == 0:
        launches = binding.dg_launch_count(model) - n0
    ms = e0.elapsed_time(e1)
    binding.dg_sync_status(model)
    barrier(world)
    ms_max = max_over_ranks(ms, world)
    value = job_throughput(world, B * C, args.steps, ms_max)
    ms_step = ms_max / args.steps

    # second pass of the same K steps with CUDA events recorded around every launch group
    # (an unrolled graph of exactly the forwards the timed loop ran, on the same canvases)
    binding.dg_profile_start(model, fwd_per_block)
    for _ in range(args.steps):
        binding.dg_generate_block(model, kv, T, w.gamma, canvas, nfwd, load)
    torch.cuda.synchronize()
    prof = binding.dg_profile_stop(model)
    units = binding.dg_expert_units(model)
    assert not bool((canvas == w.mask_id).any()), "a [MASK] survived the block"

    # end to end through the public API: pinned prompt -> prefill -> block -> canvas to host
    e2e_val = None
    kv_W = kv.W
    kv.close()
    if not args.skip_e2e:
        e2e_val = run_e2e(args, w, world, model, prompt, canvas, stream)
    blocks = run_blocks(args, w, world, model, prompt) if args.blocks > 1 else None
    selfcond = None
    if args.selfcond and w.dtype == "bf16":
        selfcond = run_selfcond(args, w, world, tensors, prompt,
                                prof["lmhead"][0] / max(prof["lmhead"][1], 1))
    annealed = None
    if args.annealed > 0:
        annealed = run_annealed(args, w, world, model, prompt,
                                prof["lmhead"][0] / max(prof["lmhead"][1], 1))
    # roofline of the dominant kernel group (routed-expert FFN); units = experts that
    # received rows, counted per (layer, forward) on the device
    ex_ms, ex_groups = prof["experts"]
    unique_mean = units / max(ex_groups, 1)
    cost = metrics.forward_cost(model.cfg, B, kv_W, [unique_mean] * w.n_layers)
    ex_bytes = unique_mean * cost["expert_bytes"]
    # DRAM traffic of the routed-expert launch: the captured bytes per streamed expert
    # (DRAM_BYTES_PER_EXPERT) times this run's experts per launch
    ex_traffic = (unique_mean * DRAM_BYTES_PER_EXPERT
                  if w.dtype == "bf16" and DRAM_BYTES_PER_EXPERT else None)
    ex_avg_s = ex_ms / 1e3 / max(ex_groups, 1)
    achieved = ex_bytes / ex_avg_s / 1e9
    peak = float(peaks["hbm_gbs"])
    fwd_ms = ms_step / max(fwd_per_block, 1)
    t_roof = max(cost["bytes"] / (peak * 1e9), cost["flops"] / (float(peaks["bf16_tflops"]) * 1e12))
    kinds = {k: {"ms_per_forward": v[0] / args.steps / max(fwd_per_block, 1),
                 "groups_per_forward": v[1] / args.steps / max(fwd_per_block, 1)}
             for k, v in prof.items()}
    main_ms = sum(v["ms_per_forward"] for k, v in kinds.items() if k != "shared")
    # router load of the last timed block: rows each expert received, summed over the
    # block's forwards and layers; and how many experts received rows per layer
    load_np = load.cpu().numpy()
    router_load = {"per_expert_rows": [int(v) for v in load_np.sum(axis=0)],
                   "experts_with_rows_per_layer": float((load_np > 0).sum(axis=1).mean()),
                   "rows_per_layer_per_forward": B * C * w.top_k,
                   "forwards": fwd_per_block}

    line = {
        "metric": "canvas tokens/sec at 1 B200 (256-tok block)", "value": value,
        "unit": "canvas tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights N(0,0.02), uniform prompt tokens)",
        "config": {"workload": w.name, "batch": B, "canvas": C, "prompt": w.prompt_len,
                   "layers": w.n_layers, "T": T, "gamma": w.gamma,
                   "l2": "inputs larger than L2 (40 GB of weights streamed per forward)",
                   "parallelism": f"replicas x{world}"},
        "ms_per_forward": fwd_ms,
        "forwards_per_block": fwd_per_block,
        "tokens_per_forward": C / max(fwd_per_block, 1),
        "forward_roofline": {"ms": t_roof * 1e3, "frac": t_roof * 1e3 / fwd_ms,
                             "alg_bytes": cost["bytes"], "alg_flops": cost["flops"],
                             "peak_src": peak_src},
        "roofline": {"kernel": "routed-expert FFN (gate/up SwiGLU + down) per layer",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": ex_traffic,
                     "alg_bytes_per_launch": ex_bytes, "avg_launch_ms": ex_avg_s * 1e3,
                     "peak_src": f"{peak_src} hbm_gbs"},
        "kernel_groups": kinds,
        "kernel_groups_main_stream_ms_per_forward": main_ms,
        "kernel_groups_note": ("second pass of the same steps and forwards with event records "
                               "around each launch group; 'shared' runs on a concurrent branch, "
                               "the other groups sum to at most ms_per_forward"),
        "router_load": router_load,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": None if e2e_val is None else {
            "value": e2e_val, "unit": "canvas tokens/s",
            "h2d_bytes_per_step": int(prompt.numel() * 4),
            "d2h_bytes_per_step": int(canvas.numel() * 4),
            "includes": "prompt H2D, dg_prefill_into (the slot's KV handle refilled), "
                        "dg_generate_block, canvas D2H, every step"},
        "experts_streamed_per_layer_forward": unique_mean,
        "blocks": blocks,
        "annealed": annealed,
        "selfcond": selfcond,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_block, desc, threads = OracleSample(w).run()
        line["cpu_baseline"] = {"value": B * C / t_block, "unit": "canvas tokens/s",
                                "cores": threads, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="full30-bf16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--selfcond", type=int, default=1,
                    help="1: also time the blocks with self-conditioning (bf16 workloads)")
    ap.add_argument("--annealed", type=int, default=1,
                    help="timed blocks of the annealed sampler (0: skip that leg)")
    ap.add_argument("--blocks", type=int, default=2,
                    help="blocks of the multi-block measurement (1: skip it)")
    args = ap.parse_args()
    from synth import workloads
    w = workloads.get(args.workload)
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, w, world, rank)
        else:
            run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
