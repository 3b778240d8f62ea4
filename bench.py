#!/usr/bin/env python
"""Draft-cycle benchmark: inject(n_new) + draft_block + verify on one B200 per rank.

Prints ONE JSON line (rank 0). Default workload: the Qwen3-8B-shaped drafter,
bf16, batch 1, context 2048, block 16.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A "step" is one full cycle over one batch: inject the features of the a+1
tokens committed by the previous verify (a = planted acceptance length), run
the drafter over the block, verify the block against planted target logits.
`value` times CUDA-graph replays of that cycle with every input resident in
HBM; `e2e` times the same cycle through the public API with inputs copied from
pinned host memory and results copied back every step. Ranks are independent
replicas (the cycle has no cross-GPU exchange); value = all ranks' cycles / max
rank time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft cycles/sec (B-token block, inject+draft+verify) + % HBM/tensor roofline"
UNIT = "cycles/s"
DEFAULT_WORKLOAD = "qwen8b_b16"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-budget-s", type=float, default=25.0)
    ap.add_argument("--block-sweep", action="store_true",
                    help="instead of the headline line: time the cycle at block sizes 4/8/10/16 at concurrency 1 "
                         "and 32 and report the dynamic block-size policy's choice (one JSON line)")
    ap.add_argument("--kv-cache-dtype", default="f16", choices=["model", "f16"],
                    help="element type of the drafter's KV cache pools: f16 (bf16 drafters; same bytes as bf16, "
                         "3 more mantissa bits, read by the attention kernel without conversion) or the model dtype")
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers

def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sus": p["bf16_tflops_sustained"],
                "src": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.idx)], stdout=self.file,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def setup_dist(backend=None):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE): NCCL when
    CUDA is present, gloo otherwise (the host-only tests of the replica logic)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time: every rank's number is device-timed, the job's is the max."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, ms_max: float) -> float:
    """Whole-job cycles/s: every rank runs `steps` cycles of its own replica in ms_max."""
    return world * steps / (ms_max / 1000.0)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------- workload

class Cycle:
    """All device state of one benchmark replica."""

    def __init__(self, w, dev, kv_cache_dtype="model"):
        import torch
        from block_diffusion_speculative_cycle_b200 import Drafter, dflash_verify_workspace_size, synth
        self.w, self.cfg = w, w.cfg
        cfg, bs, B = w.cfg, w.batch, w.block
        self.bs, self.B = bs, B
        weights = synth.make_drafter_weights(cfg, seed=w.seed)
        self.weights_cpu = weights
        wd = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in weights.items() if k != "layers"}
        wd["layers"] = [{k: v.to(dev) for k, v in lw.items()} for lw in weights["layers"]]
        self.wd = wd
        self.ctx_lens = synth.make_ctx_lens(w)
        self.table_cpu, self.num_pages = synth.make_page_table(self.ctx_lens, w.page_size, extra_tokens=B,
                                                               seed=w.seed + 4)
        self.table = self.table_cpu.to(dev)
        self.max_ctx = int(self.ctx_lens.max())
        cache_dt = torch.float16 if kv_cache_dtype == "f16" and cfg.dtype == "bf16" else cfg.torch_dtype
        self.cache_dtype = "f16" if cache_dt == torch.float16 else cfg.dtype
        self.drafter = Drafter(cfg, wd, max_block=B, max_batch=bs, max_inject_rows=bs * B, page_size=w.page_size,
                               cache_dtype=cache_dt)
        # the drafter cache is filled with seeded random K/V (its values do not change the work)
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed + 5)
        shape = (self.num_pages, cfg.n_kv_heads, w.page_size, cfg.head_dim)
        self.kc = [torch.randn(shape, generator=gen, device=dev).mul_(2.0).to(cache_dt) for _ in range(cfg.n_layers)]
        self.vc = [torch.randn(shape, generator=gen, device=dev).to(cache_dt) for _ in range(cfg.n_layers)]
        # step inputs
        self.feats_cpu = synth.make_features(cfg, bs * B, seed=w.seed + 1).reshape(bs, B, cfg.feat_dim)
        self.anchor_cpu = synth.make_tokens(cfg, bs, seed=w.seed + 2)
        self.feats = self.feats_cpu.to(dev)
        self.anchor = self.anchor_cpu.to(dev)
        self.ctx = self.ctx_lens.to(dev)
        self.draft = torch.zeros((bs, max(B - 1, 1)), dtype=torch.int32, device=dev)
        self.acc = torch.zeros(bs, dtype=torch.int32, device=dev)
        self.nxt = torch.zeros(bs, dtype=torch.int32, device=dev)
        self.ws = torch.zeros(dflash_verify_workspace_size(bs, B), dtype=torch.uint8, device=dev)
        # one untimed draft pass gives the tokens the target logits are planted against
        self.drafter.draft(self.anchor, self.ctx, bs, B, self.kc, self.vc, self.table, self.num_pages,
                           self.max_ctx, self.draft)
        self.drafter.check()
        draft_cpu = self.draft.cpu()
        self.logits_cpu, self.planted = synth.planted_logits(draft_cpu, cfg.vocab, w.logit_sigma, w.accept_mean,
                                                             seed=w.seed + 6, dtype=torch.bfloat16)
        self.logits = self.logits_cpu.to(dev)
        # steady state: the previous verify committed a+1 tokens at positions P-a-1 .. P-1
        n_new = torch.clamp(self.planted + 1, max=B).to(torch.int32)
        self.n_new_cpu = n_new
        self.start_cpu = (self.ctx_lens - n_new).clamp(min=0).to(torch.int32)
        self.n_new = n_new.to(dev)
        self.start = self.start_cpu.to(dev)

    def run(self, stream=None):
        from block_diffusion_speculative_cycle_b200 import dflash_verify
        self.drafter.inject(self.feats, self.bs, self.B, self.n_new, self.start, self.kc, self.vc, self.table,
                            self.num_pages, stream)
        self.drafter.draft(self.anchor, self.ctx, self.bs, self.B, self.kc, self.vc, self.table, self.num_pages,
                           self.max_ctx, self.draft, None, stream)
        dflash_verify(self.logits, self.draft, self.acc, self.nxt, self.ws, stream)


def algorithmic_cycle_bytes(c) -> float:
    """Every weight the cycle reads, once per use: the drafter layers' weights,
    the LM head and the fusion projection, plus every layer's Wk and Wv a second
    time for the injection; the context K/V each request attends to, the
    features and the block logits. Activations are negligible at these sizes."""
    cfg = c.cfg
    es = 2 if cfg.dtype == "bf16" else 4
    H, I, L = cfg.hidden, cfg.intermediate, cfg.n_layers
    per_layer = (2 * cfg.q_dim * H + 2 * cfg.kv_dim * H + 3 * I * H) * es
    inject_kv = L * 2 * cfg.kv_dim * H * es
    weights = L * per_layer + cfg.vocab * H * es + H * cfg.feat_dim * es + inject_kv
    kv = float(c.ctx_lens.sum()) * L * 2 * cfg.kv_dim * es
    feats = c.bs * c.B * cfg.feat_dim * es
    logits = c.bs * c.B * cfg.vocab * 2
    return weights + kv + feats + logits


# --------------------------------------------------------------------------- CPU oracle sample

class HostCycle:
    """The inputs of one cycle built on the host only (no GPU): the draft tokens
    the logits are planted against are drawn at random instead of drafted."""

    def __init__(self, w, kv_cache_dtype="model"):
        import torch
        from block_diffusion_speculative_cycle_b200 import synth
        cfg, bs, B = w.cfg, w.batch, w.block
        self.w, self.cfg, self.bs, self.B = w, cfg, bs, B
        self.cache_dtype = "f16" if kv_cache_dtype == "f16" and cfg.dtype == "bf16" else cfg.dtype
        self.weights_cpu = synth.make_drafter_weights(cfg, seed=w.seed)
        self.ctx_lens = synth.make_ctx_lens(w)
        self.feats_cpu = synth.make_features(cfg, bs * B, seed=w.seed + 1).reshape(bs, B, cfg.feat_dim)
        self.anchor_cpu = synth.make_tokens(cfg, bs, seed=w.seed + 2)
        self.draft = synth.make_tokens(cfg, bs * max(B - 1, 1), seed=w.seed + 3).reshape(bs, max(B - 1, 1))
        self.logits_cpu, self.planted = synth.planted_logits(self.draft, cfg.vocab, w.logit_sigma, w.accept_mean,
                                                             seed=w.seed + 6, dtype=torch.bfloat16)
        self.n_new_cpu = torch.clamp(self.planted + 1, max=B).to(torch.int32)
        self.start_cpu = (self.ctx_lens - self.n_new_cpu).clamp(min=0).to(torch.int32)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown CPU"


def oracle_cycle_estimate(c, budget_s: float):
    """Time the oracle (float64 NumPy, as it stands) on a bounded sample of one
    request's cycle and extrapolate to the whole batch: inject of n_new rows,
    one drafter layer (attention over the request's context + MLP), the final
    norm + LM head on a vocab slice + argmax, and verify of one block."""
    import numpy as np
    import torch
    from oracle import dflash as O
    cfg, w = c.cfg, c.weights_cpu
    B = c.B
    P = int(c.ctx_lens[0])
    g = torch.Generator().manual_seed(99)
    k_ctx = (torch.randn((P, cfg.n_kv_heads, cfg.head_dim), generator=g) * 2.0).to(cfg.torch_dtype)
    v_ctx = torch.randn((P, cfg.n_kv_heads, cfg.head_dim), generator=g).to(cfg.torch_dtype)
    k64, v64 = O.f64(k_ctx), O.f64(v_ctx)
    x = O.f64(w["embed"][[int(c.anchor_cpu[0])] + [cfg.mask_token_id] * (B - 1)])
    pos = np.arange(P, P + B)
    n_slices = 16 if cfg.vocab >= 16 * 128 else 1
    vs = cfg.vocab // n_slices
    times = {"inject": [], "layer": [], "lm_slice": [], "verify": []}
    t_end = time.time() + budget_s
    while True:
        t0 = time.perf_counter()
        O.inject(cfg, w, c.feats_cpu[0, : int(c.n_new_cpu[0])], int(c.start_cpu[0]))
        t1 = time.perf_counter()
        O.drafter_layer(cfg, w["layers"][0], x, pos, k64, v64)
        t2 = time.perf_counter()
        y = O.rms_norm(x, w["final_norm"], cfg.rms_eps)
        lg = O.linear(y[1:], w["lm_head"][:vs])
        [O.greedy_argmax(r) for r in lg]
        t3 = time.perf_counter()
        O.verify(O.f64(c.logits_cpu[0]), c.draft.cpu().numpy()[0])
        t4 = time.perf_counter()
        for k, v in zip(times, (t1 - t0, t2 - t1, t3 - t2, t4 - t3)):
            times[k].append(v)
        if time.time() > t_end or len(times["layer"]) >= 5:
            break
    med = {k: statistics.median(v) for k, v in times.items()}
    per_request = med["inject"] + cfg.n_layers * med["layer"] + n_slices * med["lm_slice"] + med["verify"]
    cycle_s = per_request * c.bs
    cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        info = [p for p in threadpool_info() if p.get("internal_api") in ("openblas", "mkl", "blis")]
        if info:
            cores = max(p.get("num_threads", 1) for p in info)
    except Exception:
        pass
    sample = (f"float64 NumPy oracle on {cpu_model()}: 1 of {c.bs} requests; inject {int(c.n_new_cpu[0])} rows "
              f"+ 1 of {cfg.n_layers} layers (context {P}) + final norm and LM head on 1/{n_slices} of the vocab "
              f"+ verify; {len(times['layer'])} repeats, median, extrapolated to the full batch cycle")
    return 1.0 / cycle_s, cores, sample


# --------------------------------------------------------------------------- arms

def run_reference(args, world, rank):
    """The oracle on the host cores, same workload / metric / unit as our arm."""
    if rank != 0:
        return
    from block_diffusion_speculative_cycle_b200 import synth
    w = synth.WORKLOADS[args.workload]
    # inputs built on the host only: this arm never loads the CUDA library
    c = HostCycle(w, args.kv_cache_dtype)
    steps = max(1, args.steps)
    budget_per_step = max(2.0, 150.0 / (steps + args.warmup))
    vals = []
    t0 = time.time()
    for i in range(args.warmup + steps):
        v, cores, sample = oracle_cycle_estimate(c, budget_per_step)
        if i >= args.warmup:
            vals.append(v)
        if time.time() - t0 > 180:
            break
    value = statistics.median(vals) if vals else v
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
           "steps": len(vals), "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(w, c),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def workload_config(w, c):
    cfg = w.cfg
    ctx = (f"{w.ctx_range[0]}-{w.ctx_range[1]} uniform" if w.ctx_range else w.ctx_len)
    return {"workload": f"{w.name}: {cfg.name}, {cfg.dtype}, H{cfg.hidden} L{cfg.n_layers} "
                        f"{cfg.n_q_heads}q/{cfg.n_kv_heads}kv x{cfg.head_dim} I{cfg.intermediate} V{cfg.vocab}, "
                        f"features {cfg.n_feat_layers}x{cfg.target_hidden}",
            "global_batch": w.batch, "block": w.block, "ctx_len": ctx, "page_size": w.page_size,
            "kv_cache_dtype": c.cache_dtype if c is not None else cfg.dtype,
            "planted_accept_mean": w.accept_mean,
            "l2": "inputs larger than L2: every cycle streams all drafter + LM-head weights (GBs) from HBM",
            "parallelism": "replicas (one independent drafter per GPU)"}


def run_ours(args, world, rank, local):
    import torch
    from block_diffusion_speculative_cycle_b200 import dflash_profile_enable, dflash_profile_read, synth
    w = synth.WORKLOADS[args.workload]
    dev = f"cuda:{local}"
    c = Cycle(w, dev, args.kv_cache_dtype)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    # eager warm-up, then capture one cycle in a CUDA graph
    with torch.cuda.stream(stream):
        for _ in range(3):
            c.run()
    torch.cuda.synchronize()
    c.drafter.check()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        c.run()
    torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()
    c.drafter.check()

    # ---- timed region: K graph replays, inputs resident in HBM
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        ev0.record()
        for _ in range(args.steps):
            graph.replay()
        ev1.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world)
    value = job_throughput(world, args.steps, ms_max)
    clk = clocks.summary()
    c.drafter.check()

    # ---- profiling pass (eager): per-kernel event timings inside the cycle
    prof_stream = torch.cuda.current_stream()
    dflash_profile_enable(c.drafter.handle, True)
    from block_diffusion_speculative_cycle_b200 import dflash_verify
    v_ms = 0.0
    for _ in range(args.profile_steps):
        c.drafter.inject(c.feats, c.bs, c.B, c.n_new, c.start, c.kc, c.vc, c.table, c.num_pages)
        c.drafter.draft(c.anchor, c.ctx, c.bs, c.B, c.kc, c.vc, c.table, c.num_pages, c.max_ctx, c.draft)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(prof_stream)
        dflash_verify(c.logits, c.draft, c.acc, c.nxt, c.ws)
        b.record(prof_stream)
        torch.cuda.synchronize()
        v_ms += a.elapsed_time(b)
    prof = dflash_profile_read(c.drafter.handle)
    dflash_profile_enable(c.drafter.handle, False)
    prof.append({"name": "verify", "launches": args.profile_steps, "total_ms": v_ms,
                 "bytes": args.profile_steps * (c.bs * c.B * c.cfg.vocab * 2 + c.bs * c.B * 8.0), "flops": 0.0})
    kernels_per_cycle = sum(e["launches"] for e in prof) / args.profile_steps

    # the dominant kernel: GEMM call sites share one kernel, so they are summed
    kinds = {}
    for e in prof:
        k = e["name"].split(":")[0]
        d = kinds.setdefault(k, {"name": k, "launches": 0, "total_ms": 0.0, "bytes": 0.0, "flops": 0.0})
        for f in ("launches", "total_ms", "bytes", "flops"):
            d[f] += e[f]
    pk = peaks()
    dom = max(kinds.values(), key=lambda e: e["total_ms"])
    avg_s = dom["total_ms"] / dom["launches"] / 1000.0
    timing = "eager, an event pair around every launch (no overlap between launches)"
    if dom["name"] == "gemm_tc":
        # Inside the cycle the GEMMs overlap each other's ramp and tail (programmatic
        # dependent launch), which event pairs around single launches remove: time a
        # CUDA graph of exactly the cycle's GEMM launches instead, K replays.
        from block_diffusion_speculative_cycle_b200 import dflash_profile_gemm_chain
        g3 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g3, stream=stream):
            dflash_profile_gemm_chain(c.drafter.handle, c.feats, c.bs, c.B, c.n_new, c.start, c.kc, c.vc, c.table,
                                      c.num_pages, c.ctx, c.B)
        for _ in range(3):
            g3.replay()
        torch.cuda.synchronize()
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(3, min(args.steps, 100))
        ga.record()
        for _ in range(reps):
            g3.replay()
        gb.record()
        torch.cuda.synchronize()
        c.drafter.check()
        chain_s = ga.elapsed_time(gb) / 1000.0 / reps
        per_cycle = dom["launches"] / args.profile_steps
        avg_s = chain_s / per_cycle
        timing = (f"in-cycle: a CUDA graph of the cycle's {per_cycle:.0f} GEMM launches (programmatic dependent "
                  f"launch on), {reps} replays, {1e6 * chain_s:.1f} us per cycle")
        del g3
    bytes_per_launch = dom["bytes"] / dom["launches"]
    flops_per_launch = dom["flops"] / dom["launches"]
    intensity = flops_per_launch / max(bytes_per_launch, 1.0)
    tensor_bound = dom["name"].startswith("gemm_tc") and intensity > pk["bf16_sus"] * 1e12 / (pk["hbm"] * 1e9)
    if tensor_bound:
        achieved = flops_per_launch / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_sus"], "peak_source": f"{pk['src']} bf16 sustained"}
    else:
        achieved = bytes_per_launch / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "peak_source": f"{pk['src']} hbm copy"}
    roof["kernel"] = dom["name"]
    roof["us_per_launch"] = 1e6 * avg_s
    roof["bytes_per_launch"] = bytes_per_launch
    roof["timing"] = timing
    roof["traffic"] = stored_traffic(dom["name"], w.name)
    cycle_bytes = algorithmic_cycle_bytes(c)
    per_gpu_cycle_s = (ms_max / 1000.0) / args.steps
    roof["cycle_hbm_frac"] = cycle_bytes / per_gpu_cycle_s / 1e9 / pk["hbm"]
    roof["cycle_bytes"] = cycle_bytes

    # ---- end to end through the public API, host buffers, copies inside the timed region.
    # Every step copies its own inputs (features of the committed tokens, the
    # target's block logits, per-request scalars) from pinned host memory and
    # reads its results (accepted length, next token, drafts) back. Inputs are
    # double-buffered: step k+1's copies run on a copy stream while step k
    # computes. The cycle itself is the public API's inject + draft + verify,
    # captured once per input buffer in a CUDA graph (all cycle-varying inputs are
    # device pointers), so a step costs one graph launch on the host.
    from block_diffusion_speculative_cycle_b200 import dflash_verify
    h_feats = c.feats_cpu.pin_memory()
    h_logits = c.logits_cpu.pin_memory()
    h_small = torch.stack([c.anchor_cpu, c.ctx_lens, c.n_new_cpu, c.start_cpu]).to(torch.int32).pin_memory()
    # results land in contiguous pinned buffers (a strided host view would make the copy synchronous)
    h_acc = torch.empty(c.bs, dtype=torch.int32).pin_memory()
    h_nxt = torch.empty(c.bs, dtype=torch.int32).pin_memory()
    h_draft = torch.empty(tuple(c.draft.shape), dtype=torch.int32).pin_memory()
    d_feats = [torch.empty_like(c.feats) for _ in range(2)]
    d_logits = [torch.empty_like(c.logits) for _ in range(2)]
    d_small = [torch.empty_like(h_small, device=dev) for _ in range(2)]
    for buf in range(2):
        d_feats[buf].copy_(h_feats)
        d_logits[buf].copy_(h_logits)
        d_small[buf].copy_(h_small)
    e2e_graphs = []
    for buf in range(2):
        g2 = torch.cuda.CUDAGraph()
        sm = d_small[buf]
        with torch.cuda.graph(g2, stream=stream):
            c.drafter.inject(d_feats[buf], c.bs, c.B, sm[2], sm[3], c.kc, c.vc, c.table, c.num_pages)
            c.drafter.draft(sm[0], sm[1], c.bs, c.B, c.kc, c.vc, c.table, c.num_pages, c.max_ctx, c.draft)
            dflash_verify(d_logits[buf], c.draft, c.acc, c.nxt, c.ws)
        e2e_graphs.append(g2)
    torch.cuda.synchronize()
    comp = stream
    copy = torch.cuda.Stream(device=dev)
    ev_ready = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = min(args.e2e_steps, args.steps)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    copy.wait_event(e0)

    def stage_inputs(k):
        buf = k % 2
        with torch.cuda.stream(copy):
            if k >= 2:
                copy.wait_event(ev_free[buf])
            d_feats[buf].copy_(h_feats, non_blocking=True)
            d_logits[buf].copy_(h_logits, non_blocking=True)
            d_small[buf].copy_(h_small, non_blocking=True)
            ev_ready[buf].record(copy)

    stage_inputs(0)
    with torch.cuda.stream(comp):
        for k in range(e2e_steps):
            if k + 1 < e2e_steps:
                stage_inputs(k + 1)
            buf = k % 2
            comp.wait_event(ev_ready[buf])
            e2e_graphs[buf].replay()
            ev_free[buf].record(comp)
            h_acc.copy_(c.acc, non_blocking=True)
            h_nxt.copy_(c.nxt, non_blocking=True)
            h_draft.copy_(c.draft, non_blocking=True)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_throughput(world, e2e_steps, e2e_ms)
    h2d = h_feats.numel() * h_feats.element_size() + h_logits.numel() * h_logits.element_size() + h_small.numel() * 4
    d2h = c.bs * (2 + max(c.B - 1, 1)) * 4
    c.drafter.check()

    # ---- CPU oracle baseline (rank 0, single GPU only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_cycle_estimate(c, args.cpu_budget_s)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.cfg.dtype == "bf16" else "f32",
               "data": "synthetic (seeded random weights, features, tokens, planted-prefix logits)",
               "config": workload_config(w, c), "roofline": roof, "cpu_baseline": cpu,
               "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "steps": e2e_steps},
               "gpu_launches": int(round(kernels_per_cycle * args.steps)),
               "kernels_per_cycle": kernels_per_cycle,
               "profile": [{"name": e["name"], "launches": e["launches"],
                            "us_per_launch": 1000.0 * e["total_ms"] / e["launches"],
                            "gbs": e["bytes"] / (e["total_ms"] / 1000.0) / 1e9 if e["total_ms"] > 0 else None}
                           for e in prof],
               "clocks": clk}
        print(json.dumps(out), flush=True)
    del graph, e2e_graphs


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture of this exact kernel
    source, else null."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "block_diffusion_speculative_cycle_b200", "csrc", rec[kernel]["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        r = rec[kernel]
        if r["sha"] == h and r["workload"] == workload:
            return r["bytes_per_launch"]
    except Exception:
        pass
    return None


def block_sweep(args, local):
    """Dynamic block-size scheduling on measured cycles: for each concurrency, the
    cycle (inject + draft + verify) is graph-timed at every candidate block size
    with the same drafter, the acceptance lengths of those cycles (the planted
    prefixes) feed the library's device acceptance counts, and the library's
    policy picks the block with the most expected tokens per measured cycle time.
    Prints one JSON line."""
    import dataclasses
    import torch
    from block_diffusion_speculative_cycle_b200 import BlockPolicy, dflash_acceptance_count, dflash_verify, synth
    cands, n_pos = [4, 8, 10, 16], 17
    out = {"metric": "block-size policy on measured cycles", "candidates": cands, "rows": []}
    dev = f"cuda:{local}"
    for name in ("qwen8b_b16_serve_bs1", "qwen8b_b16_serve_bs32"):
        w = synth.WORKLOADS[name]
        c = Cycle(dataclasses.replace(w, block=max(cands)), dev, args.kv_cache_dtype)
        counts = torch.zeros(2 * n_pos, dtype=torch.int64, device=dev)
        row = {"workload": name, "batch": w.batch, "ms_per_cycle": {}, "expected_tokens": {}}
        costs = []
        for B in cands:
            logits = c.logits[:, :B].contiguous()
            draft = torch.zeros((c.bs, max(B - 1, 1)), dtype=torch.int32, device=dev)
            n_new = torch.clamp(c.n_new, max=B).contiguous()
            ws = torch.zeros(c.ws.numel(), dtype=torch.uint8, device=dev)

            def cycle():
                c.drafter.inject(c.feats, c.bs, c.B, n_new, c.start, c.kc, c.vc, c.table, c.num_pages)
                c.drafter.draft(c.anchor, c.ctx, c.bs, B, c.kc, c.vc, c.table, c.num_pages, c.max_ctx, draft)
                dflash_verify(logits, draft, c.acc, c.nxt, ws)
            for _ in range(3):
                cycle()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                cycle()
            for _ in range(5):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 30
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            row["ms_per_cycle"][B] = ms
            costs.append(ms)
            # The synthetic target accepts a geometric prefix (mean 6, the planted law) at
            # any block size, clipped at B-1; the logits were planted against the
            # block-16 draft, so a smaller block's own verify would mismatch for a
            # synthetic reason. Clipped draws of that law feed the device counts.
            # Acceptance statistics need many draws: 4096 seeded geometric lengths per block.
            gen = torch.Generator().manual_seed(1234 + B)
            p_geo = 1.0 / (1.0 + w.accept_mean)
            u = torch.rand(4096, generator=gen, dtype=torch.float64)
            geo = torch.floor(torch.log1p(-u) / math.log1p(-p_geo))
            planted = torch.clamp(geo, max=B - 1).to(torch.int32).to(dev)
            dflash_acceptance_count(planted, B, counts)
            del g
        torch.cuda.synchronize()
        c.drafter.check()
        cnt = counts.cpu().numpy()
        pol = BlockPolicy(cands, 1.0, n_pos)
        pol.observe(cnt[:n_pos], cnt[n_pos:])
        for B in cands:
            row["expected_tokens"][B] = pol.expected_tokens(B)
        row["tokens_per_s"] = {B: c.bs * row["expected_tokens"][B] / (row["ms_per_cycle"][B] / 1e3) for B in cands}
        row["policy_choice"] = pol.choose(costs)
        row["best_by_measurement"] = max(cands, key=lambda B: row["tokens_per_s"][B])
        out["rows"].append(row)
        pol.close()
        del c
        torch.cuda.empty_cache()
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    world, rank, local = setup_dist()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.block_sweep:
            block_sweep(args, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
