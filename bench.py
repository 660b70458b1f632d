#!/usr/bin/env python3
"""Throughput of the block discrete-diffusion denoising step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
    python bench.py --impl reference --reference-sample full --steps 1 --warmup 0
    python bench.py --timeline        (per-kernel spans inside the step's graph)
    python bench.py --batch-sweep 1,2,4,8,16,32

One step = one dg_denoise_step call: embedding, 30 MoE transformer layers over
the 256-token canvas with bidirectional attention against the prefix KV cache,
the tied 262144-vocabulary LM head fused with the argmax / log-sum-exp
reduction, and the Philox re-noising sampler.  Workload: the 26B-A4B-shaped
model, batch 1, 2048-token uniform-random prefix (seeded synthetic weights
and tokens).  Each step streams ~32 GB of weights (the experts the step
actually routes to), far more than the 126 MB L2, so no flush is needed
between steps.

Multi-GPU: independent replicas (one per rank, no collective on the data
path); value = canvas tokens of all ranks / max-over-ranks time.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
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

METRIC = "canvas tokens denoised/s (batch 1, 256-tok block) and % of step roofline"
UNIT = "canvas tokens/s"


def run_timeline(args, w):
    """Per-kernel device time inside the step's CUDA graph.  The timeline build
    of the library records every CTA's start and end (%globaltimer); one
    graph-replayed step after the warm-up is rebuilt into its launch sequence:
    per kernel the launches, summed and mean spans, share of the step, and the
    idle gaps between launches.  The records add one atomic and two timer
    reads per CTA, so the step is not a bench number."""
    import torch

    import block_discrete_diffusion_denoise_b200 as dgp
    import synth_inputs as si

    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    weights = si.model_weights(w, "cuda")
    cfg = dgp.config_from_shape(w.shape, max_batch=w.batch, max_seq=w.prefix + 2 * w.canvas, canvas=w.canvas)
    ctx = dgp.Context(cfg, weights, stream=stream.cuda_stream)
    ctx.prefill(si.uniform_tokens(w, "prefix", w.batch, w.prefix, device="cuda"))
    cur = si.uniform_tokens(w, "canvas", w.batch, w.canvas, device="cuda")
    nxt = torch.empty_like(cur)
    conf = torch.empty(w.batch, w.canvas, dtype=torch.float32, device="cuda")
    for s in range(args.warmup):
        ctx.denoise_step(cur, s, w.sample_seed, si.tau_schedule(w, s), nxt, conf)
        cur, nxt = nxt, cur
    steps = []
    for s in range(args.steps):
        ctx.debug_timeline_reset()
        ctx.denoise_step(cur, s, w.sample_seed, si.tau_schedule(w, s % w.steps), nxt, conf)
        cur, nxt = nxt, cur
        rec, n = ctx.debug_timeline()
        steps.append(dgp.timeline_summary(dgp.timeline_launches(rec)))
    ctx.close()
    # the step with the median wall time
    med = sorted(steps, key=lambda x: x["wall_us"])[len(steps) // 2]
    print(json.dumps({"timeline": f"{w.name}: {w.description}", "library": os.path.basename(dgp.LIB_PATH),
                      "steps": args.steps, "warmup": args.warmup,
                      "wall_us_per_step": [round(x["wall_us"], 1) for x in steps], "median_step": med}),
          flush=True)


def run_variants(args, w):
    """Cost of the step's variants on one context: the threshold sampler (the
    bench step), the entropy-constrained sampler with the 0.8 -> 0.4
    temperature schedule and the adaptive-stop test (codemajin.net section
    3.3), and self-conditioning on (section 3.2: the probability pass, p E and
    the SwiGLU layer).  CUDA events around `steps` graph-replayed steps each."""
    import torch

    import block_discrete_diffusion_denoise_b200 as dgp
    import synth_inputs as si

    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    weights = si.model_weights(w, "cuda")
    weights.update(si.self_cond_weights(w, "cuda"))
    cfg = dgp.config_from_shape(w.shape, max_batch=w.batch, max_seq=w.prefix + 2 * w.canvas, canvas=w.canvas)
    ctx = dgp.Context(cfg, weights, stream=stream.cuda_stream)
    ctx.prefill(si.uniform_tokens(w, "prefix", w.batch, w.prefix, device="cuda"))
    B, C = w.batch, w.canvas
    cur = si.uniform_tokens(w, "canvas", B, C, device="cuda")
    nxt = torch.empty_like(cur)
    conf = torch.empty(B, C, dtype=torch.float32, device="cuda")
    am = [torch.empty(B, C, dtype=torch.int32, device="cuda") for _ in range(2)]
    ent = torch.empty(B, C, dtype=torch.float32, device="cuda")
    stopped = torch.empty(B, dtype=torch.int32, device="cuda")

    def threshold(s):
        ctx.denoise_step(cur, s, w.sample_seed, w.tau0, nxt, conf)

    def entropy(s):
        temp = 0.8 - 0.4 * min(s, 47) / 47.0
        ctx.denoise_step_entropy(cur, s, w.sample_seed, temp, 8.0, 0.5, nxt,
                                 prev_argmax=None if s == 0 else am[(s + 1) % 2], argmax_out=am[s % 2],
                                 entropy=ent, stopped=stopped)

    def timed(fn):
        nonlocal cur, nxt
        for s in range(args.warmup):
            fn(s)
            cur, nxt = nxt, cur
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(args.steps):
            fn(args.warmup + s)
            cur, nxt = nxt, cur
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    rows = {"threshold_sampler_ms": timed(threshold), "entropy_sampler_ms": timed(entropy)}
    ctx.set_self_conditioning(True)
    rows["self_conditioning_ms"] = timed(threshold)
    ctx.close()
    print(json.dumps({"variants": f"{w.name}: {w.description}", "steps": args.steps, "warmup": args.warmup,
                      **{k: round(v, 4) for k, v in rows.items()}}), flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="a4b_p2k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-sample", choices=["bounded", "full"], default="bounded",
                    help="--impl reference: time a bounded sample of each step (default, minutes in all) "
                         "or whole oracle steps over every layer and the full vocabulary (the a4b step "
                         "takes minutes per step on the host cores and holds its bf16 weights, ~50 GB, "
                         "in host memory)")
    ap.add_argument("--layers", type=int, default=0,
                    help="reduced depth (profiling captures only; not a bench number)")
    ap.add_argument("--batch-sweep", default="",
                    help="comma-separated batch sizes: step throughput and roofline bound per batch "
                         "(one JSON line of its own, not the bench line)")
    ap.add_argument("--variants", action="store_true",
                    help="step time with the threshold sampler, the entropy-constrained sampler and "
                         "self-conditioning (one JSON line of its own, not the bench line)")
    ap.add_argument("--timeline", action="store_true",
                    help="per-kernel spans and launch gaps of graph-replayed steps from libdg_timeline.so "
                         "(one JSON line of its own, not the bench line)")
    return ap.parse_args()


PEAK_NOTE = {"measured": "of measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)",
             "fallback": "of fallback (MEASURED_PEAKS.json absent: 6.65 TB/s copy, 1.59/1.4 PF/s bf16 "
                         "burst/sustained measured earlier on this GPU type)"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic bytes / flops of one step
# ---------------------------------------------------------------------------
def step_cost(w, hits):
    """bytes: every weight the step must read once (routed experts counted
    from the experts actually hit, per layer) + the KV cache read; flops:
    2 x active parameters per token + attention."""
    s = w.shape
    d, D, Hq, Hkv = s.d_model, s.head_dim, s.n_q_heads, s.n_kv_heads
    B, C, P, L = w.batch, w.canvas, w.prefix, s.n_layers
    attn_w = (s.qkv_dim * d + d * Hq * D) * 2
    router_w = s.n_experts * d * 2
    expert_w = 3 * s.expert_hidden * d * 2
    shared_w = 3 * s.shared_hidden * d * 2
    lm_w = s.vocab * d * 2
    kv = L * B * (P + C) * Hkv * D * 2 * 2
    by = sum(attn_w + router_w + hits[l] * expert_w + shared_w for l in range(L)) + lm_w + kv
    active = L * (s.qkv_dim * d + d * Hq * D + s.n_experts * d + s.top_k * 3 * s.expert_hidden * d
                  + 3 * s.shared_hidden * d) + s.vocab * d
    fl = 2.0 * active * B * C + 4.0 * Hq * D * C * (P + C) * L * B
    moe_bytes = sum(hits[l] * expert_w + shared_w for l in range(L)) / L
    return by, fl, moe_bytes


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    """nvidia-smi sampler started before the warm-up; stop(t0, t1) keeps the
    samples whose timestamps fall in the timed window [t0, t1] (host clock)."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "50"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self, t0=None, t1=None):
        if self.p is None:
            return None
        time.sleep(0.1)  # let the sampler record the end of the window
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = [[x.strip() for x in r.split(",")] for r in open(self.f.name).read().strip().splitlines()
                if r.count(",") >= 9]
        os.unlink(self.f.name)

        def stamp(r):
            try:
                return datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                return None
        if t0 is not None and t1 is not None:
            inside = [r for r in rows if (stamp(r) is not None and t0 - 0.06 <= stamp(r) <= t1 + 0.06)]
            rows = inside or rows
        if not rows:
            return None
        sm = [float(r[2]) for r in rows]
        mx = max(float(r[3]) for r in rows)
        reasons = set()
        for r in rows:
            for name, col in (("hw_slowdown", 6), ("hw_thermal_slowdown", 7), ("sw_thermal_slowdown", 8),
                              ("sw_power_cap", 9)):
                if r[col].lower().startswith("active"):
                    reasons.add(name)
        loaded = [x for x in sm if x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# replicas: one process per GPU, no collective on the data path
# ---------------------------------------------------------------------------
def code_sha256(path: str) -> str:
    """sha256 of a CUDA/C++ source with its comments removed and whitespace
    collapsed: the identity of the code a set of ncu counters was taken on,
    unchanged by edits to comments or layout, changed by any edit to code."""
    import hashlib
    import re
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256(" ".join(src.split()).encode()).hexdigest()


L2_BYTES = 126e6      # B200 L2


def l2_note(step_bytes: float) -> str:
    """How the timed steps stand to the L2: a step that streams more than the
    L2 holds needs no flush between steps; a smaller one runs from L2."""
    if step_bytes > L2_BYTES:
        return f"inputs larger than L2 ({step_bytes / 1e9:.1f} GB of weights and cache streamed per step); no flush"
    return (f"inputs fit in L2 ({step_bytes / 1e6:.0f} MB per step) and are not flushed between steps: "
            f"an L2-resident, latency-bound size")


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's value; every rank must call it (a no-op on one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replicas_value(world: int, batch: int, canvas: int, ms: float) -> float:
    """Whole-job canvas tokens/s: each of `world` ranks denoises its own batch
    of `batch` sequences in `ms` milliseconds (the slowest rank's time)."""
    return world * batch * canvas / (ms * 1e-3)


# ---------------------------------------------------------------------------
# oracle timing (host cores)
# ---------------------------------------------------------------------------
def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"),
                default=0)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count() or 1


class OracleSample:
    """The fp64 oracle timed on a bounded sample of one step: layer 0 over the
    whole canvas (scaled by the layer count) and the LM head over a fraction
    of the vocabulary (scaled up).  Weight generation and the prefix cache are
    set up once, outside the timing; bf16 -> fp64 weight conversion, which the
    oracle does as part of its step, is inside."""

    def __init__(self, w):
        import oracle
        import synth_inputs as si
        self.w = w
        self.orc = oracle.for_workload(w.with_layers(1), keep_layers=True)
        self.orc.prefill(si.uniform_tokens(w, "prefix", w.batch, w.prefix).numpy())
        self.canvas = si.uniform_tokens(w, "canvas", w.batch, w.canvas).numpy()

    VOCAB_FRAC = 1.0 / 8          # one sample definition for both the cpu_baseline and the reference arm

    def run(self, vocab_frac=VOCAB_FRAC):
        """Returns (canvas tokens/s of the full step extrapolated from the
        sample, extrapolated full-step seconds, seconds the sample took,
        description)."""
        import numpy as np
        from oracle.model import _f64, _index, lm_head_stats, rms_norm
        w, orc = self.w, self.orc
        for lw in orc._layers.values():          # keep the generated bf16 tensors, redo conversions
            lw._cache.clear()
        t0 = time.perf_counter()
        hs = []
        for b in range(w.batch):
            h = _f64(orc.embed[_index(self.canvas[b])])
            h, _, _ = orc._layer_forward(0, h, b, orc.P, causal=False)
            hs.append(h)
        t_layer = time.perf_counter() - t0
        z = rms_norm(np.concatenate(hs), orc.final_norm, w.shape.rms_eps)
        V = w.shape.vocab
        nv = max(128, int(V * vocab_frac)) // 128 * 128
        t0 = time.perf_counter()
        lm_head_stats(z, orc.embed[:nv], 1.0)
        t_lm_sample = time.perf_counter() - t0
        t_lm = t_lm_sample * V / nv
        t_step = w.shape.n_layers * t_layer + t_lm
        desc = (f"oracle (fp64 numpy) layer 0 of {w.shape.n_layers} over the {w.batch}x{w.canvas} canvas "
                f"with the {w.prefix}-token cache ({t_layer:.2f} s, scaled x{w.shape.n_layers}) + LM head "
                f"over {nv} of {V} vocabulary rows ({t_lm_sample:.2f} s, scaled to the full vocabulary); "
                f"extrapolated full step {t_step:.1f} s")
        return w.batch * w.canvas / t_step, t_step, t_layer + t_lm_sample, desc


class OracleFullStep:
    """The fp64 oracle timed on whole steps: every layer over the whole canvas,
    then the LM head over the full vocabulary and the sampler.  Each layer's
    seeded bf16 weights are generated once, during the (untimed) prefill, and
    kept in host memory; the bf16 -> fp64 conversions the oracle makes during
    its step are inside the timing, as in the bounded sample."""

    def __init__(self, w):
        import oracle
        import synth_inputs as si
        self.w = w
        bf16 = {}

        def layer_fn(l):
            if l not in bf16:
                bf16[l] = si.layer_weights(w, l, "cpu")
            return bf16[l]

        g = si.global_weights(w, "cpu")
        self.orc = oracle.Oracle(oracle.shape_of(w), layer_fn, g["embed"], g["final_norm"], g["router_bias"],
                                 batch=w.batch, keep_layers=False)
        self.orc.prefill(si.uniform_tokens(w, "prefix", w.batch, w.prefix).numpy())
        self.canvas = si.uniform_tokens(w, "canvas", w.batch, w.canvas).numpy()

    def run(self, step=0):
        """Returns (canvas tokens/s, step seconds, step seconds, description)."""
        w = self.w
        t0 = time.perf_counter()
        self.orc.denoise_step(self.canvas, step, w.sample_seed, w.tau0)
        t = time.perf_counter() - t0
        desc = (f"oracle (fp64 numpy) whole step: {w.shape.n_layers} layers over the {w.batch}x{w.canvas} canvas "
                f"with the {w.prefix}-token cache, LM head over all {w.shape.vocab} vocabulary rows, sampler")
        return w.batch * w.canvas / t, t, t, desc


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    vals, spent = [], []
    desc = ""
    full = args.reference_sample == "full"
    sample = OracleFullStep(w) if full else OracleSample(w)
    for i in range(args.warmup + args.steps):
        v, t, t_sample, desc = sample.run()
        if i >= args.warmup:
            vals.append(t)
            spent.append(t_sample)
    t = statistics.median(vals)
    value = w.batch * w.canvas / t
    cores = _cores()
    # each timed step is one bounded sample of the step (ms_per_step: the time
    # it took; value: the full step's throughput extrapolated from it), or
    # with --reference-sample full one whole step
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(spent) * 1e3,
            "extrapolated_ms_per_full_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name}: {w.description}"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if full:
        line.pop("extrapolated_ms_per_full_step")
        line["step_seconds"] = [round(x, 3) for x in vals]
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# native
# ---------------------------------------------------------------------------
def run_native(args, w):
    import torch
    import torch.distributed as dist

    import block_discrete_diffusion_denoise_b200 as dgp
    import synth_inputs as si

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    # a dedicated stream: the step is captured into a CUDA graph, which the
    # legacy default stream does not allow
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    weights = si.model_weights(w, "cuda")
    torch.cuda.synchronize()
    cfg = dgp.config_from_shape(w.shape, max_batch=w.batch, max_seq=w.prefix + 2 * w.canvas,
                                canvas=w.canvas)
    ctx = dgp.Context(cfg, weights, stream=stream.cuda_stream)
    prefix = si.uniform_tokens(w, "prefix", w.batch, w.prefix, device="cuda")
    ctx.prefill(prefix)
    ctx.sync()
    B, C = w.batch, w.canvas
    cur = si.uniform_tokens(w, "canvas", B, C, device="cuda")
    nxt = torch.empty_like(cur)
    conf = torch.empty(B, C, dtype=torch.float32, device="cuda")
    settled = torch.empty(B, dtype=torch.int32, device="cuda")
    seed = w.sample_seed

    # experts actually hit per layer (one recorded step, outside the timing)
    ctx.debug_capture(True)
    ctx.denoise_step(cur, 0, seed, w.tau0, nxt, conf, settled)
    hits = []
    for l in range(w.shape.n_layers):
        e = torch.empty(B * C, w.shape.top_k, dtype=torch.int32, device="cuda")
        ctx.debug_experts(l, e)
        ctx.sync()
        hits.append(int(torch.unique(e).numel()))
    ctx.debug_capture(False)

    clocks = Clocks(local)  # sampling from before the warm-up on
    for s in range(args.warmup):
        ctx.denoise_step(cur, s, seed, si.tau_schedule(w, s), nxt, conf, settled)
        cur, nxt = nxt, cur
    ctx.sync()

    # ---- timed region: K steps (the step runs as one CUDA graph) ----
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    n0 = ctx.launch_count
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for s in range(args.steps):
        ctx.denoise_step(cur, s, seed, si.tau_schedule(w, s % w.steps), nxt, conf, settled)
        cur, nxt = nxt, cur
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    ms = ev0.elapsed_time(ev1) / args.steps
    clk = clocks.stop(t_wall0, t_wall1)
    launches = (ctx.launch_count - n0) // args.steps
    ctx.sync()
    ms = max_over_ranks(ms, world, "cuda")

    # ---- second timed region, K steps with launches issued one by one: a CUDA
    # event pair on the library stream around every fused expert GEMM launch
    # (events cannot be placed inside the graph of the first region) ----
    ctx.debug_profile(["experts"])
    barrier()
    for s in range(args.steps):
        ctx.denoise_step(cur, s, seed, si.tau_schedule(w, s % w.steps), nxt, conf, settled)
        cur, nxt = nxt, cur
    prof = ctx.debug_profile_read()
    ctx.debug_profile([])
    barrier()

    # ---- per-class breakdown (separate short pass, informational) ----
    ctx.debug_profile(dgp.PROF_CLASSES)
    for s in range(2):
        ctx.denoise_step(cur, s, seed, w.tau0, nxt, conf, settled)
        cur, nxt = nxt, cur
    breakdown = {k: round(v[0] / 2, 4) for k, v in ctx.debug_profile_read().items()}
    ctx.debug_profile([])

    # ---- end to end through the host-buffer entry point, from pinned host
    # memory (each call copies the canvas in, runs the step, copies canvas,
    # confidences and flags out and synchronises) ----
    hin = torch.empty((B, C), dtype=torch.int32, pin_memory=True)
    hin.copy_(cur)
    hout = torch.empty((B, C), dtype=torch.int32, pin_memory=True)
    hconf = torch.empty((B, C), dtype=torch.float32, pin_memory=True)
    hset = torch.empty(B, dtype=torch.int32, pin_memory=True)
    ctx.denoise_step_host(hin, 0, seed, w.tau0, hout, hconf, hset)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(args.steps):
        ctx.denoise_step_host(hin, s, seed, w.tau0, hout, hconf, hset)
        hin, hout = hout, hin
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, "cuda")
    barrier()

    hbm, tf_burst, tf_sus, src = peaks()
    by, fl, gu_bytes = step_cost(w, hits)
    gu_ms, gu_n = prof["experts"]
    gu_avg_ms = gu_ms / max(gu_n, 1)
    achieved = gu_bytes / (gu_avg_ms * 1e-3) / 1e9
    t_roof = max(by / (hbm * 1e9), fl / (tf_sus * 1e12))
    traffic = None
    tp = os.path.join(ROOT, "profiles", "expert_gemm_traffic.json")
    if os.path.exists(tp):
        try:
            rec = json.load(open(tp))
            src_hash = code_sha256(os.path.join(ROOT, "block_discrete_diffusion_denoise_b200", "csrc", "gemm.cuh"))
            if rec.get("gemm_cuh_code_sha256") == src_hash and rec.get("workload") == w.name:
                traffic = rec["bytes_per_launch"]
        except Exception:
            traffic = None
    value = replicas_value(world, B, C, ms)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: {w.description}", "global_batch": world * B,
                       "canvas": C, "prefix": w.prefix, "parallelism": f"replicas x{world}",
                       "l2": l2_note(by)},
            "roofline": {"bound": "hbm", "kernel": "fused expert GEMM gate/up + down (tcgen05, SwiGLU epilogue)",
                         "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": traffic, "peak_source": PEAK_NOTE[src],
                         "bytes_per_launch": gu_bytes, "launch_ms": gu_avg_ms, "launches": gu_n,
                         "launch_timing": "CUDA event pair around every launch of the kernel over a "
                                          "second K-step timed region with launches issued one by one"},
            "step_roofline": {"bytes": by, "flops": fl, "t_roof_ms": t_roof * 1e3,
                              "frac": t_roof * 1e3 / ms,
                              "peaks": f"{src}: HBM {hbm} GB/s, bf16 {tf_sus} TF/s sustained"},
            "experts_hit_per_layer": hits,
            "breakdown_ms_per_step": breakdown,
            "e2e": {"value": replicas_value(world, B, C, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": B * C * 4, "d2h_bytes_per_step": B * C * 8 + B * 4,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches * args.steps,
            "gpu_launches_per_step": launches,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            v, t, _, desc = OracleSample(w).run()
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": _cores(), "kind": "oracle",
                                    "sample": desc}
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        dist.destroy_process_group()


def run_batch_sweep(args, w):
    """Where the step turns from HBM-bound to tensor-bound as the batch grows
    (codemajin.net section 5.4: above about 32 concurrent requests the
    diffusion step loses its advantage to compute load).  One context sized
    for the largest batch; per batch B: prefill B sequences, warm up, time
    `steps` graph-replayed steps with CUDA events, and count the experts hit
    for the step's algorithmic bytes."""
    import torch

    import block_discrete_diffusion_denoise_b200 as dgp
    import synth_inputs as si

    batches = [int(b) for b in args.batch_sweep.split(",") if b]
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    weights = si.model_weights(w, "cuda")
    cfg = dgp.config_from_shape(w.shape, max_batch=max(batches), max_seq=w.prefix + 2 * w.canvas,
                                canvas=w.canvas)
    ctx = dgp.Context(cfg, weights, stream=stream.cuda_stream)
    hbm, tf_burst, tf_sus, src = peaks()
    rows = []
    for B in batches:
        wb = w.with_(batch=B)
        ctx.prefill(si.uniform_tokens(wb, "prefix", B, w.prefix, device="cuda"))
        cur = si.uniform_tokens(wb, "canvas", B, w.canvas, device="cuda")
        nxt = torch.empty_like(cur)
        conf = torch.empty(B, w.canvas, dtype=torch.float32, device="cuda")
        ctx.debug_capture(True)
        ctx.denoise_step(cur, 0, w.sample_seed, w.tau0, nxt, conf)
        hits = []
        for l in range(w.shape.n_layers):
            e = torch.empty(B * w.canvas, w.shape.top_k, dtype=torch.int32, device="cuda")
            ctx.debug_experts(l, e)
            ctx.sync()
            hits.append(int(torch.unique(e).numel()))
        ctx.debug_capture(False)
        for s in range(args.warmup):
            ctx.denoise_step(cur, s, w.sample_seed, w.tau0, nxt, conf)
            cur, nxt = nxt, cur
        ctx.sync()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(args.steps):
            ctx.denoise_step(cur, s, w.sample_seed, w.tau0, nxt, conf)
            cur, nxt = nxt, cur
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        by, fl, _ = step_cost(wb, hits)
        t_hbm, t_tc = by / (hbm * 1e9) * 1e3, fl / (tf_sus * 1e12) * 1e3
        rows.append({"batch": B, "ms_per_step": ms, "canvas_tok_s": B * w.canvas / (ms * 1e-3),
                     "bytes": by, "flops": fl, "t_hbm_ms": t_hbm, "t_tensor_ms": t_tc,
                     "bound": "hbm" if t_hbm >= t_tc else "tensor", "roofline_frac": max(t_hbm, t_tc) / ms,
                     "experts_hit_mean": sum(hits) / len(hits)})
        print(json.dumps(rows[-1]), file=sys.stderr, flush=True)
    ctx.close()
    print(json.dumps({"metric": "canvas tokens denoised/s vs batch", "workload": f"{w.name}: {w.description}",
                      "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
                      "peaks": f"{src}: HBM {hbm} GB/s, bf16 {tf_sus} TF/s sustained", "sweep": rows}),
          flush=True)


def main():
    args = parse()
    if args.timeline:
        # the timeline build of the library; chosen before the package is imported
        os.environ["DG_LIBRARY"] = os.path.join(ROOT, "block_discrete_diffusion_denoise_b200", "libdg_timeline.so")
    import synth_inputs as si
    w = si.workload(args.workload)
    if args.layers:
        w = w.with_layers(args.layers)
    if args.timeline:
        run_timeline(args, w)
    elif args.variants:
        run_variants(args, w)
    elif args.batch_sweep:
        run_batch_sweep(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_native(args, w)


if __name__ == "__main__":
    main()
