#!/usr/bin/env python
"""CSA decode benchmark: steps/s of (index score -> top-k -> sparse MQA
attention) over a stack of CSA layers, on synthetic inputs shaped like the
64K-context decode workload (21 CSA layers, batch 1, N = 16384 compressed
entries per layer, 64 heads, top-512, 128-row window, bf16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lidx|reference]
                    [--workload decode-64k|decode-128k-b32|decode-500k-b4|eval-window]

The eval-window workload times one tau-window of the selection evaluation
(64 queries x 21 layers x 32768 entries: native scores and top-512, golden
dense-attention probabilities, top-p 0.6, the 3-of-21 vote and window union,
the gate, overlap counts) in windows/s.

Prints one JSON line (rank 0).  With --gpus N > 1 under torchrun every rank
runs an independent replica of the workload on its own GPU (the path does not
shard); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import tempfile
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "CSA decode steps/s (score+top-k+sparse attn) at 64K; HBM GB/s vs peak"
UNIT = "steps/s"

WORKLOADS = {
    "decode-64k": synth.DECODE_64K,
    "decode-128k-b32": synth.DECODE_128K_B32,
    "decode-500k-b4": synth.DECODE_500K_FP8,
}

KEY_ROW_BYTES = {"f32": 512, "bf16": 256, "e4m3": 64 + 1 + 128}
KV_ROW_BYTES = {"f32": 2048, "bf16": 1024, "e4m3": 448 + 7 + 128}
Q_BYTES = {"f32": 4, "bf16": 2}


def algorithmic_bytes(spec) -> dict:
    """Inputs read once and outputs written once (intermediates excluded), per
    step, per layer, and per launch of each library call (which counts the
    intermediates it reads or writes: scores, ids)."""
    B, N, H, k = spec.B, spec.N, spec.H, spec.k
    keys = B * N * KEY_ROW_BYTES[spec.key_dtype]
    q_idx = B * H * 128 * Q_BYTES[spec.q_dtype]
    w = B * H * 4
    rows = B * k * KV_ROW_BYTES[spec.kv_dtype]
    swa = B * spec.swa * KV_ROW_BYTES[spec.kv_dtype]
    q_attn = B * H * 512 * Q_BYTES[spec.q_dtype]
    out = B * H * 512 * 4
    scores = B * N * 4
    ids = B * (k + 1) * 4
    layer = keys + q_idx + w + rows + swa + q_attn + out
    per_call = {
        "score": keys + q_idx + w + scores,
        "topk": scores + ids,
        "attn": ids + rows + swa + q_attn + out + B * H * 4,
    }
    return dict(layer=layer, step=layer * spec.layers, per_call=per_call)


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# source files of each library call's kernels
CALL_SOURCES = {
    "score": ("score_tc.cu", "score_cc.cu"),
    "topk": ("topk.cu",),
    "attn": ("attn.cu", "attn_tc.cu"),
    "golden": ("golden_tc.cu", "eval.cu"),
}
CALL_NAMES = {"score": "lidx_index_score", "topk": "lidx_topk_select", "attn": "lidx_sparse_attn_decode"}


def source_hash(call: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lightning_indexer_top_index_b200", "csrc")
    for f in CALL_SOURCES[call] + ("common.cuh", "kernels.cuh", "tc.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, call: str):
    """DRAM bytes per launch of `call` from the committed ncu summary, if it
    was taken on the current source of that call's kernels; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload, {}).get(call)
    if not d or d.get("source_hash") != source_hash(call):
        return None
    return d.get("dram_bytes_per_launch")


def init_group(world: int, device=None, backend: str = "nccl"):
    """The process group of a `world`-rank run (rank and rendezvous from the
    environment torchrun sets), or None for one rank.  Replicas exchange
    nothing on the data path: the group carries barriers and the timing
    reduction only."""
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    kw = {} if device is None else {"device_id": device}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput per second: the units every rank processed over
    the slowest rank's time per step."""
    return world * units_per_rank * 1e3 / ms


def max_over_ranks(x: float, dist, device=None) -> float:
    """The largest value over the ranks of the process group (the job's time
    is its slowest replica's); `x` itself without a process group."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"lidx_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ the arms
def oracle_layer_time(spec, layers) -> tuple:
    """Time the oracle (score, top-k, attention of every sequence) on the given
    layers' inputs; returns (seconds, layers done)."""
    import oracle
    t0 = time.perf_counter()
    for inp in layers:
        for b in range(spec.B):
            N = spec.N
            s = oracle.index_score(inp["q_idx"][b].reshape(1, 1, spec.H, 128), inp["w"][b],
                                   inp["keys"].slice(b * N, (b + 1) * N), 1, 1, spec.H, N)
            ids, n, _ = oracle.topk(s[0, 0], spec.k)
            oracle.attn(inp["q_attn"][b], inp["kv"].slice(b * N, (b + 1) * N), N, ids[:n],
                        swa=inp["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=spec.swa, scale=spec.scale)
    return time.perf_counter() - t0, len(layers)


def run_reference(args, spec, cfg):
    """The oracle arm: each step is one layer of the workload on the host."""
    layers = [synth.decode_layer(spec, l % spec.layers) for l in range(min(spec.layers, 2))]
    for i in range(args.warmup):
        oracle_layer_time(spec, [layers[i % len(layers)]])
    t, n = 0.0, 0
    for i in range(args.steps):
        dt, dn = oracle_layer_time(spec, [layers[i % len(layers)]])
        t += dt
        n += dn
    step_s = t / n * spec.layers
    v = 1.0 / step_s
    sample = f"{n} single-layer samples of the {spec.layers}-layer step; steps/s = 1/(mean layer time x {spec.layers})"
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg, "impl": "reference",
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def make_replica_steps(spec, layers_inp, R, device):
    import torch
    import lightning_indexer_top_index_b200 as L
    from lightning_indexer_top_index_b200.decode import DecodeStep, LayerCache

    base = []
    for inp in layers_inp:
        base.append(LayerCache(
            L.DeviceKV.from_arrays(spec.key_dtype, 128, inp["keys"].data, inp["keys"].scale, inp["keys"].rope,
                                   batch_rows=spec.N, device=device),
            L.DeviceKV.from_arrays(spec.kv_dtype, 512, inp["kv"].data, inp["kv"].scale, inp["kv"].rope,
                                   batch_rows=spec.N, device=device),
            L.DeviceKV.from_arrays(spec.kv_dtype, 512, inp["swa"].data, inp["swa"].scale, inp["swa"].rope,
                                   batch_rows=spec.swa, device=device)))

    def clone(kv):
        return L.DeviceKV(kv.dtype, kv.dim, kv.data.clone(), None if kv.scale is None else kv.scale.clone(),
                          None if kv.rope is None else kv.rope.clone(), kv.batch_rows)

    qdt = torch.bfloat16 if spec.q_dtype == "bf16" else torch.float32
    steps = []
    for r in range(R):
        caches = base if r == 0 else [LayerCache(clone(c.keys), clone(c.kv), clone(c.swa)) for c in base]
        steps.append(DecodeStep(caches, spec.B, spec.H, spec.N, spec.k, spec.swa, spec.scale, q_dtype=qdt,
                                device=device))
    return steps


def host_queries(spec, layers_inp):
    """Per-step inputs on the host: q_idx [L][B][1][H][128], w [L][B][1][H], q_attn [L][B][H][512]."""
    import torch

    def t(x, dt):
        a = torch.from_numpy(np.ascontiguousarray(x))
        return a.view(torch.int16).view(torch.bfloat16) if dt == "bf16" else a

    q_idx = torch.stack([t(i["q_idx"], spec.q_dtype) for i in layers_inp]).reshape(spec.layers, spec.B, 1, spec.H, 128)
    w = torch.stack([torch.from_numpy(i["w"]) for i in layers_inp]).reshape(spec.layers, spec.B, 1, spec.H)
    q_attn = torch.stack([t(i["q_attn"], spec.q_dtype) for i in layers_inp])
    return q_idx, w, q_attn


def run_lidx(args, spec, cfg, rank, world, local_rank):
    import torch
    import lightning_indexer_top_index_b200 as L  # noqa: F401

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_group(world, device)

    layers_inp = [synth.decode_layer(spec, l) for l in range(spec.layers)]
    ab = algorithmic_bytes(spec)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    R = max(2, math.ceil(4 * l2 / ab["step"]))
    steps = make_replica_steps(spec, layers_inp, R, device)
    q_idx_h, w_h, q_attn_h = host_queries(spec, layers_inp)
    for s in steps:
        s.set_inputs(q_idx_h.to(device), w_h.to(device), q_attn_h.to(device))
        s.capture()
    torch.cuda.synchronize()

    # ---- device-timed steps (inputs resident)
    for i in range(args.warmup):
        steps[i % R].replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        steps[i % R].replay()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, device)
    if dist:
        dist.barrier()

    # ---- live per-call timing: the same step with external events around
    # every library call (which also shows each call's own launch latency)
    inst = steps[0]
    calls = ("score", "topk", "attn")
    events = [{c: (torch.cuda.Event(enable_timing=True, external=True),
                   torch.cuda.Event(enable_timing=True, external=True)) for c in calls} for _ in range(spec.layers)]
    g_inst = inst.capture(events)
    durs = {c: [] for c in calls}
    for i in range(max(3, min(args.steps, 20))):
        for r in range(1, R):
            steps[r].replay()  # evict the instrumented replica's caches from L2 between its replays
        g_inst.replay()
        torch.cuda.synchronize()
        for ev in events:
            for c in calls:
                durs[c].append(ev[c][0].elapsed_time(ev[c][1]))
    call_ms = {c: statistics.mean(durs[c]) for c in calls}
    del g_inst

    # ---- end to end: pinned host queries in, attention outputs back, every step
    q_idx_p, w_p, q_attn_p = q_idx_h.pin_memory(), w_h.pin_memory(), q_attn_h.pin_memory()
    out_p = torch.empty(steps[0].out.shape, dtype=torch.float32).pin_memory()
    for i in range(args.warmup):
        s = steps[i % R]
        s.set_inputs(q_idx_p, w_p, q_attn_p)
        s.replay()
        out_p.copy_(s.out, non_blocking=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for i in range(args.steps):
        s = steps[i % R]
        s.set_inputs(q_idx_p, w_p, q_attn_p)
        s.replay()
        out_p.copy_(s.out, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps, dist, device)
    h2d = sum(x.numel() * x.element_size() for x in (q_idx_p, w_p, q_attn_p))
    d2h = out_p.numel() * out_p.element_size()

    if rank == 0:
        pk = peaks()
        dom = max(calls, key=lambda c: call_ms[c])
        achieved = ab["per_call"][dom] / (call_ms[dom] * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": job_rate(1, world, ms), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if spec.key_dtype == "bf16" else spec.key_dtype,
            "data": "synthetic", "config": cfg,
            "hbm_gbs_step": ab["step"] / (ms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": profiled_traffic(args.workload, dom),
                         "kernel": CALL_NAMES[dom], "peak_source": pk["source"],
                         "bytes_per_launch": ab["per_call"][dom], "avg_launch_us": call_ms[dom] * 1e3},
            "calls": {CALL_NAMES[c]: {"avg_launch_us": call_ms[c] * 1e3, "bytes_per_launch": ab["per_call"][c],
                                      "gbs": ab["per_call"][c] / (call_ms[c] * 1e-3) / 1e9} for c in calls},
            "e2e": {"value": job_rate(1, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * steps[0].kernel_launches(),
            "clocks": clk,
        }
        if world == 1:
            sample_layers = layers_inp[:2]
            t, n = oracle_layer_time(spec, sample_layers)
            v = 1.0 / (t / n * spec.layers)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                    "sample": f"{n} of the {spec.layers} layers of one step on the host, "
                                              f"single thread; scaled by {spec.layers}/{n}"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------- eval window
EVAL_METRIC = "selection-eval windows/s (64 queries x 21 layers x 32K entries; golden TFLOP/s vs peak)"
EVAL_STAGES = ("score", "topk", "golden", "topp", "gold_topk", "vote", "gate", "overlap")


def eval_inputs(spec):
    layers = [synth.eval_layer(spec, l) for l in range(spec.L)]
    return layers, synth.eval_gate(spec)


def oracle_eval_sample(spec, layers, gate):
    """The oracle on a bounded sample of a window: golden probabilities of one
    query of one layer (all 64 heads, all N entries), its top-p set and top-k;
    returns (seconds, windows the sample stands for)."""
    import oracle
    x = layers[0]
    t0 = time.perf_counter()
    p = oracle.golden(x["qa"][:1], x["kv"], 1, spec.H, spec.N, spec.scale)
    oracle.topp(p[0])
    oracle.topk(p[0], spec.k)
    dt = time.perf_counter() - t0
    return dt, 1.0 / (spec.L * spec.T)


def run_eval(args, cfg, rank, world, local_rank, reference=False):
    spec = synth.EVAL_WINDOW
    if reference:
        layers, gate = eval_inputs(synth.scaled(spec, L=1))
        for _ in range(args.warmup):
            oracle_eval_sample(spec, layers, gate)
        t, w = 0.0, 0.0
        for _ in range(args.steps):
            dt, dw = oracle_eval_sample(spec, layers, gate)
            t, w = t + dt, w + dw
        v = w / t
        sample = ("golden probabilities, top-p and top-k of one query of one layer per step "
                  f"(1/{spec.L * spec.T} of a window), single thread")
        print(json.dumps({"metric": EVAL_METRIC, "value": v, "unit": "windows/s", "n_gpus": args.gpus,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / v,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": cfg, "impl": "reference",
                          "cpu_baseline": {"value": v, "unit": "windows/s", "cores": 1, "kind": "oracle",
                                           "sample": sample},
                          "e2e": {"value": v, "unit": "windows/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return
    import torch
    import lightning_indexer_top_index_b200 as L
    from lightning_indexer_top_index_b200.evalwin import EvalWindow

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_group(world, device)
    layers, gate = eval_inputs(spec)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16)

    keys = [L.DeviceKV.from_arrays("bf16", 128, x["keys"].data, batch_rows=spec.N, device=device) for x in layers]
    kv_all = L.DeviceKV.from_arrays("bf16", 512, np.concatenate([x["kv"].data for x in layers]),
                                    batch_rows=spec.N, device=device)
    q_idx_h = torch.stack([bf(x["q_idx"]) for x in layers])
    w_h = torch.stack([torch.from_numpy(x["w"]) for x in layers])
    qa_h = torch.stack([bf(x["qa"]) for x in layers])
    gq_h, gu_h = bf(gate["g"]), torch.from_numpy(gate["u"])
    q_idx, w, qa, gq, gu = (t.to(device) for t in (q_idx_h, w_h, qa_h, gq_h, gu_h))
    win = EvalWindow(keys, kv_all, q_idx, w, qa, gq, gu, spec.gate_layers, spec.N, spec.k,
                     (spec.top_p_num, spec.top_p_den), spec.min_votes, spec.scale)
    for _ in range(args.warmup):
        win.enqueue()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        win.enqueue()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, device)
    # per-stage times (events between stages)
    ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in EVAL_STAGES}
    stage_ms = {n: 0.0 for n in EVAL_STAGES}
    reps = max(1, min(args.steps, 5))
    for _ in range(reps):
        win.enqueue(events=ev)
        torch.cuda.synchronize()
        for n in EVAL_STAGES:
            stage_ms[n] += ev[n][0].elapsed_time(ev[n][1]) / reps
    # end to end: the window's queries in from pinned host memory, counts back
    pins = [t.pin_memory() for t in (q_idx_h, w_h, qa_h, gq_h, gu_h)]
    outs = [torch.empty(c.shape, dtype=c.dtype).pin_memory()
            for c in (win.counts_nat_gold, win.counts_nat_f, win.counts_g_f)]
    dsts = (win.q_idx, win.w, win.qa, gq, gu)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        for d, hsrc in zip(dsts, pins):
            d.copy_(hsrc, non_blocking=True)
        win.enqueue()
        for o, c in zip(outs, (win.counts_nat_gold, win.counts_nat_f, win.counts_g_f)):
            o.copy_(c, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps, dist, device)
    if rank == 0:
        pk = peaks()
        gflops = win.golden_flops()
        achieved = gflops / (stage_ms["golden"] * 1e-3) / 1e12
        peak = pk["bf16_tflops_sustained"]
        line = {
            "metric": EVAL_METRIC, "value": job_rate(1, world, ms), "unit": "windows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": profiled_traffic("eval-window", "golden"),
                         "kernel": "lidx_selection_eval (golden)",
                         "peak_source": pk["source"] + " bf16, sustained", "flops_per_launch": gflops,
                         "avg_launch_us": stage_ms["golden"] * 1e3},
            "stages_ms": stage_ms,
            "score_tflops": win.score_flops() / (stage_ms["score"] * 1e-3) / 1e12,
            "e2e": {"value": job_rate(1, world, e2e_ms), "unit": "windows/s",
                    "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pins),
                    "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs)},
            "gpu_launches": args.steps * win.kernel_launches(),
            "clocks": clk,
        }
        if world == 1:
            dt, dw = oracle_eval_sample(spec, layers, gate)
            line["cpu_baseline"] = {"value": dw / dt, "unit": "windows/s", "cores": 1, "kind": "oracle",
                                    "sample": "golden probabilities, top-p and top-k of one query of one "
                                              f"layer (1/{spec.L * spec.T} of a window), single thread"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lidx", choices=["lidx", "reference"])
    ap.add_argument("--workload", default="decode-64k", choices=sorted(WORKLOADS) + ["eval-window"])
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload == "eval-window":
        e = synth.EVAL_WINDOW
        cfg = {"workload": e.name, "layers": e.L, "queries": e.T, "heads": e.H, "entries": e.N, "top_k": e.k,
               "top_p": f"{e.top_p_num}/{e.top_p_den}", "min_votes": e.min_votes,
               "gate_layers": list(e.gate_layers), "l2": "inputs larger than L2 (704 MB of attention rows)",
               "parallelism": f"replicas x{world}"}
        if args.impl == "reference":
            if rank == 0:
                run_eval(args, cfg, rank, world, local_rank, reference=True)
            return
        run_eval(args, cfg, rank, world, local_rank)
        return
    spec = WORKLOADS[args.workload]
    ab = algorithmic_bytes(spec)
    cfg = {"workload": spec.name, "layers": spec.layers, "batch": spec.B, "entries": spec.N, "heads": spec.H,
           "top_k": spec.k, "swa": spec.swa, "key_format": spec.key_dtype, "kv_format": spec.kv_dtype,
           "algorithmic_bytes_per_step": ab["step"],
           "l2": "inputs larger than L2: rotating cache replicas, >= 4x L2 of step bytes",
           "parallelism": f"replicas x{world}"}
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, spec, cfg)
        return
    run_lidx(args, spec, cfg, rank, world, local_rank)


if __name__ == "__main__":
    main()
