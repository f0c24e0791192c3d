#!/usr/bin/env python
"""CSA decode benchmark: steps/s of (index score -> top-k -> sparse MQA
attention) over a stack of CSA layers, on synthetic inputs shaped like the
64K-context decode workload (21 CSA layers, batch 1, N = 16384 compressed
entries per layer, 64 heads, top-512, 128-row window, bf16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lidx|reference]
                    [--workload decode-64k|decode-128k-b32|decode-500k-b4|eval-window|decode-64k-model]
                    [--repeats R] [--only]

The default line is the 64K decode; under the key "workloads" it also carries
the same measurement (value, ms_per_step, roofline, e2e, clocks, launches,
oracle baseline) for the other target workloads:
  decode-500k-b4    one layer of 4 sequences x 125000 entries, E4M3 keys and
                    rows, top-1024
  decode-128k-b32   one layer of 32 sequences x 32768 entries, planted rows
  eval-window       one tau-window of the selection evaluation (64 queries x
                    21 layers x 32768 entries) in windows/s
  decode-64k-model  one token through the 43 attention layers of the hybrid
                    schedule (2 window-only, 21 CSA, 20 HCA)
--only skips them.  Each timing is the median of R (>= 5) repeats of K steps.

Prints one JSON line (rank 0).  With --gpus N > 1 under torchrun every rank
runs an independent replica of the workload on its own GPU (the path does not
shard); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import concurrent.futures
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
MODEL = "decode-64k-model"
EVAL = "eval-window"
SIDE_WORKLOADS = ("decode-500k-b4", "decode-128k-b32", EVAL, MODEL)

KEY_ROW_BYTES = {"f32": 512, "bf16": 256, "e4m3": 64 + 1 + 128}
KV_ROW_BYTES = {"f32": 2048, "bf16": 1024, "e4m3": 448 + 7 + 128}
Q_BYTES = {"f32": 4, "bf16": 2}


def algorithmic_bytes(spec) -> dict:
    """Inputs read once and outputs written once (intermediates excluded), per
    step, per layer, and per launch of each library call (a separate call
    counts the intermediates it reads or writes: scores, ids; the one-launch
    layer keeps them inside)."""
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
        "layer": layer + B * H * 4,
    }
    return dict(layer=layer, step=layer * spec.layers, per_call=per_call)


def model_bytes(spec) -> dict:
    """Algorithmic bytes of one token through the hybrid schedule: 21 CSA
    layers as above, 20 HCA layers (every one of the N/32 rows, the window,
    the query and the output) and 2 window-only layers."""
    csa = algorithmic_bytes(spec)["layer"]
    row = KV_ROW_BYTES[spec.kv_dtype]
    q_out = spec.B * spec.H * 512 * (Q_BYTES[spec.q_dtype] + 4)
    win = spec.B * spec.swa * row
    hca = spec.B * (spec.N // 32) * row + win + q_out
    swa = win + q_out
    return dict(csa=csa, hca=hca, swa=swa, step=21 * csa + 20 * hca + 2 * swa)


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
    "attn": ("attn.cu", "attn_tc.cu", "attn_wide.cu"),
    "layer": ("decode_fused.cu",),
    "golden": ("golden_tc.cu", "eval.cu"),
}
CALL_NAMES = {"score": "lidx_index_score", "topk": "lidx_topk_select", "attn": "lidx_sparse_attn_decode",
              "layer": "lidx_decode_layer"}


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


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


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
                                          "-i", str(self.gpu), "-lms", "20"], stdout=self.f,
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


# ------------------------------------------------------------ oracle timing
def run_tasks(tasks, threads: int) -> float:
    """Wall time of running the callables on `threads` host threads (the
    oracle is C called through ctypes, which releases the GIL)."""
    t0 = time.perf_counter()
    if threads <= 1:
        for t in tasks:
            t()
    else:
        with concurrent.futures.ThreadPoolExecutor(threads) as ex:
            for f in [ex.submit(t) for t in tasks]:
                f.result()
    return time.perf_counter() - t0


def oracle_decode_tasks(spec, layers_inp):
    """One task per (layer, sequence): the oracle's score, top-k and attention."""
    import oracle

    def task(inp, b):
        def run():
            N = spec.N
            s = oracle.index_score(inp["q_idx"][b].reshape(1, 1, spec.H, 128), inp["w"][b],
                                   inp["keys"].slice(b * N, (b + 1) * N), 1, 1, spec.H, N)
            ids, n, _ = oracle.topk(s[0, 0], spec.k)
            oracle.attn(inp["q_attn"][b], inp["kv"].slice(b * N, (b + 1) * N), N, ids[:n],
                        swa=inp["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=spec.swa, scale=spec.scale)
        return run

    return [task(inp, b) for inp in layers_inp for b in range(spec.B)]


def cpu_baseline_decode(spec, layers_inp, budget_s=15.0) -> dict:
    """The oracle on the host: whole steps on every core (one task per layer
    and sequence), plus a single-thread sample of one task scaled to a step."""
    cores = host_cores()
    tasks = oracle_decode_tasks(spec, layers_inp)
    t1 = run_tasks(tasks[:1], 1)
    single = 1.0 / (t1 * len(tasks))
    est = t1 * len(tasks) / min(cores, len(tasks))
    n = max(1, min(5, int(budget_s / max(est, 1e-3))))
    t = sum(run_tasks(tasks, cores) for _ in range(n))
    v = n / t
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} whole step(s) of {len(tasks)} (layer, sequence) tasks on {cores} host threads",
            "single_thread_value": single,
            "single_thread_sample": f"1 of the {len(tasks)} tasks on one thread, scaled to a step"}


# -------------------------------------------------------------- GPU timing
def timed_loop(fn, steps: int, repeats: int, dist, device, between=None, begin=None, end=None) -> tuple:
    """Median over `repeats` of the device time of `steps` calls of fn()
    (CUDA events, synchronised on both sides, after a barrier); returns
    (ms per step: the median, max over ranks; every repeat's ms).  begin()
    and end() run right after the first and right before the last event (on
    the current stream), e.g. to order a side stream inside the region."""
    import torch
    per = []
    for _ in range(repeats):
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if begin:
            begin()
        for i in range(steps):
            fn(i)
        if end:
            end()
        e1.record()
        torch.cuda.synchronize()
        per.append(e0.elapsed_time(e1) / steps)
        if between:
            between()
    ms = max_over_ranks(statistics.median(per), dist, device)
    return ms, per


def pipelined_e2e(steps, h2d, d2h):
    """End-to-end steps over the rotating replicas with the copies on two side
    streams, one per direction (PCIe carries both at once): step i copies its
    inputs into replica i % R (h2d(step)), replays it, and copies its result
    back (d2h(step, r)); the copy of step i+1's inputs and the copy of step
    i's result both overlap the steps around them.  Events keep a replica's
    inputs and outputs from being overwritten while in use.  Returns
    (step(i), begin(), end()): begin orders the side streams after the
    region's start, end makes the current stream wait for the last copies."""
    import torch
    R = len(steps)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(R)]
    used = [torch.cuda.Event() for _ in range(R)]     # the replica's step has read its inputs
    d2h_done = [torch.cuda.Event() for _ in range(R)]
    state = {"next": 0}

    def copy_in(i):
        r = i % R
        with torch.cuda.stream(up):
            up.wait_event(used[r])
            h2d(steps[r])
            h2d_done[r].record(up)

    def step(i):
        main = torch.cuda.current_stream()
        r = i % R
        if state["next"] <= i:  # this step's inputs not yet on their way
            copy_in(i)
        main.wait_event(h2d_done[r])
        main.wait_event(d2h_done[r])
        steps[r].replay()
        used[r].record(main)
        copy_in(i + 1)
        state["next"] = i + 2
        with torch.cuda.stream(down):
            down.wait_event(used[r])
            d2h(steps[r], r)
            d2h_done[r].record(down)

    def begin():
        up.wait_stream(torch.cuda.current_stream())
        down.wait_stream(torch.cuda.current_stream())
        state["next"] = 0

    def end():
        torch.cuda.current_stream().wait_stream(up)
        torch.cuda.current_stream().wait_stream(down)

    return step, begin, end


def make_caches(spec, layers_inp, device):
    import lightning_indexer_top_index_b200 as L
    from lightning_indexer_top_index_b200.decode import LayerCache

    def dk(k, rows):
        return L.DeviceKV.from_arrays(k.dtype, k.dim, k.data, k.scale, k.rope, batch_rows=rows, device=device)

    return [LayerCache(dk(x["keys"], spec.N), dk(x["kv"], spec.N), dk(x["swa"], spec.swa)) for x in layers_inp]


def clone_kv(kv):
    import lightning_indexer_top_index_b200 as L
    return L.DeviceKV(kv.dtype, kv.dim, kv.data.clone(), None if kv.scale is None else kv.scale.clone(),
                      None if kv.rope is None else kv.rope.clone(), kv.batch_rows)


LAYER_FORMS = {"auto": None, "fused": True, "calls": False}


def make_replica_steps(spec, layers_inp, R, device, fused=None):
    """R DecodeSteps over copies of the same caches (the bench rotates them).
    fused: None lets DecodeStep choose the layer form, True / False force it."""
    import torch
    from lightning_indexer_top_index_b200.decode import DecodeStep, LayerCache
    base = make_caches(spec, layers_inp, device)
    qdt = torch.bfloat16 if spec.q_dtype == "bf16" else torch.float32
    steps = []
    for r in range(R):
        caches = base if r == 0 else [LayerCache(clone_kv(c.keys), clone_kv(c.kv), clone_kv(c.swa)) for c in base]
        steps.append(DecodeStep(caches, spec.B, spec.H, spec.N, spec.k, spec.swa, spec.scale, q_dtype=qdt,
                                device=device, fused=fused))
    return steps


def bf16_tensor(x, dt):
    import torch
    a = torch.from_numpy(np.ascontiguousarray(x))
    return a.view(torch.int16).view(torch.bfloat16) if dt == "bf16" else a


def host_queries(spec, layers_inp):
    """Per-step inputs on the host: q_idx [L][B][1][H][128], w [L][B][1][H], q_attn [L][B][H][512]."""
    import torch
    q_idx = torch.stack([bf16_tensor(i["q_idx"], spec.q_dtype) for i in layers_inp]).reshape(
        len(layers_inp), spec.B, 1, spec.H, 128)
    w = torch.stack([torch.from_numpy(i["w"]) for i in layers_inp]).reshape(len(layers_inp), spec.B, 1, spec.H)
    q_attn = torch.stack([bf16_tensor(i["q_attn"], spec.q_dtype) for i in layers_inp])
    return q_idx, w, q_attn


def measure_decode(args, name, spec, world, dist, device, local_rank, rank, want_cpu, form=None) -> dict:
    """The stack of CSA layers: R cache replicas rotated so each step reads
    from HBM (R x step bytes >= 4 x L2), captured as CUDA graphs."""
    import torch
    import lightning_indexer_top_index_b200 as L

    layers_inp = [synth.decode_layer(spec, l) for l in range(spec.layers)]
    ab = algorithmic_bytes(spec)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    R = max(2, math.ceil(4 * l2 / ab["step"]))
    steps = make_replica_steps(spec, layers_inp, R, device, fused=form)
    q_idx_h, w_h, q_attn_h = host_queries(spec, layers_inp)
    for s in steps:
        s.set_inputs(q_idx_h.to(device), w_h.to(device), q_attn_h.to(device))
        s.capture()
    torch.cuda.synchronize()
    for i in range(args.warmup):
        steps[i % R].replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    ms, per = timed_loop(lambda i: steps[i % R].replay(), args.steps, args.repeats, dist, device)
    clk = clocks.stop()

    # live per-call timing: the same step with external events around every
    # library call (it also shows each call's own launch latency)
    inst = steps[0]
    calls = ("layer",) if inst.fused else ("score", "topk", "attn")
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

    # end to end: pinned host queries in, attention outputs back, every step
    q_idx_p, w_p, q_attn_p = q_idx_h.pin_memory(), w_h.pin_memory(), q_attn_h.pin_memory()
    out_ps = [torch.empty(steps[0].out.shape, dtype=torch.float32).pin_memory() for _ in range(R)]
    e2e_step, e2e_begin, e2e_end = pipelined_e2e(steps, lambda s: s.set_inputs(q_idx_p, w_p, q_attn_p),
                                                 lambda s, r: out_ps[r].copy_(s.out, non_blocking=True))
    e2e_begin()
    for i in range(args.warmup):
        e2e_step(i)
    e2e_end()
    e2e_ms, _ = timed_loop(e2e_step, args.steps, args.repeats, dist, device, begin=e2e_begin, end=e2e_end)
    h2d = sum(x.numel() * x.element_size() for x in (q_idx_p, w_p, q_attn_p))
    d2h = out_ps[0].numel() * out_ps[0].element_size()
    status = 0
    for s in steps:
        for ws in s.workspaces():
            status |= L.read_device_status(ws)

    pk = peaks()
    dom = max(calls, key=lambda c: call_ms[c])
    achieved = ab["per_call"][dom] / (call_ms[dom] * 1e-3) / 1e9
    res = {
        "metric": METRIC if name == "decode-64k" else f"{spec.name} steps/s (one step = {spec.layers} layer(s) of "
                                                      f"{spec.B} sequence(s)); HBM GB/s vs peak",
        "value": job_rate(1, world, ms), "unit": UNIT, "ms_per_step": ms,
        "ms_per_step_repeats": per,
        "dtype": "bf16" if spec.key_dtype == "bf16" else spec.key_dtype,
        "config": {"workload": spec.name, "layers": spec.layers, "batch": spec.B, "entries": spec.N,
                   "heads": spec.H, "top_k": spec.k, "swa": spec.swa, "key_format": spec.key_dtype,
                   "kv_format": spec.kv_dtype, "algorithmic_bytes_per_step": ab["step"],
                   "layer_form": "one launch per layer" if inst.fused else "three calls per layer",
                   "l2": f"inputs larger than L2: {R} rotating cache replicas, >= 4x L2 of step bytes",
                   "parallelism": f"replicas x{world}"},
        "hbm_gbs_step": ab["step"] / (ms * 1e-3) / 1e9,
        "hbm_frac_step": ab["step"] / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": profiled_traffic(name, dom),
                     "kernel": CALL_NAMES[dom], "peak_source": pk["source"] + " (burst copy)",
                     "bytes_per_launch": ab["per_call"][dom], "avg_launch_us": call_ms[dom] * 1e3},
        "calls": {CALL_NAMES[c]: {"avg_launch_us": call_ms[c] * 1e3, "bytes_per_launch": ab["per_call"][c],
                                  "gbs": ab["per_call"][c] / (call_ms[c] * 1e-3) / 1e9} for c in calls},
        "e2e": {"value": job_rate(1, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * args.repeats * steps[0].kernel_launches(),
        "gpu_launches_per_step": steps[0].kernel_launches(),
        "device_status": status,
        "clocks": clk,
    }
    if clk:
        res["clocks"]["ms_x_median_mhz"] = ms * clk["sm_mhz"]
    if want_cpu and rank == 0 and world == 1:
        res["cpu_baseline"] = cpu_baseline_decode(spec, layers_inp)
    del steps
    torch.cuda.empty_cache()
    return res


def decode_forms(args, name, spec, world, dist, device, local_rank, rank, want_cpu) -> dict:
    """--layer-form auto: where the one-launch layer covers the shape, time
    both layer forms and report the faster (both values under layer_forms)."""
    import lightning_indexer_top_index_b200 as L
    if args.layer_form != "auto":
        return measure_decode(args, name, spec, world, dist, device, local_rank, rank, want_cpu,
                              form=LAYER_FORMS[args.layer_form])
    try:
        fused = measure_decode(args, name, spec, world, dist, device, local_rank, rank, False, form=True)
    except L.LidxError as e:
        if e.status != L.ERR_UNSUPPORTED:
            raise
        return measure_decode(args, name, spec, world, dist, device, local_rank, rank, want_cpu, form=False)
    calls = measure_decode(args, name, spec, world, dist, device, local_rank, rank, want_cpu, form=False)
    best = dict(fused if fused["value"] > calls["value"] else calls)
    if "cpu_baseline" in calls:
        best["cpu_baseline"] = calls["cpu_baseline"]
    best["layer_forms"] = {r["config"]["layer_form"]: {"value": r["value"], "ms_per_step": r["ms_per_step"],
                                                        "e2e": r["e2e"]["value"], "gpu_launches_per_step":
                                                        r["gpu_launches_per_step"]} for r in (fused, calls)}
    return best


def measure_model(args, world, dist, device, local_rank, rank, want_cpu) -> dict:
    """One decode token through the 43 attention layers of the hybrid schedule
    at 64K (architecture post, section (A))."""
    import torch
    import lightning_indexer_top_index_b200 as L
    from lightning_indexer_top_index_b200.decode import LayerCache, ModelStep, model_schedule

    spec = synth.DECODE_64K
    kinds = model_schedule()
    xs = [synth.model_layer(spec, l) for l in range(len(kinds))]
    mb = model_bytes(spec)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    R = max(2, math.ceil(4 * l2 / mb["step"]))

    def dk(k, rows):
        return L.DeviceKV.from_arrays(k.dtype, k.dim, k.data, k.scale, k.rope, batch_rows=rows, device=device)

    n_hca = next(x["N"] for x in xs if x["kind"] == "hca")
    cx = [x for x in xs if x["kind"] == "csa"]
    q_idx_h = torch.stack([bf16_tensor(x["q_idx"], "bf16") for x in cx]).reshape(len(cx), 1, 1, spec.H, 128)
    w_h = torch.stack([torch.from_numpy(x["w"]) for x in cx]).reshape(len(cx), 1, 1, spec.H)
    qa_h = torch.stack([bf16_tensor(x["q_attn"], "bf16") for x in xs])
    steps = []
    for r in range(R):
        csa = [LayerCache(dk(x["keys"], spec.N), dk(x["kv"], spec.N), dk(x["swa"], spec.swa)) for x in cx]
        hca = [(dk(x["kv"], n_hca), dk(x["swa"], spec.swa)) for x in xs if x["kind"] == "hca"]
        swa = [dk(x["swa"], spec.swa) for x in xs if x["kind"] == "swa"]
        st = ModelStep(csa, hca, swa, spec.B, spec.H, spec.N, n_hca, spec.k, spec.swa, spec.scale, device=device)
        st.set_inputs(q_idx_h.to(device), w_h.to(device), qa_h.to(device))
        st.capture()
        steps.append(st)
    for i in range(args.warmup):
        steps[i % R].replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    ms, per = timed_loop(lambda i: steps[i % R].replay(), args.steps, args.repeats, dist, device)
    clk = clocks.stop()
    pins = [t.pin_memory() for t in (q_idx_h, w_h, qa_h)]
    out_ps = [torch.empty(steps[0].out.shape, dtype=torch.float32).pin_memory() for _ in range(R)]
    csa_ps = [torch.empty(steps[0].csa.out.shape, dtype=torch.float32).pin_memory() for _ in range(R)]
    out_p = out_ps[0]

    def d2h(s, r):  # the window-only and HCA layers' outputs, and the CSA layers'
        out_ps[r].copy_(s.out, non_blocking=True)
        csa_ps[r].copy_(s.csa.out, non_blocking=True)

    e2e_step, e2e_begin, e2e_end = pipelined_e2e(steps, lambda s: s.set_inputs(*pins), d2h)
    e2e_begin()
    for i in range(args.warmup):
        e2e_step(i)
    e2e_end()
    e2e_ms, _ = timed_loop(e2e_step, args.steps, args.repeats, dist, device, begin=e2e_begin, end=e2e_end)
    status = 0
    for s in steps:
        for ws in s.workspaces():
            status |= L.read_device_status(ws)
    pk = peaks()
    gbs = mb["step"] / (ms * 1e-3) / 1e9
    res = {
        "metric": "decode steps/s through the 43 attention layers of the hybrid schedule at 64K "
                  "(2 window-only, 21 CSA, 20 HCA); HBM GB/s vs peak",
        "value": job_rate(1, world, ms), "unit": UNIT, "ms_per_step": ms, "ms_per_step_repeats": per,
        "dtype": "bf16",
        "config": {"workload": MODEL, "layers": {"swa_only": 2, "csa": 21, "hca": 20}, "batch": 1,
                   "csa_entries": spec.N, "hca_entries": n_hca, "heads": spec.H, "top_k": spec.k, "swa": spec.swa,
                   "algorithmic_bytes_per_step": mb["step"],
                   "l2": f"inputs larger than L2: {R} rotating replicas, >= 4x L2 of step bytes",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / pk["hbm_gbs"], "traffic": None, "kernel": "whole step (65 launches)",
                     "peak_source": pk["source"] + " (burst copy)", "bytes_per_launch": mb["step"],
                     "avg_launch_us": ms * 1e3},
        "e2e": {"value": job_rate(1, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pins),
                "d2h_bytes_per_step": out_p.numel() * out_p.element_size() + steps[0].csa.out.numel() * 4},
        "gpu_launches": args.steps * args.repeats * steps[0].kernel_launches(),
        "gpu_launches_per_step": steps[0].kernel_launches(),
        "device_status": status,
        "clocks": clk,
    }
    if want_cpu and rank == 0 and world == 1:
        import oracle
        cores = host_cores()
        tasks = oracle_decode_tasks(spec, cx)
        for x in xs:
            if x["kind"] == "hca":
                tasks.append(lambda x=x: oracle.attn(x["q_attn"][0], x["kv"], x["N"], np.arange(x["N"], dtype=np.int32),
                                                     swa=x["swa"], swa_len=spec.swa, scale=spec.scale))
            elif x["kind"] == "swa":
                tasks.append(lambda x=x: oracle.attn(x["q_attn"][0], x["swa"], 1, np.zeros(0, dtype=np.int32),
                                                     swa=x["swa"], swa_len=spec.swa, scale=spec.scale))
        t = run_tasks(tasks, cores)
        res["cpu_baseline"] = {"value": 1.0 / t, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"1 whole step of {len(tasks)} layer tasks on {cores} host threads"}
    del steps
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------- eval window
EVAL_METRIC = "selection-eval windows/s (64 queries x 21 layers x 32K entries; golden TFLOP/s vs peak)"
EVAL_STAGES = ("score", "topk", "golden", "topp", "gold_topk", "vote", "gate", "fetched_topk", "overlap")


def eval_inputs(spec):
    layers = [synth.eval_layer(spec, l) for l in range(spec.L)]
    return layers, synth.eval_gate(spec)


def oracle_eval_tasks(spec, layers, n):
    """n tasks, each the oracle's golden probabilities of one query of one
    layer (all 64 heads, all N entries), its top-p set and top-k; each stands
    for 1/(L*T) of a window."""
    import oracle

    def task(i):
        x = layers[i % len(layers)]
        t = (i // len(layers)) % spec.T

        def run():
            p = oracle.golden(x["qa"][t:t + 1], x["kv"], 1, spec.H, spec.N, spec.scale)
            oracle.topp(p[0])
            oracle.topk(p[0], spec.k)
        return run

    return [task(i) for i in range(n)]


def eval_cfg(world):
    e = synth.EVAL_WINDOW
    return {"workload": e.name, "layers": e.L, "queries": e.T, "heads": e.H, "entries": e.N, "top_k": e.k,
            "top_p": f"{e.top_p_num}/{e.top_p_den}", "min_votes": e.min_votes,
            "gate_layers": list(e.gate_layers), "l2": "inputs larger than L2 (704 MB of attention rows)",
            "parallelism": f"replicas x{world}"}


def measure_eval(args, world, dist, device, local_rank, rank, want_cpu) -> dict:
    import torch
    import lightning_indexer_top_index_b200 as L
    from lightning_indexer_top_index_b200.evalwin import EvalWindow

    spec = synth.EVAL_WINDOW
    layers, gate = eval_inputs(spec)

    def bf(a):
        return bf16_tensor(a, "bf16")

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
    steps = max(3, min(args.steps, 20))  # a window is milliseconds: bound the timed work
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    ms, per = timed_loop(lambda i: win.enqueue(), steps, args.repeats, dist, device)
    clk = clocks.stop()
    ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in EVAL_STAGES}
    stage_ms = {n: 0.0 for n in EVAL_STAGES}
    reps = 5
    for _ in range(reps):
        win.enqueue(events=ev)
        torch.cuda.synchronize()
        for n in EVAL_STAGES:
            stage_ms[n] += ev[n][0].elapsed_time(ev[n][1]) / reps
    # end to end: pinned host queries in, the overlap counts back, every
    # window; two windows over the same caches, each with its own inputs, so
    # the next window's queries go in while this one computes
    pins = [t.pin_memory() for t in (q_idx_h, w_h, qa_h, gq_h, gu_h)]
    win2_in = [t.clone() for t in (q_idx, w, qa, gq, gu)]
    win2 = EvalWindow(keys, kv_all, *win2_in, spec.gate_layers, spec.N, spec.k,
                      (spec.top_p_num, spec.top_p_den), spec.min_votes, spec.scale)

    class _Window:  # the replica interface pipelined_e2e drives
        def __init__(self, wnd, inputs):
            self.wnd, self.inputs = wnd, inputs
            self.outs_src = (wnd.counts_nat_gold, wnd.counts_nat_f, wnd.counts_g_f, wnd.counts_natf_gold,
                             wnd.counts_natf_nat)

        def replay(self):
            self.wnd.enqueue()

    wins = [_Window(win, (q_idx, w, qa, gq, gu)), _Window(win2, win2_in)]
    outs = [[torch.empty(c.shape, dtype=c.dtype).pin_memory() for c in x.outs_src] for x in wins]

    def h2d(x):
        for d, hsrc in zip(x.inputs, pins):
            d.copy_(hsrc, non_blocking=True)

    def d2h(x, r):
        for o, c in zip(outs[r], x.outs_src):
            o.copy_(c, non_blocking=True)

    e2e_step, e2e_begin, e2e_end = pipelined_e2e(wins, h2d, d2h)
    e2e_begin()
    for i in range(2):
        e2e_step(i)
    e2e_end()
    e2e_ms, _ = timed_loop(e2e_step, steps, args.repeats, dist, device, begin=e2e_begin, end=e2e_end)
    pk = peaks()
    gflops = win.golden_flops()
    achieved = gflops / (stage_ms["golden"] * 1e-3) / 1e12
    peak = pk["bf16_tflops_sustained"]
    score_tflops = win.score_flops() / (stage_ms["score"] * 1e-3) / 1e12
    res = {
        "metric": EVAL_METRIC, "value": job_rate(1, world, ms), "unit": "windows/s", "ms_per_step": ms,
        "ms_per_step_repeats": per, "steps": steps, "dtype": "bf16", "config": eval_cfg(world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": profiled_traffic("eval-window", "golden"),
                     "kernel": "lidx_selection_eval (golden)",
                     "peak_source": pk["source"] + " bf16, sustained", "flops_per_launch": gflops,
                     "avg_launch_us": stage_ms["golden"] * 1e3},
        "stages_ms": stage_ms,
        "score_gemm": {"tflops": score_tflops, "frac_of_burst": score_tflops / pk["bf16_tflops"],
                       "frac_of_sustained": score_tflops / peak, "ms_per_window": stage_ms["score"]},
        "e2e": {"value": job_rate(1, world, e2e_ms), "unit": "windows/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pins),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs[0])},
        "gpu_launches": steps * args.repeats * win.kernel_launches(),
        "gpu_launches_per_step": win.kernel_launches(),
        "clocks": clk,
    }
    if want_cpu and rank == 0 and world == 1:
        cores = host_cores()
        n = max(cores, 4)
        t = run_tasks(oracle_eval_tasks(spec, layers, n), cores)
        res["cpu_baseline"] = {"value": n / (spec.L * spec.T) / t, "unit": "windows/s", "cores": cores,
                               "kind": "oracle",
                               "sample": f"{n} (query, layer) golden rows with their top-p and top-k on {cores} "
                                         f"host threads ({n}/{spec.L * spec.T} of a window)"}
    del win, win2, wins
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ the arms
def run_reference(args, name, rank):
    """The oracle arm: the workload's whole steps on every host core (one
    task per layer and sequence), as many as fit about a minute; `steps`
    reports the steps actually timed.  Rank 0 only."""
    if rank != 0:
        return
    cores = host_cores()
    if name == EVAL:
        spec = synth.EVAL_WINDOW
        layers, _ = eval_inputs(synth.scaled(spec, L=2))
        per_step = max(cores, 4)
        for _ in range(min(args.warmup, 1)):
            run_tasks(oracle_eval_tasks(spec, layers, per_step), cores)
        n = max(1, min(args.steps, 20))
        t = sum(run_tasks(oracle_eval_tasks(spec, layers, per_step), cores) for _ in range(n))
        v = n * per_step / (spec.L * spec.T) / t
        line = {"metric": EVAL_METRIC, "value": v, "unit": "windows/s", "n_gpus": args.gpus, "steps": n,
                "steps_requested": args.steps, "warmup": min(args.warmup, 1), "ms_per_step": t / n * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": eval_cfg(args.gpus), "impl": "reference",
                "cpu_baseline": {"value": v, "unit": "windows/s", "cores": cores, "kind": "oracle",
                                 "sample": f"each step: {per_step} (query, layer) golden rows with top-p and top-k "
                                           f"({per_step}/{spec.L * spec.T} of a window) on {cores} host threads"},
                "e2e": {"value": v, "unit": "windows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    spec = WORKLOADS[name]
    layers_inp = [synth.decode_layer(spec, l) for l in range(spec.layers)]
    tasks = oracle_decode_tasks(spec, layers_inp)
    t0 = run_tasks(tasks, cores)  # warm-up step, also the estimate
    n = max(1, min(args.steps, int(60.0 / max(t0, 1e-3))))
    t = sum(run_tasks(tasks, cores) for _ in range(n))
    v = n / t
    ab = algorithmic_bytes(spec)
    cfg = {"workload": spec.name, "layers": spec.layers, "batch": spec.B, "entries": spec.N, "heads": spec.H,
           "top_k": spec.k, "swa": spec.swa, "key_format": spec.key_dtype, "kv_format": spec.kv_dtype,
           "algorithmic_bytes_per_step": ab["step"], "parallelism": f"replicas x{args.gpus}"}
    line = {"metric": METRIC if name == "decode-64k" else name, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": n, "steps_requested": args.steps, "warmup": 1, "ms_per_step": t / n * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg, "impl": "reference",
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{n} whole step(s) of {len(tasks)} (layer, sequence) tasks on {cores} host "
                                       f"threads"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_lidx(args, rank, world, local_rank):
    import torch
    import lightning_indexer_top_index_b200 as L  # noqa: F401

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_group(world, device)

    def one(name, want_cpu=True):
        if name == EVAL:
            return measure_eval(args, world, dist, device, local_rank, rank, want_cpu)
        if name == MODEL:
            return measure_model(args, world, dist, device, local_rank, rank, want_cpu)
        return decode_forms(args, name, WORKLOADS[name], world, dist, device, local_rank, rank, want_cpu)

    head = one(args.workload)
    side = {}
    if not args.only and args.workload == "decode-64k":
        for name in SIDE_WORKLOADS:
            side[name] = one(name)
    if rank == 0:
        line = {"metric": head.pop("metric"), "value": head.pop("value"), "unit": head.pop("unit"),
                "n_gpus": world, "steps": head.pop("steps", args.steps), "warmup": args.warmup,
                "repeats": args.repeats, "ms_per_step": head.pop("ms_per_step"), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": head.pop("dtype"), "data": "synthetic",
                "config": head.pop("config")}
        line.update(head)
        if side:
            line["workloads"] = side
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--repeats", type=int, default=5, help="timed repeats of the step loop (median, >= 5)")
    ap.add_argument("--impl", default="lidx", choices=["lidx", "reference"])
    ap.add_argument("--workload", default="decode-64k", choices=sorted(WORKLOADS) + [EVAL, MODEL])
    ap.add_argument("--only", action="store_true", help="time the named workload alone")
    ap.add_argument("--layer-form", default="auto", choices=sorted(LAYER_FORMS),
                    help="CSA decode layers: one launch per layer, three calls, or (auto) time both and "
                         "report the faster")
    args = ap.parse_args()
    args.repeats = max(5, args.repeats)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if args.workload == MODEL:
            args.workload = "decode-64k"
        run_reference(args, args.workload, rank)
        return
    run_lidx(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
