#!/usr/bin/env python
"""Benchmark of the B200 W4A16 mixture-of-experts layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl chord|reference]
                    [--workload all|ep8_decode|ep8_prefill|tp8_decode|tp8_prefill|skew|tiny
                                |grouped_contiguous_ep8_gate_up|grouped_contiguous_ep8_down
                                |grouped_masked_ep8_gate_up|grouped_masked_ep8_down]

One step = one layer call through the C ABI: routing sort (chord_moe_align) then
chord_moe_forward (gate_up GEMM + SiLU*up, down GEMM, top-k weighted combine), on a
synthetic Kimi-K2-shaped batch already resident in HBM. Weights (1.09-1.19 GB) exceed the
126 MB L2, so no flush is needed between steps.

By default (--workload all) every layer workload of the metric runs in turn -- EP8 decode,
EP8 prefill, TP8 decode, TP8 prefill and the skewed-routing stress case -- each for K
timed steps, and one JSON line is printed (rank 0): `value` is the EP8 decode shard
(128 tokens, hidden 7168, moe_intermediate 2048, experts 0..47 of 384 local, top-8 from
uniform router logits) in microseconds per layer call for the whole job, i.e. the max over
ranks of the timed region divided by (steps x ranks), since each rank runs an independent
replica (the layer does not shard across GPUs here); `per_workload` holds the same record
for every workload: µs/call, per-kernel times, the roofline of the dominant kernel (HBM
for the weight-streaming decode schedule, BF16 tensor for the tensor-core prefill one),
the end-to-end number and the clocks seen.

The grouped_* workloads time the grouped operators instead (one step = one
chord_grouped_contiguous / chord_grouped_masked call: routing pass + GEMM) on an EP8 shard
(48 experts) at the rows per expert the blog's grouped table uses.

The exchange workloads time the device steps around a sharded layer on one GPU (the
collectives between them need several): ep8_exchange_decode / _prefill = chord_ep_plan +
chord_ep_pack + chord_ep_combine for the EP8 decode (128 tokens) or prefill (8192 tokens)
batch of one rank over 8 ranks (the returned rows synthetic), tp8_reduce =
chord_round_bf16 of the TP8 prefill partial sums, and tp8_reduce_peers = the all-reduce
and rounding by chord_tp_reduce_round over 8 rank buffers of one GPU (all 8 ranks' calls).

--impl reference times the CPU oracle (test infrastructure) on the headline workload on
the host cores: rank 0 only, other ranks exit without work.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a16_int4_mixture_align_b200 import inputs  # noqa: E402

METRIC = "W4A16 MoE layer µs/call; decode eff. HBM GB/s, prefill TFLOPS vs roofline"
UNIT = "us/call"
GATE_UP_BYTES_PER_EXPERT = None  # computed from the config
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
EV_EVERY = 8  # steps per step that records the per-kernel timing events
DEFAULT_STEPS = {"ep8_decode": 2000, "tp8_decode": 2000, "tiny": 2000, "ep8_prefill": 200,
                 "tp8_prefill": 400, "skew": 100}
EXCHANGE_WORKLOADS = ("ep8_exchange_decode", "ep8_exchange_prefill", "tp8_reduce", "tp8_reduce_peers")


def describe(cfg: inputs.MoEConfig) -> str:
    shard = f"experts 0..{cfg.E - 1} of {cfg.E_global} local" if cfg.E < cfg.E_global else f"all {cfg.E} experts"
    return (f"{cfg.name}: T={cfg.T} H={cfg.H} I={cfg.I} {shard} top-{cfg.topk} "
            f"{cfg.routing} router logits, int4 group-32 bf16 scales")


def peaks():
    try:
        with open(PEAKS_PATH) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def algorithmic_work(cfg: inputs.MoEConfig, ids: np.ndarray):
    """Bytes and FLOPs a layer call must move/compute, from the routing alone."""
    E, H, I = cfg.E, cfg.H, cfg.I
    flat = ids.reshape(-1)
    local = flat[(flat >= 0) & (flat < E)]
    R = int(local.size)
    active = int(np.unique(local).size)
    gu_w = 2 * I * H // 2 + 2 * I * (H // 32) * 2        # codes + scales of one expert
    dn_w = H * I // 2 + H * (I // 32) * 2
    tokens_local = int(((ids >= 0) & (ids < E)).any(axis=1).sum())
    gate_up = {"weights": active * gu_w, "x": tokens_local * H * 2, "a": R * I * 2}
    down = {"weights": active * dn_w, "a": R * I * 2, "y": R * H * 4}
    combine = {"y": R * H * 4, "out": cfg.T * H * 2}
    return {
        "R": R, "active_experts": active,
        "gate_up_bytes": sum(gate_up.values()), "down_bytes": sum(down.values()),
        "combine_bytes": sum(combine.values()),
        "layer_bytes": active * (gu_w + dn_w) + cfg.T * H * 2 * 2,
        "gate_up_flops": 2 * R * H * 2 * I, "down_flops": 2 * R * I * H,
        "unit_gate_up_bytes": gu_w,
    }


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU works."""

    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sms, maxes, reasons, n = [], [], set(), 0
        for ts, line in self.lines:
            if ts < t0 - 0.2 or ts > t1 + 0.2:
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            n += 1
            try:
                sms.append(float(parts[2]))
                maxes.append(float(parts[3]))
            except ValueError:
                pass
            for nm, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sms) if sms else None,
                "sm_max_mhz": max(maxes) if maxes else None,
                "reasons": sorted(reasons), "samples": n}


# ------------------------------------------------------------------------------ chord arm

def src_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if its kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)[kernel_key][workload]
    except Exception:
        return None
    if rec.get("src_sha") != src_digest(rec["sources"]):
        return None
    return rec["dram_bytes_per_launch"]


def pipelined_e2e_ms(K, W, copy_in, compute, copy_out, stream, dev, world):
    """Device time of K end-to-end steps: every step copies its inputs in from pinned host
    memory, runs the layer through the public API and copies the result back. Two buffer
    slots: step k + 1's copy in (one stream) and step k - 1's copy out (another) overlap
    step k's compute, as a serving loop runs them (PCIe is full duplex). Events order
    each slot's reuse: inputs are rewritten only after the compute that read them, outputs
    only after their copy out. The timed region runs from an event that both copy streams
    wait on to one recorded after the last copy out."""
    import torch

    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for k in range(n):
            s = k % 2
            if k >= 2:
                h2d.wait_event(done[s])
            with torch.cuda.stream(h2d):
                copy_in(s)
            in_ready[s].record(h2d)
            stream.wait_event(in_ready[s])
            if k >= 2:
                stream.wait_event(out_read[s])
            with torch.cuda.stream(stream):
                compute(s)
            done[s].record(stream)
            d2h.wait_event(done[s])
            with torch.cuda.stream(d2h):
                copy_out(s)
            out_read[s].record(d2h)

    run(W)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    last = torch.cuda.Event()
    start.record(stream)
    h2d.wait_event(start)
    d2h.wait_event(start)
    run(K)
    last.record(d2h)
    stream.wait_event(last)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(stop)


HEADLINE = "ep8_decode"
LAYER_WORKLOADS = ["ep8_decode", "ep8_prefill", "tp8_decode", "tp8_prefill", "skew"]


def tensor_peak(clocks, tf_burst, tf_sust, pk_kind):
    """The BF16 denominator for a tensor-bound kernel, chosen from the run's own clock
    record: the burst cuBLAS figure while the SM clock stays near its maximum, the
    sustained (power-capped) figure only when the clock record shows it pulled down."""
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm and mx and sm < 0.9 * mx and "sw_power_cap" in clocks.get("reasons", []):
        return tf_sust, f"{pk_kind} bf16_tflops_sustained (SM clock {sm:.0f} of {mx:.0f} MHz under sw_power_cap)"
    return tf_burst, f"{pk_kind} bf16_tflops burst (SM clock {sm} of {mx} MHz)"


class WeightCache:
    """Repacked layers keyed by their weight shape: the EP8 workloads share one set of
    weights (48 experts, intermediate 2048) and the TP8 ones another (384 experts, 256)."""

    def __init__(self, dev):
        self.dev, self.key, self.layer_args = dev, None, None

    def get(self, cfg):
        key = (cfg.E, cfg.H, cfg.I, cfg.seed)
        if key != self.key:
            self.layer_args = None
            w = inputs.make_weights(cfg)
            self.key, self.layer_args = key, (w[0], w[1].view(np.int16), w[2], w[3].view(np.int16))
        return self.layer_args


def run_workload(name, args, rank, world, local_rank, weights, sampler):
    """One layer workload: `value` graph (K plain steps), an instrumented graph (K steps,
    per-kernel events on every step) and the end-to-end leg; returns rank 0's record."""
    import torch
    from w4a16_int4_mixture_align_b200 import chord

    dev = torch.device("cuda", local_rank)
    cfg = inputs.CONFIGS[name]
    rcfg = inputs.MoEConfig(**{**cfg.__dict__, "seed": cfg.seed + rank})  # each replica its own batch
    ids_np, tw_np = inputs.make_routing(rcfg)
    x_np = inputs.make_hidden(rcfg)
    work = algorithmic_work(cfg, ids_np)
    qw13, s13, qw2, s2 = weights.get(cfg)
    layer = chord.ChordMoE(qw13, s13, qw2, s2, topk=cfg.topk, E_global=cfg.E_global, max_tokens=cfg.T, device=dev)
    x = torch.from_numpy(x_np.view(np.int16)).to(dev).view(torch.bfloat16)
    ids = torch.from_numpy(ids_np).to(dev)
    tw = torch.from_numpy(tw_np).to(dev)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    # all GPU work of the timed legs runs on one side stream (graph capture needs one)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    K = args.steps if args.steps is not None else DEFAULT_STEPS.get(name, 200)
    W = args.warmup

    def step():
        layer.forward(x, ids, tw, out=out)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    assert layer.check_status() == 0

    # The K timed steps are captured once into a CUDA graph (the library enqueues
    # everything on the caller's stream and never reads back, so a step is capturable),
    # then replayed: the timed region runs exactly the K steps' kernels, without the host
    # launch gaps of an eager loop, and with the early (programmatic) launches of the
    # production path.
    launches0 = chord.chord_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(K):
            layer.align(ids)
            chord.chord_moe_forward(x, ids, tw, layer.sorted_ids, layer.expert_ids, layer.ntp, layer.block_m,
                                    layer.w13, layer.w2, layer.I, layer.E, out, layer.workspace)
    launches = chord.chord_launch_count() - launches0  # kernels per replay (captured once)
    # The same K steps with the library's per-kernel timing events on every step: [start,
    # align done, gate_up done, down done, combine done]. An event between two kernels
    # orders them fully (no early launch), so these per-kernel times are each kernel's own
    # duration, and their sum is a little above the production step time.
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        for k in range(K):
            ev[k][0].record(stream)
            layer.align(ids)
            chord.chord_set_timing_events(ev[k][1:5])
            chord.chord_moe_forward(x, ids, tw, layer.sorted_ids, layer.expert_ids, layer.ntp, layer.block_m,
                                    layer.w13, layer.w2, layer.I, layer.E, out, layer.workspace)
            chord.chord_set_timing_events(None)
    graph.replay()  # one untimed replay of each
    graph_ev.replay()
    torch.cuda.synchronize()

    time.sleep(0.25)  # a few clock samples before the timed region
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    graph.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    elapsed_ms = start.elapsed_time(stop)
    graph_ev.replay()
    torch.cuda.synchronize()
    assert layer.check_status() == 0
    del graph, graph_ev
    seg = np.array([[ev[k][i].elapsed_time(ev[k][i + 1]) for i in range(4)] for k in range(K)])
    seg_ms = seg.mean(axis=0)  # align(+prep), gate_up, down, combine

    # ---- end to end: pinned host buffers, copies inside the timed region
    x_h = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    ids_h = torch.from_numpy(ids_np).pin_memory()
    tw_h = torch.from_numpy(tw_np).pin_memory()
    out_h = [torch.empty((cfg.T, cfg.H), dtype=torch.int16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    idsd = [torch.empty_like(ids) for _ in range(2)]
    twd = [torch.empty_like(tw) for _ in range(2)]
    outd = [torch.empty_like(out) for _ in range(2)]

    def copy_in(s):
        xd[s].view(torch.int16).copy_(x_h, non_blocking=True)
        idsd[s].copy_(ids_h, non_blocking=True)
        twd[s].copy_(tw_h, non_blocking=True)

    def compute(s):
        layer.forward(xd[s], idsd[s], twd[s], out=outd[s])

    def copy_out(s):
        out_h[s].copy_(outd[s].view(torch.int16), non_blocking=True)

    e2e_ms = pipelined_e2e_ms(K, W, copy_in, compute, copy_out, stream, dev, world)
    h2d = x_h.numel() * 2 + ids_h.numel() * 4 + tw_h.numel() * 4
    d2h = out_h[0].numel() * 2
    router_us = time_router(chord, cfg, rcfg, dev) if name == HEADLINE else None
    torch.cuda.set_stream(torch.cuda.default_stream(dev))
    block_m = layer.block_m
    del layer, xd, idsd, twd, outd
    torch.cuda.empty_cache()

    # ---- max over ranks (outside the timed regions)
    stats = max_over_ranks([elapsed_ms, e2e_ms, *seg_ms.tolist()], world, device=dev)
    elapsed_ms, e2e_ms, seg_ms = stats[0], stats[1], np.array(stats[2:])
    if rank != 0:
        return None

    hbm, tf_burst, tf_sust, pk_kind = peaks()
    clocks = sampler.summary(t_wall0, t_wall1)
    us_call = job_us_per_call(elapsed_ms, K, world)
    gu_us, dn_us = seg_ms[1] * 1000.0, seg_ms[2] * 1000.0
    decode = block_m <= 32
    tf_peak, tf_src = tensor_peak(clocks, tf_burst, tf_sust, pk_kind)
    if decode:
        achieved = work["gate_up_bytes"] / (gu_us * 1e-6) / 1e9
        achieved_dn = work["down_bytes"] / (dn_us * 1e-6) / 1e9
        roofline = {"bound": "hbm", "kernel": "stream_gemm gate_up", "achieved": round(achieved, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "peak_source": f"{pk_kind} hbm_gbs (burst copy; kernel timed alone by its events)",
                    "traffic": recorded_traffic("stream_gemm_gate_up", name),
                    "algorithmic_bytes_per_launch": work["gate_up_bytes"],
                    "down": {"achieved": round(achieved_dn, 1), "frac": round(achieved_dn / hbm, 4),
                             "algorithmic_bytes_per_launch": work["down_bytes"]}}
    else:
        achieved = work["gate_up_flops"] / (gu_us * 1e-6) / 1e12
        achieved_dn = work["down_flops"] / (dn_us * 1e-6) / 1e12
        roofline = {"bound": "tensor", "kernel": "tc_gemm gate_up", "achieved": round(achieved, 1),
                    "peak": tf_peak, "unit": "TFLOP/s", "frac": round(achieved / tf_peak, 4),
                    "peak_source": tf_src,
                    "frac_of_burst": round(achieved / tf_burst, 4), "frac_of_sustained": round(achieved / tf_sust, 4),
                    "traffic": recorded_traffic("tc_gemm_gate_up", name),
                    "algorithmic_flops_per_launch": work["gate_up_flops"],
                    "down": {"achieved": round(achieved_dn, 1), "frac": round(achieved_dn / tf_peak, 4),
                             "algorithmic_flops_per_launch": work["down_flops"]}}
    layer_us = elapsed_ms * 1000.0 / K
    rec = {
        "workload": describe(cfg), "us_per_call": round(us_call, 3), "steps": K, "warmup": W,
        "block_m": block_m, "schedule": "weight-streaming" if decode else "tensor-core",
        "routed_pairs": work["R"], "active_experts": work["active_experts"],
        "l2": "no flush: weights %.2f GB > 126 MB L2" % (work["layer_bytes"] / 1e9),
        "kernels_us": {"align+prep": round(seg_ms[0] * 1000, 2), "gate_up": round(gu_us, 2),
                       "down": round(dn_us, 2), "combine": round(seg_ms[3] * 1000, 2),
                       "gate_up+down": round(gu_us + dn_us, 2),
                       "how": "each kernel alone: CUDA events around it on every step of an "
                              "instrumented replay of the same K steps (no early launch)"},
        "layer": {"GB/s": round(work["layer_bytes"] / (layer_us * 1e-6) / 1e9, 1),
                  "hbm_frac": round(work["layer_bytes"] / (layer_us * 1e-6) / 1e9 / hbm, 4),
                  "TFLOP/s": round((work["gate_up_flops"] + work["down_flops"]) / (layer_us * 1e-6) / 1e12, 2),
                  "tensor_frac": round((work["gate_up_flops"] + work["down_flops"]) / (layer_us * 1e-6) / 1e12
                                       / tf_peak, 4)},
        "roofline": roofline,
        "e2e": {"value": round(job_us_per_call(e2e_ms, K, world), 3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if router_us is not None:
        rec["router_topk_align"] = {
            "us_per_call": round(router_us, 2),
            "what": "chord_router_topk_align on fp32 logits [T, E_global], top-%d, then the routing sort "
                    "(not part of value)" % cfg.topk}
    return rec


def run_chord(args, rank, world, local_rank):
    """The layer workloads: the headline (EP8 decode) as `value`, every workload of the
    metric in `per_workload` (or one workload when --workload names it)."""
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    names = LAYER_WORKLOADS if args.workload == "all" else [args.workload]
    head = HEADLINE if args.workload == "all" else args.workload
    weights = WeightCache(dev)
    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else local_rank)
    sampler.start()
    recs = {}
    try:
        for name in names:
            recs[name] = run_workload(name, args, rank, world, local_rank, weights, sampler)
    finally:
        sampler.stop()
    if rank != 0:
        return None
    h = recs[head]
    cfg = inputs.CONFIGS[head]
    line = {
        "metric": METRIC, "value": h["us_per_call"], "unit": UNIT, "n_gpus": world,
        "steps": h["steps"], "warmup": h["warmup"], "ms_per_step": round(h["us_per_call"] * world / 1000.0, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": describe(cfg), "block_m": h["block_m"], "schedule": h["schedule"],
                   "routed_pairs": h["routed_pairs"], "active_experts": h["active_experts"],
                   "l2": h["l2"], "parallelism": f"replicas x{world}"},
        "kernels_us": h["kernels_us"], "layer": h["layer"], "roofline": h["roofline"], "e2e": h["e2e"],
        "gpu_launches": h["gpu_launches"], "clocks": h["clocks"],
    }
    if "router_topk_align" in h:
        line["router_topk_align"] = h["router_topk_align"]
    if len(recs) > 1:
        line["per_workload"] = recs
    return line


def time_router(chord, cfg, rcfg, dev, calls=20, replays=10):
    """Device µs per chord_router_topk_align call on seeded N(0,1) logits of the workload's
    shape, from CUDA-graph replays of `calls` back-to-back calls."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(rcfg.seed)
    T, G, k, E = cfg.T, cfg.E_global, cfg.topk, cfg.E
    bm = chord.chord_select_block_m(T, k, E, G, cfg.H, cfg.I)
    logits = torch.randn((T, G), dtype=torch.float32, device=dev, generator=g)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    s = torch.empty(chord.chord_moe_align_capacity(T, k, E, bm), dtype=torch.int32, device=dev)
    e = torch.empty(max(chord.chord_moe_align_num_blocks(T, k, E, bm), 1), dtype=torch.int32, device=dev)
    n = torch.empty(2, dtype=torch.int32, device=dev)  # padded count, routing tag
    wsb = chord.chord_moe_align_workspace_bytes(T, k, E)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev) if wsb else None
    side = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(side):
        for _ in range(3):
            chord.chord_router_topk_align(logits, k, E, bm, ids, w, s, e, n, None, ws)
        side.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for _ in range(calls):
                chord.chord_router_topk_align(logits, k, E, bm, ids, w, s, e, n, None, ws)
        graph.replay()
        side.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(side)
        for _ in range(replays):
            graph.replay()
        b.record(side)
        side.synchronize()
    del graph
    return a.elapsed_time(b) * 1000.0 / (calls * replays)


# ------------------------------------------------------------------------------ grouped operators

GROUPED_METRIC = "W4A16 grouped GEMM µs/call; eff. HBM GB/s (masked decode) or TFLOPS (contiguous prefill)"


def describe_grouped(cfg) -> str:
    lay = (f"masked, max_m={cfg.max_m}, masked_m={cfg.rows} ({cfg.balance})" if cfg.mode == "masked"
           else f"contiguous, {cfg.rows} rows/expert ({cfg.balance}), runs padded to 128")
    return (f"{cfg.name}: E={cfg.E} N={cfg.N} K={cfg.K}, {lay}, int4 group-32 bf16 scales")


def grouped_work(cfg, counts):
    valid = int(counts.sum())
    active = int((counts > 0).sum())
    w_bytes = active * (cfg.N * cfg.K // 2 + cfg.N * (cfg.K // 32) * 2)
    return {"valid_rows": valid, "active_experts": active,
            "bytes": w_bytes + valid * cfg.K * 2 + valid * cfg.N * 2,
            "flops": 2 * valid * cfg.N * cfg.K}


def run_grouped(args, rank, world, local_rank):
    """One step = one grouped operator call (routing pass + GEMM) through the C ABI."""
    import torch
    from w4a16_int4_mixture_align_b200 import chord

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = inputs.GROUPED_CONFIGS[args.workload]
    d = inputs.make_grouped(inputs.GroupedConfig(**{**cfg.__dict__, "seed": cfg.seed + rank}))
    work = grouped_work(cfg, d["counts"])
    w = chord.pack_w4a16_grouped(d["qweight"], d["scales"].view(np.int16), cfg.mode, device=dev)
    del d["qweight"], d["scales"]
    x_np = d["x"]
    x = torch.from_numpy(x_np.view(np.int16)).to(dev).view(torch.bfloat16)
    M = x_np.size // cfg.K
    out = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
    route_np = d["m_indices"] if cfg.mode == "contiguous" else d["masked_m"]
    route = torch.from_numpy(route_np).to(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    flags = {"auto": 0, "stream": chord.CHORD_FLAG_FORCE_STREAM, "tensor": chord.CHORD_FLAG_FORCE_TENSOR}[args.schedule]
    expected_m = args.expected_m or cfg.rows

    def call(xx, rr, oo):
        if cfg.mode == "contiguous":
            chord.contiguous(xx, w, rr, out=oo, flags=flags)
        else:
            chord.masked(xx, w, rr, expected_m, out=oo, flags=flags)

    K, W = args.steps, args.warmup
    for _ in range(W):
        call(x, route, out)
    torch.cuda.synchronize()
    assert w.check_status() == 0
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    # timing events on every EV_EVERY-th call only (event nodes add gaps between kernels)
    timed_steps = [k for k in range(K) if k % EV_EVERY == 0]
    launches0 = chord.chord_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for k in range(K):
            timed = k % EV_EVERY == 0
            if timed:
                ev[k][0].record(stream)
                chord.chord_set_timing_events([ev[k][1], ev[k][2], ev[k][2], ev[k][2]])
            call(x, route, out)
            if timed:
                chord.chord_set_timing_events(None)
    launches = chord.chord_launch_count() - launches0
    graph.replay()
    torch.cuda.synchronize()
    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else local_rank)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    graph.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    elapsed_ms = start.elapsed_time(stop)
    assert w.check_status() == 0
    del graph
    seg = np.array([[ev[k][0].elapsed_time(ev[k][1]), ev[k][1].elapsed_time(ev[k][2])] for k in timed_steps])
    seg_ms = seg.mean(axis=0)  # routing pass, GEMM

    # end to end: activations and routing from pinned host memory, the result back
    x_h = torch.from_numpy(x_np.view(np.int16)).pin_memory()
    r_h = torch.from_numpy(route_np).pin_memory()
    out_h = [torch.empty((M, cfg.N), dtype=torch.int16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    rd = [torch.empty_like(route) for _ in range(2)]
    outd = [torch.empty_like(out) for _ in range(2)]

    def copy_in(s):
        xd[s].view(torch.int16).copy_(x_h, non_blocking=True)
        rd[s].copy_(r_h, non_blocking=True)

    def compute(s):
        call(xd[s], rd[s], outd[s])

    def copy_out(s):
        out_h[s].copy_(outd[s].view(torch.int16), non_blocking=True)

    e2e_ms = pipelined_e2e_ms(K, W, copy_in, compute, copy_out, stream, dev, world)
    sampler.stop()
    stats = max_over_ranks([elapsed_ms, e2e_ms, *seg_ms.tolist()], world, device=dev)
    elapsed_ms, e2e_ms, seg_ms = stats[0], stats[1], np.array(stats[2:])
    if rank != 0:
        return None

    hbm, tf_burst, tf_sust, pk_kind = peaks()
    clocks = sampler.summary(t_wall0, t_wall1)
    gemm_us = seg_ms[1] * 1000.0
    # the library's default schedule: expected rows per expert (masked: the expected_m hint;
    # contiguous: padded rows / E) above 16 go to the tensor cores
    expected = expected_m if cfg.mode == "masked" else -(-M // cfg.E)
    tensor = args.schedule == "tensor" or (args.schedule == "auto" and expected > 16)
    unit = ((32 if expected <= 32 else 64 if expected <= 64 else 128 if expected <= 128 else 256) if tensor
            else (8 if expected <= 8 else (16 if expected <= 16 else 32)))
    if tensor:
        achieved = work["flops"] / (gemm_us * 1e-6) / 1e12
        tf_peak, tf_src = tensor_peak(clocks, tf_burst, tf_sust, pk_kind)
        roofline = {"bound": "tensor", "kernel": "tc_gemm (plain epilogue)", "achieved": round(achieved, 1),
                    "peak": tf_peak, "unit": "TFLOP/s", "frac": round(achieved / tf_peak, 4), "peak_source": tf_src,
                    "frac_of_burst": round(achieved / tf_burst, 4), "frac_of_sustained": round(achieved / tf_sust, 4),
                    "traffic": recorded_traffic("tc_gemm_plain", args.workload),
                    "algorithmic_flops_per_launch": work["flops"]}
    else:
        achieved = work["bytes"] / (gemm_us * 1e-6) / 1e9
        roofline = {"bound": "hbm", "kernel": "stream_gemm (plain epilogue)", "achieved": round(achieved, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4), "peak_source": f"{pk_kind} hbm_gbs",
                    "traffic": recorded_traffic("stream_gemm_plain", args.workload),
                    "algorithmic_bytes_per_launch": work["bytes"]}
    return {
        "metric": GROUPED_METRIC, "value": round(job_us_per_call(elapsed_ms, K, world), 3), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(elapsed_ms / K, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe_grouped(cfg), "schedule": "tensor-core" if tensor else "weight-streaming",
                   "unit_rows": unit, "expected_m": expected_m if cfg.mode == "masked" else None,
                   "valid_rows": work["valid_rows"], "active_experts": work["active_experts"],
                   "l2": "no flush: weights %.2f GB > 126 MB L2" % (work["bytes"] / 1e9),
                   "parallelism": f"replicas x{world}"},
        "kernels_us": {"routing": round(seg_ms[0] * 1000, 2), "gemm": round(gemm_us, 2)},
        "roofline": roofline,
        "e2e": {"value": round(job_us_per_call(e2e_ms, K, world), 3), "unit": UNIT,
                "h2d_bytes_per_step": x_h.numel() * 2 + r_h.numel() * 4, "d2h_bytes_per_step": out_h[0].numel() * 2},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }


def grouped_cpu_baseline(cfg, n_experts=2, d=None):
    """The oracle's grouped GEMM on a bounded sample: every valid row of n_experts experts
    (seeded choice among the active ones), scaled to the full call by active experts."""
    import oracle
    oracle.build()
    d = inputs.make_grouped(cfg) if d is None else d
    if cfg.mode == "contiguous":
        ex = d["m_indices"].astype(np.int64)
    else:
        r = np.arange(cfg.E * cfg.max_m)
        ex = np.where(r % cfg.max_m < d["masked_m"][r // cfg.max_m], r // cfg.max_m, -1)
    active = np.unique(ex[ex >= 0])
    pick = np.random.default_rng(0).choice(active, min(n_experts, active.size), replace=False)
    rows = np.nonzero(np.isin(ex, pick))[0]
    threads = os.cpu_count() or 1
    t0 = time.time()
    oracle.grouped_gemm(d["x"].reshape(-1, cfg.K)[rows], d["qweight"], d["scales"],
                        m_indices=ex[rows].astype(np.int32), n_threads=threads)
    el = time.time() - t0
    us = el * 1e6 * active.size / pick.size
    return {"value": round(us, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"all {rows.size} valid rows of {pick.size} of {active.size} active experts "
                      f"(seeded), scaled by active experts"}


def max_over_ranks(vals, world, device=None):
    """Element-wise max of `vals` over all ranks (one all-reduce; identity for world 1)."""
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def job_us_per_call(max_elapsed_ms: float, steps: int, world: int) -> float:
    """Whole-job microseconds per layer call: every rank ran `steps` independent calls."""
    return max_elapsed_ms * 1000.0 / (steps * world)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------ oracle arms

def oracle_call(d, threads):
    import oracle
    return oracle.moe_forward(d["x"], d["topk_ids"], d["topk_weights"], d["qw13"], d["s13"],
                              d["qw2"], d["s2"], n_threads=threads)


def cpu_baseline(cfg, max_seconds=30.0):
    """The oracle as it stands on the host cores: full layer calls, repeated while the
    total stays within ~max_seconds (at least one call)."""
    import oracle
    oracle.build()
    d = inputs.make_inputs(cfg)
    threads = os.cpu_count() or 1
    times = []
    t_total = time.time()
    while True:
        t0 = time.time()
        oracle_call(d, threads)
        times.append(time.time() - t0)
        if time.time() - t_total + times[-1] > max_seconds or len(times) >= 5:
            break
    us = statistics.median(times) * 1e6
    return {"value": round(us, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{len(times)} full layer call(s) of the workload (all {cfg.T} tokens), median"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    if args.workload in EXCHANGE_WORKLOADS:
        return {"impl": "reference", "unavailable": "the oracle has no exchange steps: they only move rows "
                "(bit-exact against their definitions in the tests)"}
    import oracle
    oracle.build()
    if args.workload in inputs.GROUPED_CONFIGS:
        return run_reference_grouped(args, world)
    cfg = inputs.CONFIGS[HEADLINE if args.workload == "all" else args.workload]
    d = inputs.make_inputs(cfg)
    threads = os.cpu_count() or 1
    for _ in range(args.warmup):
        oracle_call(d, threads)
    t0 = time.time()
    for _ in range(args.steps):
        oracle_call(d, threads)
    el = time.time() - t0
    us = el * 1e6 / args.steps
    return {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1000 / args.steps, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": {"workload": describe(cfg), "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"each step one full layer call of the workload (all {cfg.T} tokens)"},
        "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_grouped(args, world):
    """Each step: the oracle's grouped GEMM on a 64-row seeded sample of the workload,
    scaled to the full call by valid rows."""
    cfg = inputs.GROUPED_CONFIGS[args.workload]
    d = inputs.make_grouped(cfg)
    for _ in range(args.warmup):
        grouped_cpu_baseline(cfg, d=d)
    vals = [grouped_cpu_baseline(cfg, d=d) for _ in range(args.steps)]
    us = statistics.mean(v["value"] for v in vals)
    base = dict(vals[0], value=round(us, 1))
    return {
        "impl": "reference", "metric": GROUPED_METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1000, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": {"workload": describe_grouped(cfg), "parallelism": "rank 0 only"},
        "cpu_baseline": base,
        "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------ main

def run_exchange(args, rank, world, local_rank):
    """The device steps of a sharded layer's exchange on one GPU (the collectives between
    them need several GPUs and are not timed here).

    ep8_exchange_decode / _prefill: the EP8 decode (128 tokens) or prefill (8192 tokens)
    batch of one rank, top-8 of 384 experts by global id, over 8 expert-parallel ranks of
    48 experts: chord_ep_plan (send rows by destination rank),
    chord_ep_pack (hidden rows, local ids and weights of every send row) and
    chord_ep_combine (the returned rows summed per token in rank order; synthetic rows
    stand in for what the other ranks send back). tp8_reduce: chord_round_bf16 of one
    TP8 prefill output, FP32 [4096, 7168], after the all-reduce."""
    import torch
    from w4a16_int4_mixture_align_b200 import chord

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    K, W = args.steps, args.warmup
    if args.workload.startswith("ep8_exchange"):
        cfg = inputs.CONFIGS["ep8_decode" if args.workload.endswith("decode") else "ep8_prefill"]
        rcfg = inputs.MoEConfig(**{**cfg.__dict__, "seed": cfg.seed + rank})
        ids_np, tw_np = inputs.make_routing(rcfg, global_ids=True)
        x_np = inputs.make_hidden(rcfg)
        T, H, k, E_rank, Wr = cfg.T, cfg.H, cfg.topk, cfg.E, cfg.E_global // cfg.E
        host_in = [torch.from_numpy(x_np.view(np.int16)), torch.from_numpy(ids_np), torch.from_numpy(tw_np)]
        send_rows = torch.empty(T * Wr, dtype=torch.int32, device=dev)
        offsets = torch.empty(Wr + 1, dtype=torch.int32, device=dev)
        row_of = torch.empty(T * Wr, dtype=torch.int32, device=dev)
        ws = torch.empty(max(chord.chord_ep_plan_workspace_bytes(T, Wr), 256), dtype=torch.uint8, device=dev)
        send_x = torch.empty((T * Wr, H), dtype=torch.bfloat16, device=dev)
        send_ids = torch.empty((T * Wr, k), dtype=torch.int32, device=dev)
        send_w = torch.empty((T * Wr, k), dtype=torch.float32, device=dev)
        # the rows the other ranks return: one per send row (counted on the host)
        n_send = sum(1 for t in range(T) for d in range(Wr)
                     if np.any((ids_np[t] >= d * E_rank) & (ids_np[t] < (d + 1) * E_rank)))
        back = torch.from_numpy(np.random.default_rng(rank).standard_normal((max(n_send, 1), H)).astype(np.float32))
        back = back.to(dev).to(torch.bfloat16)
        out_shape, out_dtype = (T, H), torch.bfloat16

        def steps(xin, oo):
            xx, ii, ww = xin
            xx = xx.view(torch.bfloat16)
            return [lambda: chord.chord_ep_plan(ii, E_rank, Wr, send_rows, offsets, row_of, ws),
                    lambda: chord.chord_ep_pack(xx, ii, ww, E_rank, Wr, send_rows, offsets, row_of, send_x, send_ids,
                                                send_w),
                    lambda: chord.chord_ep_combine(back, row_of, Wr, oo)]
        names = ["plan", "pack", "combine"]
        # algorithmic bytes: plan reads the ids and writes the send rows and row_of; pack
        # reads each hidden row once (a row sent to several ranks is read again from L2)
        # and writes every send row (+ its ids and weights); combine reads the returned rows
        # and writes out
        nbytes = [T * k * 4 + 2 * T * Wr * 4 + (Wr + 1) * 4,
                  T * H * 2 + n_send * H * 2 + n_send * k * 8 + n_send * 4 + T * Wr * 4,
                  n_send * H * 2 + T * Wr * 4 + T * H * 2]
        desc = (f"{args.workload}: EP8 batch T={T} top-{k} (global ids) over {Wr} ranks x {E_rank} experts, "
                f"H={H}: {n_send} send rows; plan + pack + combine (the all-to-all legs not included)")
    elif args.workload == "tp8_reduce_peers":
        # 8 ranks' FP32 partials and BF16 outputs as buffers of this GPU; one step runs every
        # rank's call (its slice reduced in rank order and stored into all 8 outputs): the
        # whole all-reduce of one TP8 prefill output, emulated on one GPU
        cfg = inputs.CONFIGS["tp8_prefill"]
        T, H, Wr = cfg.T, cfg.H, 8
        rng = np.random.default_rng(rank)
        host_in = [torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)) for _ in range(Wr)]
        out_shape, out_dtype = (T, H), torch.bfloat16
        peer_outs = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(Wr - 1)]

        def steps(xin, oo):
            outs = [oo] + peer_outs
            return [lambda r=r: chord.chord_tp_reduce_round(list(xin), outs, r) for r in range(Wr)]
        names = [f"rank{r}" for r in range(Wr)]
        nbytes = [Wr * (T * H // Wr) * 4 + Wr * (T * H // Wr) * 2] * Wr
        desc = (f"tp8_reduce_peers: chord_tp_reduce_round over {Wr} rank buffers of one GPU, FP32 [{T}, {H}] each "
                f"-> BF16 into all {Wr} outputs (one step = every rank's call)")
    else:
        cfg = inputs.CONFIGS["tp8_prefill"]
        T, H = cfg.T, cfg.H
        host_in = [torch.from_numpy(np.random.default_rng(rank).standard_normal((T, H)).astype(np.float32))]
        out_shape, out_dtype = (T, H), torch.bfloat16

        def steps(xin, oo):
            return [lambda: chord.chord_round_bf16(xin[0], oo)]
        names = ["round"]
        nbytes = [T * H * 4 + T * H * 2]
        desc = f"tp8_reduce: chord_round_bf16 of a TP8 prefill output, FP32 [{T}, {H}] -> BF16 (after the all-reduce)"

    dev_in = [t.to(dev) for t in host_in]
    out = torch.empty(out_shape, dtype=out_dtype, device=dev)
    fns = steps(dev_in, out)

    def step():
        for f in fns:
            f()

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    # timed: one graph replay of the K steps; per kernel: a second graph with events between
    launches0 = chord.chord_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(K):
            step()
    launches = chord.chord_launch_count() - launches0
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(fns) + 1)] for _ in range(K)]
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        for kk in range(K):
            ev[kk][0].record(stream)
            for i, f in enumerate(fns):
                f()
                ev[kk][i + 1].record(stream)
    graph.replay()
    g2.replay()
    torch.cuda.synchronize()
    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else local_rank)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    graph.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    elapsed_ms = start.elapsed_time(stop)
    g2.replay()
    torch.cuda.synchronize()
    seg_ms = np.array([[ev[kk][i].elapsed_time(ev[kk][i + 1]) for i in range(len(fns))] for kk in range(K)]).mean(0)
    del graph, g2

    # end to end: the inputs from pinned host memory, the output back, two buffer slots
    host_pin = [t.pin_memory() for t in host_in]
    din = [[torch.empty_like(t) for t in dev_in] for _ in range(2)]
    outd = [torch.empty_like(out) for _ in range(2)]
    out_h = [torch.empty(out_shape, dtype=torch.int16).pin_memory() for _ in range(2)]
    slot_fns = [steps(din[s], outd[s]) for s in range(2)]

    def copy_in(s):
        for dst, src in zip(din[s], host_pin):
            dst.copy_(src, non_blocking=True)

    def compute(s):
        for f in slot_fns[s]:
            f()

    def copy_out(s):
        out_h[s].copy_(outd[s].view(torch.int16), non_blocking=True)

    e2e_ms = pipelined_e2e_ms(K, W, copy_in, compute, copy_out, stream, dev, world)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    stats = max_over_ranks([elapsed_ms, e2e_ms, *seg_ms.tolist()], world, device=dev)
    elapsed_ms, e2e_ms, seg_ms = stats[0], stats[1], np.array(stats[2:])
    if rank != 0:
        return None
    hbm = peaks()[0]
    top = int(np.argmax(nbytes))  # the kernel that moves the most bytes
    achieved = nbytes[top] / (seg_ms[top] * 1e-3) / 1e9
    return {
        "metric": "exchange steps of a sharded layer, µs/call; HBM GB/s vs roofline",
        "value": round(job_us_per_call(elapsed_ms, K, world), 3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(elapsed_ms / K, 5), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": desc, "l2": "no flush (each step rewrites its outputs)",
                   "parallelism": f"replicas x{world}"},
        "kernels_us": {n: round(v * 1000, 2) for n, v in zip(names, seg_ms)},
        "roofline": {"bound": "hbm", "kernel": names[top], "achieved": round(achieved, 1), "peak": hbm,
                     "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                     "algorithmic_bytes_per_launch": int(nbytes[top])},
        "e2e": {"value": round(job_us_per_call(e2e_ms, K, world), 3), "unit": UNIT,
                "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host_in)),
                "d2h_bytes_per_step": int(out.numel() * 2)},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["chord", "reference"], default="chord")
    ap.add_argument("--workload", choices=["all"] + list(inputs.CONFIGS) + sorted(inputs.GROUPED_CONFIGS)
                    + list(EXCHANGE_WORKLOADS),
                    default="all",
                    help="all (default): the EP8 decode headline plus every layer workload of the metric")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", choices=["auto", "stream", "tensor"], default="auto",
                    help="grouped workloads: force the GEMM schedule")
    ap.add_argument("--expected-m", type=int, default=None,
                    help="grouped masked workloads: the expected_m hint (default: the rows per expert)")
    args = ap.parse_args()
    if args.steps is None and (args.impl == "reference" or args.workload in inputs.GROUPED_CONFIGS
                               or args.workload in EXCHANGE_WORKLOADS):
        args.steps = 3 if args.impl == "reference" else 200
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the oracle runs on rank 0 alone; other ranks exit without work
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    grouped = args.workload in inputs.GROUPED_CONFIGS
    exchange = args.workload in EXCHANGE_WORKLOADS
    line = (run_exchange if exchange else run_grouped if grouped else run_chord)(args, rank, world, local_rank)
    if line is not None:
        if exchange:
            line["cpu_baseline"] = None
        elif world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = (grouped_cpu_baseline(inputs.GROUPED_CONFIGS[args.workload]) if grouped
                                    else cpu_baseline(inputs.CONFIGS[HEADLINE if args.workload == "all"
                                                                         else args.workload]))
        else:
            line["cpu_baseline"] = None
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
