#!/usr/bin/env python
"""Gated-prefill benchmark: input tokens/s of one TokenGate prefill step on B200.

A step is one pass of the whole hot path over one synthetic batch: gate scores and
their sequence RMSNorm, prunable-only top-K with compaction, the row gather, then per
gated layer the RMSNorm-folded QKV projection, RoPE at original positions, the
compacted KV-cache write, token-gated attention and the output projection.

Default workload: N=16384 (16320 document + 64 question tokens), budget 1638 kept,
28 stacked gated layers, Qwen3-1.7B-sized heads (16 q / 8 kv, head_dim 128).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload n16k|n128k|...]
  python bench.py --impl reference ...   # the CPU oracle timed on the host cores

Multi-GPU (torchrun, one rank per GPU): every rank runs an independent replica on
its own batch (no collective on the data path); value = all ranks' tokens / the
slowest rank's time.

Timing: W untimed warm-up steps; then K steps, each a replay of a CUDA graph of the step
between two CUDA events; L2 is flushed (a 512 MiB write) before every timed step, outside
the events.  SM clocks and throttle reasons are sampled through NVML during that loop.  A
second loop of K replays of the same step captured with timing events at every stage
boundary gives the per-stage times (and the roofline of the dominant kernel).
Workloads named by `--also` (default: the 128k one) are measured the same way after
the main one and reported under "workloads" in the same line.

Alongside (`--dense-steps`, default 3): the same layer stack over every token with no
gate (K = N, gamma = 0, tau = 1) on the same kernels, the GPU's own full-context
prefill, reported under "dense_reference" with the gated step's speedup over it.
`--lower-layers L` puts L full-context layers below the gate (the gate then scores
their output and their caches are trimmed to the kept rows).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-prefill input tokens/s at N=16k/128k; attn TFLOP/s & select GB/s vs peak"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="n16k")
    ap.add_argument("--launch", choices=["graph", "eager"], default="graph")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the end-to-end loop (default: --steps); the loop's "
                         "first upload is not overlapped, so fewer steps weigh it more")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-layers", type=int, default=12)
    ap.add_argument("--lower-layers", type=int, default=0,
                    help="full-context layers below the gate (their caches trimmed to the "
                         "kept rows); 0 = the gate reads the input rows directly")
    ap.add_argument("--full-layers", action="store_true",
                    help="full layer bodies (weighted norms, QK-norm, SwiGLU MLP of width "
                         "6144) instead of attention-only layers")
    ap.add_argument("--bias-grad-steps", type=int, default=10,
                    help="timed calls of the attention backward w.r.t. the gate (0 skips it)")
    ap.add_argument("--scorer-bwd-steps", type=int, default=5,
                    help="timed calls of the scorer backward (parameter gradients from a "
                         "seeded d kept_bias; 0 skips it)")
    ap.add_argument("--also", default="n128k,n16k@bucket",
                    help="comma-separated workloads measured after the main one and "
                         "reported as sub-records of the same line ('' for none); "
                         "'name@bucket' or 'name@ROWS' runs the layers above the gate on a "
                         "padded row count (the fixed-padding graph form)")
    ap.add_argument("--fuse-boundaries", choices=("on", "off"), default=None,
                    help="one launch per layer boundary, the output projection and the next "
                         "layer's QKV (tg_out_proj_qkv_next; default: the library's choice)")
    ap.add_argument("--launch-overlap", choices=("on", "off"), default=None,
                    help="programmatic dependent launch between the library's kernels "
                         "(tg_set_launch_overlap; default: the library's choice)")
    ap.add_argument("--rope-rows", choices=("on", "off"), default=None,
                    help="QKV RoPE from the per-row table of tg_rope_rows (default: the "
                         "library's choice)")
    ap.add_argument("--k-pad", default=None,
                    help="run the layers above the gate on a padded row count: an integer, "
                         "or 'bucket' for the kept total rounded up to a multiple of 256 "
                         "(the fixed-padding graph form; tokens/s still counts the input "
                         "tokens, the padding rows are extra work)")
    ap.add_argument("--dense-steps", type=int, default=3,
                    help="timed steps of the full-context reference (0 skips it)")
    args = ap.parse_args()
    if args.e2e_steps is None:
        args.e2e_steps = args.steps
    return args


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload(name):
    import synthetic_inputs as S
    table = S.all_workloads()
    if name not in table:
        raise SystemExit(f"unknown workload {name}; choose from {sorted(table)}")
    return table[name]


# ------------------------------------------------------------------ replicas (N > 1)

def replica_workload(wl, rank, world):
    """Rank r's own batch: the same shapes and weights, request seeds offset by 1000 r (no
    data is shared between ranks: the path shards by request, replicas only)."""
    if world <= 1:
        return wl
    import synthetic_inputs as S
    return S.Workload(**{**wl.__dict__, "seeds": tuple(s + 1000 * rank for s in wl.seeds)})


def max_over_ranks(ms, world, device):
    """The slowest rank's time (every rank takes this collective step, in the same order)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_step, world, steps, total_ms):
    """Tokens/s of the whole job: every rank's tokens over the slowest rank's time."""
    return tokens_per_step * world * steps / (total_ms / 1e3)


# ------------------------------------------------------------------ algorithmic work

def stage_work(wl, kept_counts, ffn=0):
    """Algorithmic bytes / flops per launch of each stage (see the design notes)."""
    T = wl.total_tokens
    Ks = [kept_counts[b + 1] - kept_counts[b] for b in range(wl.batch)]
    K = sum(Ks)
    H, F, hq, hkv, d = wl.hidden, wl.scorer_width, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    nqkv = (hq + 2 * hkv) * d
    attn_pairs = sum(k * (k + 1) // 2 for k in Ks)
    return {
        "gate_score": {"bound": "hbm", "bytes": T * H * 2 + F * H * 2 + T * 4 * 3 + T,
                       "flops": 2 * T * H * F},
        "seq_rmsnorm": {"bound": "hbm", "bytes": T * 13},
        "topk_compact": {"bound": "hbm", "bytes": T * 5 + K * 12},
        "gather": {"bound": "hbm", "bytes": 2 * K * H * 2 + K * 4},
        "rope_rows": {"bound": "hbm", "bytes": 2 * K * d * 4 + K * 4},
        "qkv_rope_cache": {"bound": "tensor", "flops": 2 * K * H * nqkv,
                           "bytes": K * H * 2 + nqkv * H * 2 + K * nqkv * 2 + K * 4
                           + K * (H // 128) * 4},
        "out_proj_qkv": {"bound": "tensor", "flops": 2 * K * hq * d * H + 2 * K * H * nqkv},
        "qkv_proj": {"bound": "tensor", "flops": 2 * K * H * nqkv,
                     "bytes": K * H * 2 + nqkv * H * 2 + K * nqkv * 2},
        "rope": {"bound": "hbm", "bytes": 2 * K * (hq + hkv) * d * 2 + K * 4},
        "kv_compact": {"bound": "hbm", "bytes": 2 * 2 * K * hkv * d * 2},
        "attention": {"bound": "tensor", "flops": 4 * d * hq * attn_pairs},
        "out_proj": {"bound": "tensor", "flops": 2 * K * hq * d * H,
                     "bytes": K * hq * d * 2 + H * hq * d * 2 + 2 * K * H * 2},
        # layers below the gate: the same kernels over all T tokens, and the trim of
        # their caches to the kept rows (one launch per lower layer)
        "lower_qkv_rope_cache": {"bound": "tensor", "flops": 2 * T * H * nqkv},
        "lower_attention": {"bound": "tensor",
                            "flops": 4 * d * hq * sum(n * (n + 1) // 2 for n in wl.lengths)},
        "lower_out_proj": {"bound": "tensor", "flops": 2 * T * hq * d * H},
        "lower_kv_trim": {"bound": "hbm", "bytes": 2 * 2 * K * hkv * d * 2 + K * 4},
        # full layer body: the SwiGLU MLP (gate/up GEMM with the SiLU product, down
        # projection with the residual)
        "mlp_gate_up": {"bound": "tensor", "flops": 2 * K * H * 2 * ffn},
        "mlp_down": {"bound": "tensor", "flops": 2 * K * ffn * H},
        "lower_mlp_gate_up": {"bound": "tensor", "flops": 2 * T * H * 2 * ffn},
        "lower_mlp_down": {"bound": "tensor", "flops": 2 * T * ffn * H},
    }


def kept_total(wl):
    """Total kept rows from the budgets (the same host rule as the library's planner:
    K_b = Q_b + min(D_b, max(0, budget_b - Q_b)))."""
    k = 0
    for n, q, b in zip(wl.lengths, wl.questions, wl.budgets):
        k += q + min(n - q, max(0, b - q))
    return k


def k_pad_rows(wl, spec):
    """Padded row count of the layers above the gate for a --k-pad value ('bucket': the
    kept total rounded up to a multiple of 256, the library's k_bucket), or None."""
    if spec is None:
        return None
    if spec == "bucket":
        return max(256, -(-kept_total(wl) // 256) * 256)
    return int(spec)


def config_dict(wl, args, world, k_pad=None):
    """The `config` of the JSON line, the same for both arms."""
    out = {"workload": wl.name, "batch": wl.batch,
            "tokens_per_request": list(wl.lengths) if wl.batch <= 8 else None,
            "question_tokens": list(wl.questions) if wl.batch <= 8 else None,
            "kept": kept_total(wl), "gated_layers": wl.n_layers,
            "lower_layers": args.lower_layers,
            "layer_body": "full (QK-norm, SwiGLU 6144)" if args.full_layers
            else "attention only",
            "hidden": wl.hidden, "heads": f"{wl.n_q_heads}q/{wl.n_kv_heads}kv x {wl.head_dim}",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (512 MiB write, outside the timing)",
            "launch": "cuda_graph" if args.launch == "graph" else "eager"}
    rows = k_pad_rows(wl, k_pad if k_pad is not None else getattr(args, "k_pad", None))
    if rows is not None:
        out["k_pad"] = rows
    return out


def topk_latency_floor(tg, dev, stream, flush, reps=20):
    """Average time of one tg_topk_compact call on a single 64-token request (32 prunable,
    32 kept): the select's fixed dependent chain (cluster launch, three radix passes and
    the compaction, each with a cluster-wide exchange) with almost no keys to count."""
    import torch
    z = torch.linspace(-1, 1, 64, device=dev)
    pr = torch.ones(64, dtype=torch.uint8, device=dev)
    pr[32:] = 0
    cu_h = torch.tensor([0, 64], dtype=torch.int32)
    ck_h = torch.tensor([0, 48], dtype=torch.int32)
    cu, ck = cu_h.to(dev), ck_h.to(dev)
    idx = torch.empty(48, dtype=torch.int32, device=dev)
    pos = torch.empty_like(idx)
    bias = torch.empty(48, dtype=torch.float32, device=dev)

    def call():
        tg.tg_topk_compact(z, pr, cu, cu_h, ck, ck_h, idx, pos, bias, stream=stream)
    for _ in range(3):
        call()
    ms = []
    for _ in range(reps):
        flush.fill_(1.0)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    return sorted(ms)[len(ms) // 2]


# ------------------------------------------------------------------ clocks (NVML)

class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU every ~20 ms in a thread."""

    def __init__(self, device_index):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, not a guess
            self.err = str(e)

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                active = [k for k, bit in names.items() if r & bit]
                self.samples.append((mhz, active))
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ our arm

def run_ours(args, rank, world):
    import torch
    out = measure(args, args.workload, rank, world, extras=True)
    subs = {}
    for name in [w for w in args.also.split(",") if w and w != args.workload]:
        torch.cuda.empty_cache()
        sub = measure(args, name, rank, world, extras=False)
        key = sub["config"]["workload"]
        if "k_pad" in sub["config"]:
            key += f"@k_pad{sub['config']['k_pad']}"
        subs[key] = {k: sub[k] for k in (
            "value", "unit", "ms_per_step", "steps", "warmup", "config", "e2e", "gpu_launches",
            "roofline", "rooflines", "stages", "clocks")}
    if subs:
        out["workloads"] = subs
    return out


def measure(args, wl_name, rank, world, extras):
    """One workload, timed as described at the top of this file.  With `extras`, also the
    gate backward kernels and the dense full-context reference."""
    import numpy as np
    import torch

    import learned_token_pruning_scoring_b200 as tg
    import synthetic_inputs as S

    dev = torch.device("cuda", torch.cuda.current_device())
    # "name@pad": the workload with the layers above the gate on a padded row count
    wl_name, _, pad_spec = wl_name.partition("@")
    pad_spec = pad_spec or args.k_pad
    wl = workload(wl_name)
    # replicas: rank r draws its own batch (seed offset), same weights
    wl = replica_workload(wl, rank, world)
    h = S.hidden_rows(wl)
    pr = S.prunable_mask(wl)
    gate = {k: v.to(dev) for k, v in S.gate_weights(wl).items()}
    def to_dev(d):
        return {k: (to_dev(v) if isinstance(v, dict) else v.to(dev) if torch.is_tensor(v) else v)
                for k, v in d.items()}

    layers = []
    for i in range(wl.n_layers):
        L = S.layer_weights(wl, i)
        if args.full_layers:
            L = dict(L, **S.layer_body_parts(wl, i))
        layers.append(to_dev(L))
    scores = S.drawn_scores(wl).to(dev) if wl.planted_cluster else None
    lower = None
    if args.lower_layers:
        lower_w = S.lower_layer_weights(wl, args.lower_layers)
        if args.full_layers:
            lower_w = [dict(L, **S.layer_body_parts(wl, i, lower=True))
                       for i, L in enumerate(lower_w)]
        lower = tg.FullContextLayers([to_dev(L) for L in lower_w],
                                     wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.rope_theta,
                                     device=dev)
    pipe = tg.GatedPrefill(gate, layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                           wl.rope_theta, device=dev, lower=lower)
    if args.rope_rows is not None:
        pipe.rope_rows = args.rope_rows == "on"
    if args.launch_overlap is not None:
        tg.tg_set_launch_overlap(args.launch_overlap == "on")
    if args.fuse_boundaries is not None:
        pipe.fuse_boundaries = args.fuse_boundaries == "on"
    P = pipe.plan(wl.lengths, wl.questions, wl.budgets, k_pad=k_pad_rows(wl, pad_spec))
    h_dev = h.to(dev)
    pr_dev = pr.to(dev)
    stream = torch.cuda.current_stream()

    def step(hd=None, prd=None):
        pipe.run(h_dev if hd is None else hd, pr_dev if prd is None else prd, scores=scores)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    status = tg.tg_status_read(pipe.status)
    if status:
        raise SystemExit(f"device status {status:#x} after warm-up")

    # Two CUDA graphs of the same step: a plain one for the headline timing, and one with
    # external timing events at every stage boundary for the per-stage breakdown (event
    # nodes between kernels cost a little time, so they stay out of the headline).
    use_graph = args.launch == "graph"
    marks = []

    def capture(with_marks, hd=None, prd=None):
        evs = []
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                cap = torch.cuda.current_stream()
                if with_marks:
                    e0 = torch.cuda.Event(enable_timing=True, external=True)
                    e0.record(cap)
                    evs.append(("start", e0))

                    def marker(name):
                        e = torch.cuda.Event(enable_timing=True, external=True)
                        e.record(cap)
                        evs.append((name, e))
                    pipe.marker = marker
                step(hd, prd)
                pipe.marker = None
        stream.wait_stream(side)
        return g, evs

    launches_before = tg.launch_count
    if use_graph:
        graph_plain, _ = capture(False)
        launches_per_step = tg.launch_count - launches_before
        graph_marked, marks = capture(True)
    else:
        graph_plain = graph_marked = None
        step()
        launches_per_step = tg.launch_count - launches_before
    torch.cuda.synchronize()

    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    per_stage = {}
    step_ms = []
    marked_ms = []

    def run_step_plain():
        flush.fill_(1.0)  # evict L2 (outside the step's events)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if use_graph:
            graph_plain.replay()
        else:
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e1))

    def run_step_marked():
        flush.fill_(1.0)
        if use_graph:
            graph_marked.replay()
            evs = marks
        else:
            evs = []
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            evs.append(("start", e0))

            def marker(name):
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                evs.append((name, e))
            pipe.marker = marker
            step()
            pipe.marker = None
        torch.cuda.synchronize()
        prev = evs[0][1]
        for name, e in evs[1:]:
            per_stage.setdefault(name, []).append(prev.elapsed_time(e))
            prev = e
        marked_ms.append(evs[0][1].elapsed_time(evs[-1][1]))

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            run_step_plain()
    torch.cuda.synchronize()
    gpu_launches = launches_per_step * args.steps
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    if world > 1:
        torch.distributed.barrier()
    # per-stage breakdown (second timed loop, same step with stage events)
    for _ in range(args.steps):
        run_step_marked()
    status = tg.tg_status_read(pipe.status)
    if status:
        raise SystemExit(f"device status {status:#x} after timed steps")

    tokens_per_step = wl.total_tokens
    value = whole_job_rate(tokens_per_step, world, args.steps, total_ms)

    # ---- end to end through the public API: host inputs in, result out, every step.
    # With graphs, two input buffers: step i+1's inputs cross the host link on a copy
    # stream while step i computes, and the result leaves through a staging buffer the
    # same way (how a server feeds back-to-back batches); the L2 flush stays inside the
    # loop.  Eagerly, the copies and the step run in series.
    h_pin = h.pin_memory()
    pr_pin = pr.pin_memory()
    x_host = torch.empty(P["x"].shape, dtype=P["x"].dtype).pin_memory()
    e2e_ms = []
    if use_graph and args.e2e_steps > 0:
        h_dev2, pr_dev2 = torch.empty_like(h_dev), torch.empty_like(pr_dev)
        graph_b, _ = capture(False, h_dev2, pr_dev2)
        bufs = [(h_dev, pr_dev, graph_plain), (h_dev2, pr_dev2, graph_b)]
        x_stage = [torch.empty_like(P["x"]), torch.empty_like(P["x"])]
        copy = torch.cuda.Stream()
        ev_in = [torch.cuda.Event(), torch.cuda.Event()]      # inputs of buffer b landed
        ev_done = [torch.cuda.Event(), torch.cuda.Event()]    # step on buffer b finished
        ev_out = [torch.cuda.Event(), torch.cuda.Event()]     # result of buffer b left

        def upload(b):
            with torch.cuda.stream(copy):
                bufs[b][0].copy_(h_pin, non_blocking=True)
                bufs[b][1].copy_(pr_pin, non_blocking=True)
            ev_in[b].record(copy)

        def run_pipelined(n):
            torch.cuda.synchronize()
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(copy)
            upload(0)
            for i in range(n):
                b = i & 1
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # staging buffer b has been read out
                flush.fill_(1.0)
                bufs[b][2].replay()
                x_stage[b].copy_(P["x"], non_blocking=True)
                ev_done[b].record(stream)
                if i + 1 < n:
                    if i >= 1:
                        copy.wait_event(ev_done[1 - b])  # step i-1 no longer reads it
                    upload(1 - b)
                copy.wait_event(ev_done[b])
                with torch.cuda.stream(copy):
                    x_host.copy_(x_stage[b], non_blocking=True)
                ev_out[b].record(copy)
            t1.record(copy)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        run_pipelined(2)  # warm-up of the copy path
        e2e_ms = [run_pipelined(args.e2e_steps)]
        e2e_steps_done = args.e2e_steps
    else:
        for i in range(args.e2e_steps + 1):
            flush.fill_(1.0)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            h_dev.copy_(h_pin, non_blocking=True)
            pr_dev.copy_(pr_pin, non_blocking=True)
            step()
            x_host.copy_(P["x"], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i:  # first one is a warm-up of the copy path
                e2e_ms.append(e0.elapsed_time(e1))
        e2e_steps_done = len(e2e_ms)
    e2e_total = max_over_ranks(sum(e2e_ms), world, dev)
    e2e_value = whole_job_rate(tokens_per_step, world, e2e_steps_done, e2e_total)
    h2d = h.numel() * h.element_size() + pr.numel() * pr.element_size()
    d2h = x_host.numel() * x_host.element_size()

    # ---- per-stage roofline
    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    work = stage_work(wl, [int(x) for x in P["ck_h"].tolist()],
                      S.FFN if args.full_layers else 0)
    topk_floor_ms = topk_latency_floor(tg, dev, stream, flush)
    stages = {}
    for name, ms_list in per_stage.items():
        n_launch = len(ms_list)
        avg_ms = sum(ms_list) / n_launch
        w = work.get(name, {})
        entry = {"launches": n_launch, "total_ms": sum(ms_list), "avg_ms": avg_ms}
        if w.get("bound") == "tensor" and "flops" in w:
            # kernels of a step of a few ms: the burst peak applies (the sustained figure
            # is a seconds-long loop under the power cap), reported beside it
            ach = w["flops"] / (avg_ms / 1e3) / 1e12
            entry.update(bound="tensor", achieved=ach, unit="TFLOP/s",
                         peak=peaks["bf16_tflops"], frac=ach / peaks["bf16_tflops"],
                         frac_of_sustained=ach / peaks["bf16_tflops_sustained"])
        elif name in ("topk_compact",) and "bytes" in w:
            # a few hundred KB: bound by the dependent chain of the select (three radix
            # passes and the compaction, each a cluster-wide exchange), not by HBM
            ach = w["bytes"] / (avg_ms / 1e3) / 1e9
            entry.update(bound="latency", achieved_gbs=ach, floor_ms=topk_floor_ms,
                         frac=topk_floor_ms / avg_ms if topk_floor_ms else None,
                         hbm_frac=ach / peaks["hbm_gbs"],
                         floor="the same kernel on one 64-token request: its fixed chain of "
                               "three radix passes and the compaction")
        elif "bytes" in w:
            ach = w["bytes"] / (avg_ms / 1e3) / 1e9
            entry.update(bound="hbm", achieved=ach, unit="GB/s", peak=peaks["hbm_gbs"],
                         frac=ach / peaks["hbm_gbs"])
        stages[name] = entry
    tot = sum(v["total_ms"] for v in stages.values())
    for v in stages.values():
        v["share"] = v["total_ms"] / tot if tot else None

    def roof(kernel):
        d = stages[kernel]
        return {"kernel": kernel, "bound": d.get("bound"), "achieved": d.get("achieved"),
                "peak": d.get("peak"), "unit": d.get("unit"), "frac": d.get("frac"),
                "traffic": load_traffic(kernel, wl.name),
                "peak_source": f"{peak_src}: burst bf16 for tensor-bound kernels (timed "
                               f"inside a step of a few ms), copy bandwidth for hbm",
                "sm_mhz": clocks.get("sm_mhz")}
    dom = max(stages, key=lambda k: stages[k]["total_ms"])
    roofline = roof(dom)
    rooflines = {k: roof(k) for k in ("attention", "gather", "gate_score", "qkv_rope_cache",
                                      "out_proj") if k in stages and k != dom}

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(wl, args, world, pad_spec),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps_done,
                "copies": "double-buffered: next step's H2D and this step's D2H overlap the "
                          "compute on a copy stream" if use_graph else "in series",
                "l2": "flushed before every step, inside the timed loop"},
        "gpu_launches": gpu_launches,
        "ms_per_step_with_stage_events": sum(marked_ms) / max(1, len(marked_ms)),
        "roofline": roofline,
        "rooflines": rooflines,
        "stages": {k: {kk: (round(vv, 5) if isinstance(vv, float) else vv)
                       for kk, vv in v.items()} for k, v in stages.items()},
        "clocks": clocks,
    }
    if not extras:
        return out
    if args.bias_grad_steps > 0 and int(P["K"]) > 0:
        out["bias_grad"] = bias_grad_timing(tg, wl, P, pipe, flush, stream,
                                            args.bias_grad_steps, peaks)
    if args.scorer_bwd_steps > 0 and int(P["K"]) > 0:
        out["scorer_bwd"] = scorer_bwd_timing(tg, wl, P, pipe, h_dev, pr_dev, flush, stream,
                                              args.scorer_bwd_steps, peaks)
    if args.dense_steps > 0:
        out["dense_reference"] = dense_reference(tg, wl, layers, h_dev, flush, stream,
                                                 args.dense_steps, peaks,
                                                 total_ms / args.steps)
    return out


def bias_grad_timing(tg, wl, P, pipe, flush, stream, steps, peaks):
    """The attention backward w.r.t. the gate (key bias, gains, temperature scale) on the
    last gated layer's Q and compacted K/V of the step just run, with a seeded dO: CUDA
    events around each call (its four launches), L2 flushed before each."""
    import torch
    nq = wl.n_q_heads * wl.head_dim
    L = pipe.layers[-1]
    q = P["qkv"][:, :nq]
    ck, cv = P["caches"][-1]
    K = int(P["K"])
    dev = q.device
    lse = torch.empty((wl.n_q_heads, K), dtype=torch.float32, device=dev)
    o = tg.tg_gated_attention(q, ck, cv, P["ck"], P["ck_h"], wl.n_q_heads, wl.n_kv_heads,
                              P["kept_pos"], P["kept_bias"], L.gamma, L.beta, lse=lse)
    g = torch.Generator(device="cpu").manual_seed(17)
    d_o = torch.randn((K, nq), generator=g).to(torch.bfloat16).to(dev)
    d_bias = torch.empty(K, dtype=torch.float32, device=dev)
    d_gamma = torch.empty(wl.n_q_heads, dtype=torch.float32, device=dev)
    d_beta = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, tg.tg_gated_attention_bias_grad_workspace_size(
        P["ck_h"], wl.n_q_heads, wl.n_kv_heads)), dtype=torch.uint8, device=dev)

    def call():
        tg.tg_gated_attention_bias_grad(q, ck, cv, o, d_o, lse, P["ck"], P["ck_h"],
                                        wl.n_q_heads, wl.n_kv_heads, P["kept_pos"],
                                        P["kept_bias"], L.gamma, L.beta, d_bias=d_bias,
                                        d_gamma=d_gamma, d_beta=d_beta, workspace=ws,
                                        status=pipe.status)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.fill_(1.0)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    status = tg.tg_status_read(pipe.status)
    if status:
        raise SystemExit(f"device status {status:#x} in the attention backward")
    avg = sum(ms) / len(ms)
    Ks = [int(P["ck_h"][b + 1] - P["ck_h"][b]) for b in range(wl.batch)]
    flops = 4 * wl.head_dim * wl.n_q_heads * sum(k * (k + 1) // 2 for k in Ks)
    tf = flops / (avg / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"what": "d kept_bias, d gamma, d beta of the last gated layer's attention, "
                    "seeded dO (preparation + tcgen05 kernel + two reductions)",
            "kept": K, "calls": steps, "avg_ms": avg, "achieved": tf, "unit": "TFLOP/s",
            "peak": peak, "frac": tf / peak,
            "flops_counted": "S^T = K Q^T and dP^T = V dO^T over the causal pairs"}


def scorer_bwd_timing(tg, wl, P, pipe, h_dev, pr_dev, flush, stream, steps, peaks):
    """The scorer's backward (ds, dW1, dw2, d norm_w) from a seeded d kept_bias on the kept
    set of the step just run: CUDA events around each call, L2 flushed before each.  Its
    work is the scorer GEMM twice (the recompute and the weight gradient, 2THF flops
    each) with h streamed twice and r*du written and read once."""
    import torch
    dev = h_dev.device
    K = int(P["K"])
    g = torch.Generator(device="cpu").manual_seed(19)
    dkb = torch.randn(K, generator=g).to(dev)
    W1, w2, nw = pipe.gate["W1"], pipe.gate["w2"], pipe.gate.get("norm_w")
    T, H = h_dev.shape
    F = W1.shape[0]
    ds = torch.empty(T, dtype=torch.float32, device=dev)
    dW1 = torch.empty((F, H), dtype=torch.float32, device=dev)
    dw2 = torch.empty(F, dtype=torch.float32, device=dev)
    dnw = torch.empty(H, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, tg.tg_gate_score_backward_workspace_size(T, H, F, wl.batch)),
                     dtype=torch.uint8, device=dev)

    def call():
        tg.tg_gate_score_backward(h_dev, W1, w2, P["s"], P["cu"], P["cu_h"], pr_dev, P["ck"],
                                  P["ck_h"], P["kept_idx"], dkb, norm_w=nw, ds_out=ds, dW1=dW1,
                                  dnorm_w=dnw, dw2=dw2, workspace=ws, status=pipe.status)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.fill_(1.0)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    status = tg.tg_status_read(pipe.status)
    if status:
        raise SystemExit(f"device status {status:#x} in the scorer backward")
    avg = sum(ms) / len(ms)
    flops = 4 * T * H * F
    nbytes = 2 * (2 * T * H) + 2 * (2 * T * F) + 2 * F * H
    tf = flops / (avg / 1e3) / 1e12
    gbs = nbytes / (avg / 1e3) / 1e9
    floor_ms = max(flops / (peaks["bf16_tflops"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    return {"what": "ds, dW1, dw2, d norm_w of the scorer from a seeded d kept_bias "
                    "(ds kernels + scorer GEMM with gradient epilogue + weight-gradient "
                    "GEMM + reductions)",
            "tokens": T, "calls": steps, "avg_ms": avg, "tflops": tf, "gbs": gbs,
            "floor_ms": floor_ms, "frac_of_floor": floor_ms / avg,
            "counted": "4THF flops; h read twice, r*du written and read, W1 once"}


def dense_reference(tg, wl, layers, h_dev, flush, stream, steps, peaks, gated_ms):
    """The same layer stack over every token (K = N, gamma = 0, tau = 1, no gate): the
    GPU's own full-context prefill on the same kernels, timed like the gated step
    (L2 flushed before each step, CUDA events on the stream, eager launches)."""
    import torch
    full = tg.FullContextLayers(layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                                wl.rope_theta, device=h_dev.device)
    full.plan(wl.lengths, wl.hidden)
    for _ in range(2):
        full.run(h_dev)
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.fill_(1.0)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        full.run(h_dev)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    # one step with an event after every launch, for the attention kernel's own time
    evs = []
    flush.fill_(1.0)
    e = torch.cuda.Event(enable_timing=True)
    e.record(stream)
    evs.append(("start", e))

    def marker(name):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        evs.append((name, ev))
    full.marker = marker
    full.run(h_dev)
    full.marker = None
    torch.cuda.synchronize()
    status = tg.tg_status_read(full.status)
    if status:
        raise SystemExit(f"device status {status:#x} in the full-context reference")
    attn = [p[1].elapsed_time(c[1]) for p, c in zip(evs, evs[1:]) if c[0] == "attention"]
    d_ms = sum(ms) / len(ms)
    pairs = sum(n * (n + 1) // 2 for n in wl.lengths)
    attn_ms = sum(attn) / len(attn) if attn else None
    tf = 4 * wl.head_dim * wl.n_q_heads * pairs / (attn_ms / 1e3) / 1e12 if attn else None
    peak = peaks["bf16_tflops"]
    return {"what": "same layers over all tokens: K = N, gamma = 0, tau = 1, no gate",
            "kept": wl.total_tokens, "layers": len(layers), "steps": steps,
            "ms_per_step": d_ms, "tokens_per_s": wl.total_tokens / (d_ms / 1e3),
            "gated_speedup": d_ms / gated_ms,
            "attention": {"avg_ms": attn_ms, "achieved": tf, "unit": "TFLOP/s",
                          "peak": peak, "frac": tf / peak if tf else None,
                          "frac_of_sustained": (tf / peaks["bf16_tflops_sustained"]
                                                if tf else None)}}


def load_traffic(kernel, workload_name):
    """Per-launch DRAM bytes from a committed ncu summary, if one exists for this kernel
    and was taken on the kernel source as it is now (sha256 match); else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            e = json.load(f)[workload_name][kernel]
        with open(os.path.join(ROOT, e["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != e["source_sha256"]:
                return None
        return int(e["bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ CPU oracle arm

def oracle_sample(wl, n_layers_sample):
    """Time the oracle on a bounded sample of the workload and scale to one full step.

    Sample: the whole gate (scorer + sequence RMSNorm + selection + gather) over all N
    tokens, then `n_layers_sample` of the gated layers; the per-layer time is scaled to
    the workload's layer count."""
    import numpy as np

    import oracle as O
    import synthetic_inputs as S
    h = S.hidden_rows(wl)
    pr = S.prunable_mask(wl)
    gate = S.gate_weights(wl)
    t0 = time.perf_counter()
    s = O.gate_score(h, gate["norm_w"], gate["W1"], gate["w2"])
    if wl.planted_cluster:
        s = O.as_f64(S.drawn_scores(wl))
    z, _ = O.sequence_rmsnorm(s, wl.cu_seqlens(), pr)
    ck = O.kept_counts(pr, wl.cu_seqlens(), wl.budgets)
    idx, pos, kb = O.select_topk(z.astype(np.float32), pr, wl.cu_seqlens(), ck)
    x = O.gather_rows(h, idx)
    t1 = time.perf_counter()
    nl = max(1, min(n_layers_sample, wl.n_layers))
    for i in range(nl):
        L = S.layer_weights(wl, i)
        x, _, _, _ = O.gated_layer(x, L["Wqkv"], L["Wo"], L["gamma"], L["beta"], ck, pos, kb,
                                   wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.rope_theta)
    t2 = time.perf_counter()
    full_s = (t1 - t0) + (t2 - t1) / nl * wl.n_layers
    return {"seconds_per_step": full_s, "measured_s": t2 - t0, "layers_run": nl}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, n_layers_sample):
    r = oracle_sample(wl, n_layers_sample)
    return {"value": wl.total_tokens / r["seconds_per_step"], "unit": UNIT,
            "cores": blas_threads(), "kind": "oracle",
            "sample": (f"float64 NumPy oracle: gate over all {wl.total_tokens} tokens + "
                       f"{r['layers_run']} of {wl.n_layers} gated layers "
                       f"({r['measured_s']:.1f} s measured), layer time scaled to "
                       f"{wl.n_layers} layers")}


def run_reference(args, rank, world):
    """The oracle on the host cores.  Each timed step is a bounded sample of the workload's
    step: the whole gate over all N tokens plus ONE of the gated layers.  `steps` and
    `ms_per_step` are the samples actually timed and their measured time; `value` is the
    workload's tokens over the full step's time extrapolated from the sample (the gate's
    time plus the one layer's time times the layer count), marked as such."""
    wl = workload(args.workload)
    for _ in range(args.warmup):
        oracle_sample(wl, 1)
    full, measured = [], []
    for _ in range(args.steps):
        r = oracle_sample(wl, 1)
        full.append(r["seconds_per_step"])
        measured.append(r["measured_s"])
    value = wl.total_tokens * len(full) / sum(full)
    cores = blas_threads()
    sample = (f"per step: gate over all {wl.total_tokens} tokens + 1 of {wl.n_layers} gated "
              f"layers (measured), the full step's time extrapolated from that one layer")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": len(measured), "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(measured) / len(measured),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(wl, args, world),
        "extrapolated_from_layers": 1,
        "ms_per_full_step_extrapolated": 1e3 * sum(full) / len(full),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        out = run_ours(args, rank, world)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(workload(args.workload), args.cpu_sample_layers)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
