"""Benchmark: Switch-layer forward tokens/s on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one full forward pass of the layer (router logits, softmax/argmax,
dispatch scan + aux loss, gather, expert GEMM1, expert GEMM2 + combine) over
one batch of seeded synthetic tokens already resident in HBM.  Default
workload: the many-expert layer, the largest of the five that fits one GPU
(T=65536 tokens, d=1024, d_ff=2048, N=2048 experts, capacity factor 1.0, C=32,
17 GB of bf16 expert weights, fp32 router); the other four are reachable with
--workload.

Multi-GPU (torchrun, one rank per GPU): one global batch, each rank holding a
contiguous range of T tokens and all weights; one NCCL all-gather of
per-expert counts and sums of p per step gives every rank the whole batch's
positions, capacity and aux loss (weak scaling: per-GPU work fixed).  The
timed region is bracketed by barriers and the max over ranks is reported.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only): every
token routed, the expert FFNs of a bounded sample of experts, scaled to the
whole batch.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from sparse_mixture_experts_argmax_b200 import dist as swl_dist  # noqa: E402

DEFAULT_WORKLOAD = "many_T65536_d1024_N2048"
METRIC = "Switch-layer fwd tokens/sec on 1 B200; expert-GEMM % of bf16 tensor peak"
L2_FLUSH_BYTES = 256 << 20
E2E_STREAMS = 3          # end-to-end steps in flight (each on its own stream and workspace)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_init():
    info = swl_dist.init("nccl")
    return info.world_size, info.rank, info.local_rank


def _barrier(ws):
    swl_dist.barrier(swl_dist.rank_info())


def _max_over_ranks(ws, v: float) -> float:
    return swl_dist.max_over_ranks(swl_dist.rank_info(), v)


def _traffic_entry(kernel: str, workload: str):
    """Per-launch DRAM bytes of ``kernel`` from a committed ncu capture, or None
    if absent or if the kernel's source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel, {}).get(workload)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if h != ent.get("source_sha256"):
        return None
    return float(ent["dram_bytes_per_launch"])


# ----------------------------------------------------------------------------- GPU arm
def algorithmic_bytes(T, d, d_ff, N, elem, touched, K_kept):
    """(expert FFN launch bytes, whole-layer bytes) that the work needs at least.

    FFN (both GEMMs): the weights and biases of every touched expert once,
    (2*d*d_ff + d + d_ff) * elem each, and per kept token its packed input row
    in and its output row out, 2*d*elem, plus its destination index and gate
    (8 bytes).  The hidden rows between the two GEMMs are an intermediate, not
    algorithmic traffic.  Layer: the router (x, fp32 W_r and bias), the dispatch
    (kept rows into the packed buffer, zero rows of dropped tokens, expert index
    / gate / position per token; the aux loss is negligible) and the FFN above."""
    w_bytes = touched * (2 * d * d_ff + d + d_ff) * elem
    act_bytes = K_kept * 2 * d * elem + K_kept * 8
    ffn_bytes = w_bytes + act_bytes
    layer_bytes = (T * d * elem + N * d * 4 + N * 4 + 2 * K_kept * d * elem +
                   (T - K_kept) * d * elem + 3 * 4 * T + ffn_bytes)
    return ffn_bytes, layer_bytes


def run_gpu(args):
    import sparse_mixture_experts_argmax_b200 as swl

    ws_n, rank, local = _dist_init()
    dev = torch.device("cuda", local)
    spec = synth.WORKLOADS[args.workload]
    T, d, d_ff, N, cf = spec.T, spec.d, spec.d_ff, spec.N, spec.cf
    # set before the workspace is sized (the two routers need different scratch)
    swl.switch_layer_set_router_mode(swl.SWL_ROUTER_FFMA if args.router == "ffma"
                                     else swl.SWL_ROUTER_TENSOR)
    router_desc = ("fp32 FFMA" if args.router == "ffma" or spec.dtype != "bf16" else
                   "fp32 on tensor cores (exact three-piece bf16 split of W_r, fp32 accumulation)")
    redraws = synth.load_gap_redraws(spec.name) if rank == 0 else {}
    inputs = synth.make_layer_inputs(spec, seed=rank, device=dev, redraws=redraws)
    act = inputs["x"].dtype
    work = swl.alloc_workspace(T, d, d_ff, N, act, cf, device=dev)
    outs = swl.alloc_outputs(T, d, act, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    S = swl.SWL_NUM_STAGES

    def step(events=None):
        swl.switch_layer_forward(inputs["x"], inputs["W_r"], inputs["W1"], inputs["b1"],
                                 inputs["W2"], inputs["b2"], cf, outs["out"],
                                 outs["expert_idx"], outs["gate"], outs["pos_in_expert"],
                                 outs["aux_loss"], b_r=inputs["b_r"], workspace=work,
                                 stream=stream, stage_events=events)

    launches_per_forward = 0          # kernels one forward enqueues (library's own count)
    for _ in range(args.warmup):
        flush.fill_(1)
        c0 = swl.switch_layer_launch_count()
        step()
        launches_per_forward = swl.switch_layer_launch_count() - c0
    torch.cuda.synchronize()
    if swl.switch_layer_device_status(work, stream) != 0:
        raise RuntimeError("device status not OK after warm-up")

    # One forward per step is replayed from a CUDA graph captured from the C-ABI
    # call (its six launches, programmatic-dependent edges included), so the host
    # enqueue cost of a step never leaves the GPU idle inside the timed region.
    S_EV = [torch.cuda.Event(enable_timing=True) for _ in range(S + 1)]
    for e in S_EV:
        e.record(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    graph_timed = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            swl.switch_layer_forward(inputs["x"], inputs["W_r"], inputs["W1"], inputs["b1"],
                                     inputs["W2"], inputs["b2"], cf, outs["out"],
                                     outs["expert_idx"], outs["gate"], outs["pos_in_expert"],
                                     outs["aux_loss"], b_r=inputs["b_r"], workspace=work,
                                     stream=cap)
        with torch.cuda.graph(graph_timed, stream=cap):
            swl.switch_layer_forward(inputs["x"], inputs["W_r"], inputs["W1"], inputs["b1"],
                                     inputs["W2"], inputs["b2"], cf, outs["out"],
                                     outs["expert_idx"], outs["gate"], outs["pos_in_expert"],
                                     outs["aux_loss"], b_r=inputs["b_r"], workspace=work,
                                     stream=cap, stage_events=S_EV)
    stream.wait_stream(cap)
    for _ in range(args.warmup):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps, L2 flushed between steps (outside the step events)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    for a, b in step_ev:
        a.record(stream)            # create the CUDA events before timing
        b.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    _barrier(ws_n)
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        step_ev[k][0].record(stream)
        graph.replay()
        step_ev[k][1].record(stream)
    torch.cuda.synchronize()
    launches = launches_per_forward * args.steps      # kernels in the replayed graph
    _barrier(ws_n)
    clk = clocks.stop()
    step_ms = np.array([a.elapsed_time(b) for a, b in step_ev])
    total_ms = _max_over_ranks(ws_n, float(step_ms.sum()))
    ms_per_step = total_ms / args.steps
    value = swl_dist.aggregate_throughput(swl_dist.rank_info(), T, args.steps, total_ms)
    if swl.switch_layer_device_status(work, stream) != 0:
        raise RuntimeError("device status not OK after the timed steps")

    # ---- per-kernel times: K more steps replaying the graph that records an
    # event between every two stages
    _barrier(ws_n)
    rows = []
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        graph_timed.replay()
        torch.cuda.synchronize()
        rows.append([S_EV[i].elapsed_time(S_EV[i + 1]) for i in range(S)])
    _barrier(ws_n)
    stage_ms = np.array(rows)
    del graph, graph_timed

    # ---- end to end through the host-I/O entry point (pinned host x and outputs).
    # E2E_STREAMS streams, each with its own workspace, take the steps in turn:
    # a step's copy in, forward and copy out are serial on its stream, so with
    # three steps in flight the host-to-device engine, the SMs and the
    # device-to-host engine each work on a different step.  Every step copies its
    # x in and its outputs back inside the timed region, into host buffers of its
    # own (up to 33 sets, reused in order), and every step's outputs are compared
    # with the device-resident run afterwards.  The expert weights (larger than
    # L2) stream from HBM in every step, so no L2 flush is interposed.
    NS = E2E_STREAMS
    e2e_streams = [stream] + [torch.cuda.Stream(dev) for _ in range(NS - 1)]
    work_h = [swl.alloc_workspace(T, d, d_ff, N, act, cf, host_io=True, device=dev)
              for _ in range(NS)]
    xh = [inputs["x"].cpu().pin_memory() for _ in range(NS)]
    # a multiple of NS: each output set stays on one stream
    n_sets = min(NS * 11, (args.steps + NS - 1) // NS * NS)

    def out_set():
        return [torch.empty((T, d), dtype=act).pin_memory(),
                torch.empty(T, dtype=torch.int32).pin_memory(),
                torch.empty(T, dtype=torch.float32).pin_memory(),
                torch.empty(T, dtype=torch.int32).pin_memory(),
                torch.empty(1, dtype=torch.float32).pin_memory()]

    oh = [out_set() for _ in range(max(NS, n_sets))]

    def step_e2e(k):
        j = k % NS
        swl.switch_layer_forward_host_io(xh[j], inputs["W_r"], inputs["W1"], inputs["b1"],
                                         inputs["W2"], inputs["b2"], cf, *oh[k % len(oh)],
                                         b_r=inputs["b_r"], workspace=work_h[j],
                                         stream=e2e_streams[j])

    for k in range(max(NS, args.warmup)):
        step_e2e(k)
    torch.cuda.synchronize()
    for o in oh:
        o[0].fill_(0)
        o[1].fill_(-1)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws_n)
    torch.cuda.synchronize()
    e_start.record(e2e_streams[0])
    for st in e2e_streams[1:]:
        st.wait_event(e_start)
    for k in range(args.steps):
        step_e2e(k)
    for st in e2e_streams[1:]:
        ev_side = torch.cuda.Event()
        ev_side.record(st)
        e2e_streams[0].wait_event(ev_side)
    e_end.record(e2e_streams[0])
    e_end.synchronize()             # every step's result is on the host
    _barrier(ws_n)
    e2e_total = _max_over_ranks(ws_n, float(e_start.elapsed_time(e_end)))
    e2e_value = ws_n * T * args.steps / (e2e_total / 1e3)
    for j in range(NS):
        if swl.switch_layer_device_status(work_h[j], e2e_streams[j]) != 0:
            raise RuntimeError("device status not OK after the end-to-end steps (stream %d)" % j)
    ref_host = [outs[k].cpu() for k in ("out", "expert_idx", "gate", "pos_in_expert",
                                        "aux_loss")]
    for k in range(max(0, args.steps - len(oh)), args.steps):
        if not all(torch.equal(a, b) for a, b in zip(oh[k % len(oh)], ref_host)):
            raise RuntimeError("end-to-end outputs of step %d differ from the device-resident "
                               "run" % k)
    elem = 2 if act == torch.bfloat16 else 4
    h2d = T * d * elem
    d2h = T * d * elem + 3 * 4 * T + 4

    # ---- roofline of the dominant kernel (algorithmic bytes / launch duration)
    e_idx = outs["expert_idx"].long()
    kept = outs["pos_in_expert"].long() < swl.switch_layer_capacity(T, N, cf)
    counts = torch.bincount(e_idx, minlength=N)
    touched = int((counts > 0).sum())
    K_kept = int(kept.sum())
    avg_stage = stage_ms.mean(axis=0)
    names = [swl.switch_layer_stage_name(i) for i in range(S)]
    # stages that launch no kernel for this shape report 0, not the event gap
    plan = swl.switch_layer_describe_plan(T, d, d_ff, N, swl.dtype_code(act), cf,
                                          torch.cuda.get_device_properties(dev).multi_processor_count)
    if plan["softmax"] == "fused":
        avg_stage[names.index("router_softmax")] = 0.0
    if plan["dispatch"] == "fused":
        avg_stage[names.index("dispatch_gather")] = 0.0
    ffn_bytes, layer_bytes = algorithmic_bytes(T, d, d_ff, N, elem, touched, K_kept)
    dom = "expert_ffn"
    dom_s = avg_stage[names.index(dom)] / 1e3
    peaks = _peaks()
    achieved = ffn_bytes / dom_s / 1e9
    traffic = _traffic_entry(dom, spec.name)
    gemm_flops = 4.0 * K_kept * d * d_ff
    tensor_frac = gemm_flops / dom_s / (peaks["bf16_tflops"] * 1e12)
    # whole layer: the slower of its GEMM FLOPs at the bf16 peak and its bytes at
    # the HBM peak, against the measured step time
    layer_floor_s = max(layer_bytes / (peaks["hbm_gbs"] * 1e9),
                        (gemm_flops + 2.0 * T * d * N) / (peaks["bf16_tflops"] * 1e12))

    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": ws_n,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if act == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; x ~ N(0,1), T5 truncated-normal init s=0.1)",
        "config": {
            "workload": spec.name, "T": T, "d": d, "d_ff": d_ff, "N": N,
            "capacity_factor": cf, "capacity": swl.switch_layer_capacity(T, N, cf),
            "router": router_desc, "parallelism": "single GPU",
            "l2": "flushed between timed steps (256 MiB write, outside the step events); "
                  "expert weights %.0f MB > 126 MB L2" % (2 * N * d * d_ff * elem / 1e6),
        },
        "stages_us": {n: round(float(v) * 1e3, 2) for n, v in zip(names, avg_stage)},
        "stages_note": "per-stage CUDA events in a second pass of K graph replays (the events "
                       "split the programmatic-launch overlap); value uses whole-step events "
                       "around replays of the forward's CUDA graph",
        "roofline": {
            "kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "algorithmic_bytes": ffn_bytes, "peak_source": peaks["source"] + " (burst copy)",
        },
        "layer_roofline": {
            "bytes": layer_bytes, "flops": gemm_flops + 2.0 * T * d * N,
            "floor_us": layer_floor_s * 1e6, "step_us": ms_per_step * 1e3,
            "frac": layer_floor_s / (ms_per_step / 1e3),
            "note": "the slower of the layer's FLOPs at the measured bf16 peak and its bytes at "
                    "the measured HBM copy bandwidth, over the measured step time",
        },
        "expert_gemm_tensor_frac": {
            "value": tensor_frac, "flops_per_step": gemm_flops,
            "peak_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"],
            "note": "GEMM1+GEMM2 kept-token FLOPs / the expert-FFN time / dense bf16 peak; the "
                    "stage is bound by streaming expert weights, see roofline",
        },
        "routing": {"experts_touched": touched, "kept_tokens": K_kept,
                    "dropped_tokens": T - K_kept, "max_load": int(counts.max()),
                    "aux_loss": float(outs["aux_loss"][0])},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "switch_layer_forward_host_io per step (pinned host x in, out / "
                        "expert_idx / gate / pos_in_expert / aux_loss back), alternate steps on "
                        "three streams so copies overlap the other steps' kernels"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(spec, inputs, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(res), flush=True)
    swl_dist.finalize(swl_dist.rank_info())


VARIANTS = ("top2", "ntlb", "geglu", "jitter", "backward")


def run_variant(args):
    """One JSON line for a layer variant on one GPU: the top-2 layer, No-Token-
    Left-Behind, GEGLU experts, router input jitter (forward passes), or the
    backward pass of the top-1 layer.  Same method as the default line (graph
    replay, L2 flushed between steps, device events, clocks sampled), with the
    variant's own algorithmic bytes (forward) or FLOPs (backward)."""
    import dataclasses
    import sparse_mixture_experts_argmax_b200 as swl

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--variant runs on one GPU")
    dev = torch.device("cuda", 0)
    base = synth.WORKLOADS[args.workload]
    v = args.variant
    spec = dataclasses.replace(base, name=base.name + "_geglu", activation="geglu") \
        if v == "geglu" else base
    T, d, d_ff, N, cf = spec.T, spec.d, spec.d_ff, spec.N, spec.cf
    inputs = synth.make_layer_inputs(spec, device=dev,
                                     redraws=synth.load_gap_redraws(base.name))
    act = inputs["x"].dtype
    elem = 2 if act == torch.bfloat16 else 4
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    noise = synth.router_noise(spec, device=dev) if v == "jitter" else None
    if v == "top2":
        ws = swl.alloc_workspace(T, d, d_ff, N, act, cf, device=dev, top2=True)
        fn = lambda st: swl.forward_top2(inputs, cf, True, workspace=ws, stream=st, check=False)
    elif v == "ntlb":
        ws = swl.alloc_workspace(T, d, d_ff, N, act, cf, device=dev, ntlb=True)
        fn = lambda st: swl.forward_ntlb(inputs, cf, workspace=ws, stream=st, check=False)
    elif v in ("geglu", "jitter"):
        var = swl.make_variant(1, True, "geglu" if v == "geglu" else "relu", noise)
        ws = torch.empty(max(256, swl.switch_layer_variant_workspace_size(
            T, d, d_ff, N, swl.dtype_code(act), cf, var)), dtype=torch.uint8, device=dev)
        act_name = "geglu" if v == "geglu" else "relu"
        fn = lambda st: swl.forward_variant(inputs, cf, 1, True, act_name, noise, workspace=ws,
                                            stream=st, check=False)
    else:   # backward of the top-1 layer, after one forward
        ws = swl.alloc_workspace(T, d, d_ff, N, act, cf, device=dev)
        fwd = swl.forward(inputs, cf, workspace=ws)
        dout = synth.draw((0, spec.name, "dout"), (T, d), "normal", 1.0, spec.dtype, dev)
        fn = lambda st: swl.backward(inputs, cf, fwd, ws, dout, daux=1.0, stream=st, check=False)

    launches = 0
    for _ in range(args.warmup):
        flush.fill_(1)
        c0 = swl.switch_layer_launch_count()
        out = fn(stream)
        launches = swl.switch_layer_launch_count() - c0
    torch.cuda.synchronize()
    if swl.switch_layer_device_status(ws, stream) != 0:
        raise RuntimeError("device status not OK after warm-up")
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            gout = fn(cap)
    stream.wait_stream(cap)
    for _ in range(args.warmup):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        ev[k][0].record(stream)
        graph.replay()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if swl.switch_layer_device_status(ws, stream) != 0:
        raise RuntimeError("device status not OK after the timed steps")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    peaks = _peaks()
    C1 = swl.switch_layer_capacity(T, N, cf)
    if v == "backward":
        kept = (fwd["pos_in_expert"].long() < C1)
        K = int(kept.sum())
        # dW1, dW2 (K d d_ff each), dh and dx through both matrices (K d d_ff each),
        # router: dW_r and dx (T d N each), 2 flop per multiply-add
        flops = 2.0 * (4.0 * K * d * d_ff + 2.0 * T * d * N)
        if act == torch.bfloat16:
            # the expert GEMMs run on the tensor cores (bf16 operands, fp32 accumulation)
            peak, bound = peaks["bf16_tflops"], "tensor"
            src = peaks["source"] + " bf16 (burst); the router's fp32 part runs on the CUDA cores"
        else:
            peak = 2.0 * 128 * torch.cuda.get_device_properties(dev).multi_processor_count * \
                1.965e9 / 1e12
            bound, src = "alu", "fp32 FMA issue: 148 SMs x 128 lanes x 2 flop x 1965 MHz"
        roof = {"kernel": "whole backward", "bound": bound, "achieved": flops / (ms / 1e3) / 1e12,
                "peak": peak, "unit": "TFLOP/s", "frac": flops / (ms / 1e3) / 1e12 / peak,
                "traffic": None, "algorithmic_flops": flops, "peak_source": src}
        routing = {"kept_tokens": K}
    else:
        e = gout["expert_idx"].long().reshape(T, -1)
        pos = gout["pos_in_expert"].long().reshape(T, -1)
        if v == "top2":
            Ck = swl.switch_layer_capacity(2 * T, N, cf)
            keptm = pos < Ck
        elif v == "ntlb":
            keptm = torch.stack([pos[:, 0] < C1, (pos[:, 0] >= C1) & (pos[:, 1] >= 0) &
                                 (pos[:, 1] < C1)], dim=1)
        else:
            keptm = pos < C1
        K = int(keptm.sum())
        touched = int(torch.unique(e[keptm]).numel())
        w_per = (3 if v == "geglu" else 2) * d * d_ff + d + (2 if v == "geglu" else 1) * d_ff
        ffn_bytes = touched * w_per * elem + K * (2 * d * elem + 8)
        layer_bytes = (T * d * elem + N * d * 4 + T * d * elem + (4 * T * d if noise is not None
                                                                   else 0) + ffn_bytes)
        achieved = layer_bytes / (ms / 1e3) / 1e9
        roof = {"kernel": "whole layer", "bound": "hbm", "achieved": achieved,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "traffic": None, "algorithmic_bytes": layer_bytes,
                "peak_source": peaks["source"] + " (burst copy)"}
        routing = {"experts_touched": touched, "kept_assignments": K}
    res = {
        "metric": "Switch-layer %s tokens/sec on 1 B200" % (
            "backward" if v == "backward" else v + " variant fwd"),
        "value": T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if act == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; x ~ N(0,1), T5 truncated-normal init s=0.1)",
        "config": {"workload": spec.name, "variant": v, "T": T, "d": d, "d_ff": d_ff, "N": N,
                   "capacity_factor": cf,
                   "l2": "flushed between timed steps (256 MiB write, outside the step events)"},
        "roofline": roof, "routing": routing, "gpu_launches": int(launches * args.steps),
        "clocks": clk,
    }
    print(json.dumps(res), flush=True)


def run_gpu_sharded(args):
    """N > 1 ranks: ONE global batch of N x T tokens, rank g holding the g-th
    contiguous range of T tokens (rank 0 the workload's own seeded tokens, rank
    g > 0 tokens drawn with seed g) and a full copy of the weights (seed 0).
    Positions, capacity C = ceil(cf * N * T / experts) and the aux loss are
    those of the whole batch: a step is the library's shard step 1 (routing and
    this rank's exchange record), an NCCL all-gather of the records (12 bytes
    per expert and rank), and shard step 3 (offsets of earlier ranks, dispatch,
    expert FFN).  Per-GPU work is fixed as N grows: weak scaling."""
    import sparse_mixture_experts_argmax_b200 as swl

    ws_n, rank, local = _dist_init()
    info = swl_dist.rank_info()
    dev = torch.device("cuda", local)
    spec = synth.WORKLOADS[args.workload]
    T, d, d_ff, N, cf = spec.T, spec.d, spec.d_ff, spec.N, spec.cf
    T_total = ws_n * T
    swl.switch_layer_set_router_mode(swl.SWL_ROUTER_FFMA if args.router == "ffma"
                                     else swl.SWL_ROUTER_TENSOR)
    inputs = synth.make_layer_inputs(spec, seed=0, device=dev,
                                     redraws=synth.load_gap_redraws(spec.name))
    if rank > 0:
        inputs["x"] = synth.make_x(spec, seed=rank, device=dev)
    act = inputs["x"].dtype
    elem = 2 if act == torch.bfloat16 else 4
    work = swl.alloc_workspace(T, d, d_ff, N, act, cf, device=dev)
    outs = swl.alloc_outputs(T, d, act, device=dev)
    record = torch.empty(swl.switch_layer_shard_record_bytes(N), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(x, ev=None):
        swl.switch_layer_forward_shard_begin(x, inputs["W_r"], cf, T_total, outs["expert_idx"],
                                             outs["gate"], outs["pos_in_expert"], record, d_ff,
                                             b_r=inputs["b_r"], workspace=work, stream=stream)
        gathered = swl_dist.exchange_records(info, record)
        if ev is not None:
            ev.record(stream)
        swl.switch_layer_forward_shard_end(x, inputs["W1"], inputs["b1"], inputs["W2"],
                                           inputs["b2"], cf, T_total, rank, ws_n, gathered,
                                           outs["out"], outs["expert_idx"], outs["gate"],
                                           outs["pos_in_expert"], outs["aux_loss"],
                                           workspace=work, stream=stream)

    launches_per_step = 0
    for _ in range(args.warmup):
        flush.fill_(1)
        c0 = swl.switch_layer_launch_count()
        step(inputs["x"])
        launches_per_step = swl.switch_layer_launch_count() - c0
    torch.cuda.synchronize()
    if swl.switch_layer_device_status(work, stream) != 0:
        raise RuntimeError("device status not OK after warm-up")

    # ---- timed region: K steps, L2 flushed between steps (outside the step events)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for e3 in ev:
        for e in e3:
            e.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    _barrier(ws_n)
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        ev[k][0].record(stream)
        step(inputs["x"], ev[k][1])
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    _barrier(ws_n)
    clk = clocks.stop()
    step_ms = np.array([a.elapsed_time(c) for a, _, c in ev])
    end_ms = np.array([b.elapsed_time(c) for _, b, c in ev])
    total_ms = _max_over_ranks(ws_n, float(step_ms.sum()))
    ms_per_step = total_ms / args.steps
    value = swl_dist.aggregate_throughput(info, T, args.steps, total_ms)
    if swl.switch_layer_device_status(work, stream) != 0:
        raise RuntimeError("device status not OK after the timed steps")
    ref_host = [outs[k].cpu() for k in ("out", "expert_idx", "gate", "pos_in_expert",
                                        "aux_loss")]

    # ---- end to end through the public API: pinned host x copied in, the two
    # shard steps and the all-gather, outputs copied back, every step
    xh = inputs["x"].cpu().pin_memory()
    x_dev = torch.empty_like(inputs["x"])
    oh = [[torch.empty_like(t, device="cpu").pin_memory() for t in ref_host]
          for _ in range(min(32, args.steps))]

    def step_e2e(k):
        x_dev.copy_(xh, non_blocking=True)
        step(x_dev)
        for h, key in zip(oh[k % len(oh)], ("out", "expert_idx", "gate", "pos_in_expert",
                                            "aux_loss")):
            h.copy_(outs[key], non_blocking=True)

    for k in range(args.warmup):
        step_e2e(k)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws_n)
    torch.cuda.synchronize()
    e_start.record(stream)
    for k in range(args.steps):
        step_e2e(k)
    e_end.record(stream)
    e_end.synchronize()
    _barrier(ws_n)
    e2e_total = _max_over_ranks(ws_n, float(e_start.elapsed_time(e_end)))
    e2e_value = ws_n * T * args.steps / (e2e_total / 1e3)
    if swl.switch_layer_device_status(work, stream) != 0:
        raise RuntimeError("device status not OK after the end-to-end steps")
    for k in range(max(0, args.steps - len(oh)), args.steps):
        if not all(torch.equal(a, b) for a, b in zip(oh[k % len(oh)], ref_host)):
            raise RuntimeError("end-to-end outputs of step %d differ" % k)

    C = swl.switch_layer_capacity(T_total, N, cf)
    kept = outs["pos_in_expert"].long() < C
    counts = torch.bincount(outs["expert_idx"].long()[kept], minlength=N)
    touched = int((counts > 0).sum())
    K_kept = int(kept.sum())
    ffn_bytes, layer_bytes = algorithmic_bytes(T, d, d_ff, N, elem, touched, K_kept)
    gather_bytes = 2 * K_kept * d * elem + (T - K_kept) * d * elem
    end_s = float(end_ms.mean()) / 1e3
    peaks = _peaks()
    achieved = (ffn_bytes + gather_bytes) / end_s / 1e9
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if act == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; x ~ N(0,1), T5 truncated-normal init s=0.1)",
        "config": {
            "workload": spec.name, "T": T, "d": d, "d_ff": d_ff, "N": N, "capacity_factor": cf,
            "global_batch": T_total, "capacity": C,
            "parallelism": "dp%d: one global batch, contiguous token range per rank, weights "
                           "replicated; one all-gather of per-expert counts and sums of p "
                           "per step" % ws_n,
            "l2": "flushed between timed steps (256 MiB write, outside the step events); "
                  "expert weights %.0f MB > 126 MB L2" % (2 * N * d * d_ff * elem / 1e6),
        },
        "stages_us": {"shard_end": round(float(end_ms.mean()) * 1e3, 2),
                      "begin_and_exchange": round(float((step_ms - end_ms).mean()) * 1e3, 2)},
        "roofline": {
            "kernel": "shard step 3 (combine, gather, expert FFN)", "bound": "hbm",
            "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": None,
            "algorithmic_bytes": ffn_bytes + gather_bytes,
            "peak_source": peaks["source"] + " (burst copy)",
        },
        "routing": {"experts_touched_here": touched, "kept_tokens_here": K_kept,
                    "aux_loss": float(outs["aux_loss"][0])},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * d * elem,
                "d2h_bytes_per_step": T * d * elem + 3 * 4 * T + 4,
                "note": "per step: pinned host x in, both shard steps and the all-gather, "
                        "out / expert_idx / gate / pos_in_expert / aux_loss back"},
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    swl_dist.finalize(info)


# ----------------------------------------------------------------------------- oracle arm
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_estimate(spec, x, W_r, b_r, weights, ffn_budget_s=None, experts=None) -> dict:
    """The fp64 oracle on a bounded sample of one batch, scaled to the batch.

    Every token is routed (fp64 logits, softmax, argmax, positions and the
    capacity cut: oracle.switch_forward_sampled with no output rows); then the
    oracle's expert FFN and gate scaling run on the kept rows of the experts in
    ``experts`` (or of experts 0, 1, ... until ``ffn_budget_s`` of FFN time).
    The whole-batch time estimate is the routing time plus the FFN time scaled
    by (kept tokens / sampled kept tokens).  ``weights(e)`` supplies expert e's
    host tensors outside the timed part."""
    import oracle
    t0 = time.perf_counter()
    r = oracle.switch_forward_sampled(x, W_r, spec.cf, [], weights, b_r=b_r)
    t_route = time.perf_counter() - t0
    e, kept, g = r["expert_idx"], r["kept"], r["gate"]
    K = int(kept.sum())
    t_ffn, K_s, used = 0.0, 0, []
    for i in (experts if experts is not None else range(spec.N)):
        rows = np.nonzero((e == i) & kept)[0]
        used.append(int(i))
        if rows.size == 0:
            continue
        w = weights(int(i))
        t1 = time.perf_counter()
        u = oracle.expert_ffn(x[torch.from_numpy(rows)], w["W1"], w["b1"], w["W2"], w["b2"])
        y = g[rows, None] * u
        t_ffn += time.perf_counter() - t1
        K_s += int(rows.size)
        del y
        if experts is None and t_ffn >= ffn_budget_s:
            break
    est = t_route + (t_ffn * K / K_s if K_s else 0.0)
    return {"t_route": t_route, "t_ffn": t_ffn, "kept": K, "kept_sampled": K_s,
            "experts": used, "estimate_s": est}


def _sample_text(spec, m) -> str:
    return ("every one of the %d tokens routed by the fp64 oracle (%.2f s); its expert FFN "
            "timed on the %d kept rows of experts %d..%d (%.2f s) and scaled to all %d kept "
            "rows" % (spec.T, m["t_route"], m["kept_sampled"], m["experts"][0],
                      m["experts"][-1], m["t_ffn"], m["kept"]))


def cpu_baseline(spec, inputs, budget_s: float = 20.0):
    """The fp64 oracle on the host cores, on a bounded sample of the batch that
    the GPU arm ran (its seeded inputs, copied to the host)."""
    x = inputs["x"].cpu()
    W_r = inputs["W_r"].cpu()
    b_r = inputs["b_r"].cpu() if inputs["b_r"] is not None else None

    def weights(e):
        return {k: inputs[k][e].cpu() for k in ("W1", "b1", "W2", "b2")}

    m = oracle_estimate(spec, x, W_r, b_r, weights, ffn_budget_s=0.6 * budget_s)
    return {"value": spec.T / m["estimate_s"], "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle", "sample": _sample_text(spec, m)}


def run_reference(args):
    ws_n = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import functools
    spec = synth.WORKLOADS[args.workload]
    rd = synth.load_gap_redraws(spec.name)
    x = synth.make_x(spec, 0, "cpu", rd)
    r = synth.make_router(spec, 0, "cpu")

    @functools.lru_cache(maxsize=None)
    def weights(e):
        w = synth.expert_slice(spec, [e], 0, "cpu")
        return {k: v[0] for k, v in w.items()}

    # the expert sample is fixed by a first (untimed) pass with a small FFN budget,
    # so that warm-up and timed steps stay within a few minutes
    m0 = oracle_estimate(spec, x, r["W_r"], r["b_r"], weights, ffn_budget_s=args.cpu_budget / 10)
    experts = m0["experts"]
    for _ in range(args.warmup):
        oracle_estimate(spec, x, r["W_r"], r["b_r"], weights, experts=experts)
    ms = [oracle_estimate(spec, x, r["W_r"], r["b_r"], weights, experts=experts)
          for _ in range(args.steps)]
    total = sum(m["estimate_s"] for m in ms)
    v = spec.T * args.steps / total
    cores = _blas_threads()
    sample = "each step: " + _sample_text(spec, ms[-1])
    res = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": spec.name, "T": spec.T, "d": spec.d, "d_ff": spec.d_ff,
                   "N": spec.N, "capacity_factor": spec.cf},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--shape", default=None,
                    help="ad-hoc layer T,d,d_ff,N,capacity_factor[,dtype] (dtype bf16, the "
                         "default, or f32) instead of a named workload")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--router", default="tensor", choices=["tensor", "ffma"],
                    help="fp32 router logits of bf16 layers: tensor cores on the exact bf16 "
                         "split of W_r (default) or FFMA on the CUDA cores")
    ap.add_argument("--variant", default=None, choices=VARIANTS,
                    help="measure a layer variant instead (one GPU): top2, ntlb "
                         "(No-Token-Left-Behind), geglu, jitter, or backward")
    ap.add_argument("--global-batch", action="store_true",
                    help="use the multi-rank global-batch path (shard steps and the record "
                         "all-gather) also on a single GPU")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)     # at least 3 untimed warm-up steps
    if args.shape:
        fields = args.shape.split(",")
        T, d, d_ff, N, cf = fields[:5]
        dt = fields[5] if len(fields) > 5 else "bf16"
        if dt not in ("bf16", "f32"):
            raise SystemExit("--shape dtype must be bf16 or f32")
        spec = synth.LayerSpec("shape_T%s_d%s_f%s_N%s_cf%s%s" % (T, d, d_ff, N, cf,
                                                                 "" if dt == "bf16" else "_f32"),
                               int(T), int(d), int(d_ff), int(N), float(cf), dt)
        synth.WORKLOADS[spec.name] = spec
        args.workload = spec.name
    if args.impl == "reference":
        run_reference(args)
    elif args.variant:
        run_variant(args)
    elif int(os.environ.get("WORLD_SIZE", "1")) > 1 or args.global_batch:
        run_gpu_sharded(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
