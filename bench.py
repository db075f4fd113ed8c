"""Benchmark of the Sparsely-Gated MoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload lm-flat] [--impl ours|reference]

One step = one full forward pass (gate, dispatch, experts, combine, balancing
statistics) of one batch of the workload through the fused C-ABI call
``moe_forward``, its launches replayed from a CUDA graph captured from that
call (``MoELayer.forward_graph_``; ``--no-graph`` times direct calls).  Inputs
are resident in HBM; L2 is flushed (256 MiB write)
before every timed step, and every step is timed on the device with CUDA
events on the launching stream; the total is the max over ranks.  With N > 1
(launched by torchrun) every rank runs its own independent batch on its own
GPU (replicas, weak scaling; the layer has no cross-batch exchange).

The JSON line also carries: e2e (same metric through the Python/C-ABI call
with pinned host buffers, copies inside the timed region), the roofline of the
dominant kernel (per-kernel CUDA-event times recorded by the library around
its own launches), the expert-FFN TFLOP/s and routing GB/s of the metric,
clocks sampled during the timed region, the count of library kernel launches,
and the oracle's CPU baseline on a bounded sample.  ``--impl reference`` times
the oracle itself (the reference arm of this comparison).

``--backward``: one step is the forward pass followed by the backward pass
(``moe_backward``: dx and every parameter's gradient for an upstream gradient
dy plus the weighted balancing losses); the metric is then training tokens/s.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s; expert-FFN TFLOP/s vs bf16 peak; routing HBM GB/s"
METRIC_TRAIN = "MoE-layer training tokens/s (forward + backward, all gradients)"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS, FP32_LANES = 148, 128  # B200: 148 SMs x 128 FP32 lanes


# ------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(total_ms: float, tokens_per_rank: int, steps: int, world: int, group=None):
    """Max of the device time over ranks; value = tokens of all ranks / that
    time.  Works for any torch.distributed backend (the test uses gloo)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([total_ms], dtype=torch.float64)
    if world > 1:
        if dist.get_backend(group) == "nccl":
            t = t.cuda()
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    ms = float(t.item())
    value = world * tokens_per_rank * steps / (ms / 1e3) if ms > 0 else 0.0
    return ms, value


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load)}


def src_sha(name: str) -> str:
    with open(os.path.join(ROOT, "sparsely_gated_mixture_gate_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


KERNEL_SRC = {"expert_ffn_tcgen05": "expert_tc.cu",
              "gate_gemm_fp32": "gate_gemm.cu", "route_topk": "route.cu", "combine": "combine.cu",
              "dispatch_place": "dispatch.cu", "dispatch_hist": "dispatch.cu",
              "expert_bwd_tcgen05": "expert_tc.cu", "wgrad_tcgen05": "wgrad_tc.cu",
              "gate_wgrad_fp32": "grad_gemm.cu", "gate_dgrad_fp32": "grad_gemm.cu",
              "combine_bwd": "backward.cu", "dx_gather": "backward.cu", "gate_bwd": "backward.cu",
              "bias_grad": "backward.cu"}


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_SRC:
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(workload, {}).get(kernel)
    if not rec or rec.get("csrc_sha") != src_sha(KERNEL_SRC[kernel]):
        return None
    return rec.get("dram_bytes_per_launch")


def kernel_work(w, name: str, S_kept: int):
    """Algorithmic work of one launch: (bound, flops, bytes)."""
    T, d, n, k, f = w.T, w.d, w.n, w.k, w.f
    S = T * k
    ng = w.hier_a if w.hier_a else n
    esz = 2 if w.expert_bf16 else 4
    if name == "expert_ffn_tcgen05":
        # both layers in one persistent launch: every weight once, x_perm in,
        # y_perm out (the hidden layer's round trip through memory is this
        # implementation's choice, not counted as algorithmic traffic)
        return "tensor", 4.0 * S_kept * d * f, n * 2 * d * f * esz + 2 * S_kept * d * esz
    if name == "shared_expert_ffn_tcgen05":
        # one expert on all T tokens: its weights once, x rows in, rows out
        return "tensor", 4.0 * T * d * f, 2 * d * f * esz + 2 * T * d * esz
    if name == "gate_gemm_fp32":
        return "alu", 2.0 * T * d * ng * (2 if w.noise else 1), 4 * (T * d + d * ng * 2 + 2 * T * ng)
    if name == "gate_gemm_tf32x3":
        # the fp32-equivalent contraction; three tf32 MMAs carry it
        return "tensor_tf32x3", 2.0 * T * d * ng * (2 if w.noise else 1), \
            4 * (2 * T * d + 2 * d * ng * 2 + 2 * T * ng)
    if name == "expert_ffn_fp32":
        # both layers of every expert on its rows, fp32 weights streamed once
        return "hbm", 4.0 * S_kept * d * f, n * 2 * d * f * 4 + S_kept * d * 4 * 2
    # ---- backward pass
    if name == "expert_bwd_tcgen05":
        # dhid = (dy_perm W2) * mask, dx_perm = dhid W1: both weights once, dy_perm and the
        # forward's hid in, dhid (needed again by the weight gradients) and dx_perm out
        return "tensor", 4.0 * S_kept * d * f, \
            n * 2 * d * f * esz + S_kept * (2 * d + 2 * f) * esz
    if name == "wgrad_tcgen05":
        # dW2 = dy_perm^T hid, dW1 = dhid^T x_perm per expert: four activations in, fp32 out
        return "tensor", 4.0 * S_kept * d * f, S_kept * 2 * (d + f) * esz + n * 2 * d * f * 4
    if name == "combine_bwd":
        return "hbm", 0.0, T * d * 4 + 2 * S_kept * d * esz + 12 * T * k
    if name == "dx_gather":
        return "hbm", 0.0, S_kept * d * esz + T * d * 4 + 4 * T * k
    if name == "bias_grad":
        return "hbm", 0.0, S_kept * (d + f) * esz + n * (d + f) * 4
    if name == "gate_bwd":
        return "hbm", 0.0, 4 * T * ng * (2 if w.noise else 1) * 2 + 16 * T * k + 16 * T
    if name in ("gate_wgrad_fp32", "gate_dgrad_fp32"):
        # one launch carries the clean and the noise products (two with noise)
        nprod = 2 if w.noise else 1
        return "alu", nprod * 2.0 * T * d * ng, 4 * (T * d + nprod * (d * ng + T * ng))
    if name == "route_topk":
        return "hbm", 0.0, 4 * T * ng * (2 if w.noise else 1) + 8 * T * k
    if name == "combine":
        return "hbm", 0.0, S_kept * d * esz + T * d * 4 + 8 * T * k
    if name == "dispatch_place":
        # x read, kept rows written; per pair: id, gate, block rank and base
        # read, row and sorted gate written; per kept row its token
        return "hbm", 0.0, T * d * 4 + S_kept * d * esz + 24 * S + 4 * S_kept
    return None, 0.0, 0.0


# ------------------------------------------------------------------ arms
def run_ours(args, w, world, rank, local):
    import torch
    import torch.distributed as dist

    from sparsely_gated_mixture_gate_b200 import moe as M
    from sparsely_gated_mixture_gate_b200 import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    # every rank: its own batch (x seeded by rank), the same weights
    inp = synth.make_inputs(w, device=dev)
    if rank:
        inp["x"] = synth.make_inputs(w.with_(seed=rank), device=dev, experts=False)["x"]
    cfg = M.Config.from_workload(w)
    if args.backward:
        cfg = dataclasses.replace(cfg, backward=1)
    layer = M.MoELayer(cfg, inp, dev)
    x = inp["x"]
    dy = synth.make_dy(w.with_(seed=w.seed + rank), device=dev) if args.backward else None
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    # the forward pass's launches are replayed from a CUDA graph (one host call
    # per step; the same kernels on the same buffers) unless --no-graph
    use_graph = not args.no_graph

    def direct_step():
        layer.forward_(x)
        if dy is not None:
            layer.backward_(x, dy)

    def step():
        if not use_graph:
            direct_step()
        elif dy is None:
            layer.forward_graph_(x)
        else:
            layer.train_graph_(x, dy)

    # kernels per step, counted on one direct call (a graph replay launches the
    # same kernels without passing through the library's launch counter)
    l0 = M.launch_count()
    direct_step()
    per_step_launches = M.launch_count() - l0

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    st = M.status_bits(layer.status)
    if st:
        raise SystemExit(f"device status {st} after warm-up")
    S_kept = int(layer.counts.clamp(max=M.capacity(cfg) if w.capacity_factor > 0 else 2**31 - 1).sum())

    # ---- timed region: K device-timed steps (no per-kernel events inside)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = M.launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    launches = per_step_launches * args.steps if use_graph else M.launch_count() - launches0
    clk = clocks.stop()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms, value = aggregate(total_ms, w.T, args.steps, world)

    # ---- second timed pass for the roofline: CUDA events recorded by the
    # library around each of its launches, on the launching stream (the
    # events add a little time per launch, so this pass is not the value;
    # direct calls, so it times every kernel without the graph's tighter gaps)
    t_steps = max(3, min(args.steps, 300))
    M.trace_reset()
    M.trace_enable(True)
    torch.cuda.synchronize()
    for i in range(t_steps):
        flush.fill_(float(i))
        direct_step()  # the library's events need its own launches, not a graph replay
    torch.cuda.synchronize()
    M.trace_enable(False)
    per_kernel = M.trace_read()

    # ---- e2e: host buffers, copies inside the timed region.  Every step
    # copies its batch from pinned host memory and its y and losses back;
    # consecutive steps overlap copies with compute on separate streams.
    e_steps = max(3, min(args.steps, 200))
    xh = x.cpu().pin_memory()
    yh = [torch.empty(w.T, w.d, dtype=torch.float32).pin_memory() for _ in range(2)]
    lh = [torch.empty(layer.losses.numel(), dtype=torch.float32).pin_memory() for _ in range(2)]
    if dy is None:
        layer.forward_host_batches([xh] * 3, [yh[i & 1] for i in range(3)],
                                   [lh[i & 1] for i in range(3)], graph=use_graph)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        d2h = layer.forward_host_batches([xh] * e_steps, [yh[i & 1] for i in range(e_steps)],
                                         [lh[i & 1] for i in range(e_steps)], graph=use_graph)
        stream.wait_stream(d2h)
        e1.record(stream)
        torch.cuda.synchronize()
        h2d_bytes, d2h_bytes = w.T * w.d * 4, w.T * w.d * 4 + 4 * layer.losses.numel()
    else:
        # training steps from host memory: x and dy in, y, the losses and dx
        # out every step (the parameter gradients stay on the device for the
        # optimizer); copies of neighbouring steps overlap compute
        dyh = dy.cpu().pin_memory()
        dxh = [torch.empty(w.T, w.d, dtype=torch.float32).pin_memory() for _ in range(2)]

        def host_steps(m):
            return layer.train_host_batches([xh] * m, [dyh] * m, [yh[i & 1] for i in range(m)],
                                            [lh[i & 1] for i in range(m)],
                                            [dxh[i & 1] for i in range(m)], graph=use_graph)

        host_steps(3)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        d2h = host_steps(e_steps)
        stream.wait_stream(d2h)
        e1.record(stream)
        torch.cuda.synchronize()
        h2d_bytes = 2 * w.T * w.d * 4
        d2h_bytes = 2 * w.T * w.d * 4 + 4 * layer.losses.numel()
    e_ms, e_value = aggregate(e0.elapsed_time(e1), w.T, e_steps, world)
    st = M.status_bits(layer.status)

    # ---- the other gate mode on the same weights (short run, reported apart)
    alt = None
    if args.alt_gate and world == 1 and dy is None:
        other = 0 if w.gate_precision else 1
        alt_layer = M.MoELayer(M.Config.from_workload(w.with_(gate_precision=other)), inp, dev)
        alt_step = alt_layer.forward_graph_ if use_graph else alt_layer.forward_
        for _ in range(3):
            flush.fill_(1.0)
            alt_step(x)
        torch.cuda.synchronize()
        a_steps = max(3, min(args.steps, 300))
        as_ = [torch.cuda.Event(enable_timing=True) for _ in range(a_steps)]
        ae_ = [torch.cuda.Event(enable_timing=True) for _ in range(a_steps)]
        for i in range(a_steps):
            flush.fill_(float(i))
            as_[i].record(stream)
            alt_step(x)
            ae_[i].record(stream)
        torch.cuda.synchronize()
        a_ms = sum(p.elapsed_time(q) for p, q in zip(as_, ae_))
        alt = {"gate": "tf32x3" if other else "fp32", "value": round(w.T * a_steps / (a_ms / 1e3), 1),
               "ms_per_step": round(a_ms / a_steps, 5), "steps": a_steps,
               "device_status": M.status_bits(alt_layer.status)}
        alt_layer.release_graph()
        del alt_layer

    if rank != 0:
        return None

    # ---- roofline of the dominant kernel and the metric's two side figures
    kstats = {}
    # launches on the library's side stream run beside the main chain; their
    # event spans include waits for SMs the main chain holds, so they take no
    # share of the step and cannot be the dominant kernel
    main_chain = {k: v for k, v in per_kernel.items() if not k.endswith("[side stream]")}
    main_ms = max(sum(r["ms"] for r in main_chain.values()), 1e-9)
    for name, rec in per_kernel.items():
        per_launch_ms = rec["ms"] / max(rec["launches"], 1)
        bound, flops, nbytes = kernel_work(w, name, S_kept)
        e = {"launches": rec["launches"], "ms_per_launch": round(per_launch_ms, 5)}
        if name in main_chain:
            e["share"] = round(rec["ms"] / main_ms, 4)
        else:
            e["overlapped"] = True
        if bound:
            e["gbs"] = round(nbytes / (per_launch_ms / 1e3) / 1e9, 1)
            if flops:
                e["tflops"] = round(flops / (per_launch_ms / 1e3) / 1e12, 2)
        kstats[name] = e
    dom = max(main_chain, key=lambda k: main_chain[k]["ms"])
    bound, flops, nbytes = kernel_work(w, dom, S_kept)
    dom_ms = per_kernel[dom]["ms"] / per_kernel[dom]["launches"]
    sustained = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    if bound == "tensor":
        ai = flops / nbytes
        ridge = sustained * 1e12 / (pk["hbm_gbs"] * 1e9)
        if ai < ridge:  # the weights stream from HBM: bandwidth bound
            roof = {"bound": "hbm", "achieved": nbytes / (dom_ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                    "unit": "GB/s"}
        else:
            roof = {"bound": "tensor", "achieved": flops / (dom_ms / 1e3) / 1e12, "peak": sustained,
                    "unit": "TFLOP/s"}
    elif bound == "tensor_tf32x3":
        # tf32 dense peak = bf16 peak / 2 (nominal ratio); three MMAs per product
        tf32_peak = sustained / 2.0
        roof = {"bound": "tensor", "achieved": 3 * flops / (dom_ms / 1e3) / 1e12, "peak": tf32_peak,
                "unit": "TFLOP/s (tf32, 3 MMAs per fp32 product)"}
    elif bound == "alu":
        fp32_peak = SMS * FP32_LANES * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": flops / (dom_ms / 1e3) / 1e12, "peak": round(fp32_peak, 1),
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / (dom_ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                "unit": "GB/s"}
    roof["achieved"] = round(roof["achieved"], 2)
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["kernel"] = dom
    roof["peak_source"] = pk["source"]
    roof["traffic"] = ncu_traffic(dom, w.name)

    ffn_ms = sum(per_kernel[k]["ms"] / per_kernel[k]["launches"] for k in per_kernel
                 if k.startswith("expert_ffn_tcgen05"))
    ffn_flops = 4.0 * S_kept * w.d * w.f
    route_names = [k for k in main_chain if k.startswith(("route", "dispatch", "combine"))]
    route_ms = sum(per_kernel[k]["ms"] / per_kernel[k]["launches"] for k in route_names)
    route_bytes = sum(kernel_work(w, k, S_kept)[2] for k in route_names)

    line = {
        "metric": METRIC_TRAIN if dy is not None else METRIC, "value": round(value, 1),
        "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp32",
        "data": "synthetic (seeded; random-init weights of the workload's shapes)",
        "config": {"workload": w.name + (" (forward + backward)" if dy is not None else ""),
                   "T": w.T, "d_model": w.d, "experts": w.n, "k": w.k,
                   "d_ff": w.f, "hier": [w.hier_a, w.hier_b] if w.hier_a else None,
                   "router": "switch-top1" if w.router else "noisy-top-k",
                   "gate": "3-pass TF32 on tensor cores (fp32-level)" if w.gate_precision
                   else "fp32 multiply-adds",
                   "capacity_factor": w.capacity_factor or None,
                   "l2": "flushed before every timed step (256 MiB write)",
                   "launch": (("one CUDA graph replay per step (captured from moe_forward"
                               + (" and moe_backward)" if dy is not None else ")"))
                              if use_graph else "direct C-ABI calls"),
                   "parallelism": f"replicas x{world}"},
        "expert_ffn_tflops": round(ffn_flops / (ffn_ms / 1e3) / 1e12, 2) if ffn_ms else None,
        "expert_ffn_frac_bf16_peak": round(ffn_flops / (ffn_ms / 1e3) / 1e12 / sustained, 4) if ffn_ms else None,
        "routing_hbm_gbs": round(route_bytes / (route_ms / 1e3) / 1e9, 1) if route_ms else None,
        "roofline": roof,
        "kernels": kstats,
        "kernel_timing": f"second pass of {t_steps} steps, CUDA events around every library launch",
        "gpu_launches": int(launches),
        "gpu_launches_per_step": int(per_step_launches),
        "e2e": {"value": round(e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes, "steps": e_steps,
                "how": ("pinned host x in, y and losses out every step; copies of neighbouring "
                        "steps overlap compute on two copy streams"
                        + ("; each step's forward replayed from a CUDA graph" if use_graph else ""))
                       if dy is None else
                       ("pinned host x and dy in, y, losses and dx out every step; copies of "
                        "neighbouring steps overlap compute on two copy streams (parameter "
                        "gradients stay on the device)")},
        "clocks": clk,
        "alt_gate_mode": alt,
        "wall_s": round(wall, 3),
        "device_status": st,
    }
    return line


def oracle_sample_inputs(w, T_s):
    import torch

    from sparsely_gated_mixture_gate_b200 import synth
    inp = synth.make_inputs(w, T=T_s)
    return {k: (None if v is None else (synth.bf16_bits(v) if v.dtype == torch.bfloat16 else v.numpy()))
            for k, v in inp.items()}


def oracle_step(w, T_s, backward=False):
    """One oracle step on the first T_s tokens: the forward pass, and with
    backward the backward pass too (as a function of no arguments)."""
    from oracle import oracle as orc
    orc.build()
    npin = oracle_sample_inputs(w, T_s)
    cfg = dict(w.cfg(), T=T_s)
    if not backward:
        return lambda: orc.forward(cfg, npin)
    from sparsely_gated_mixture_gate_b200 import synth
    dy = synth.make_dy(w, T=T_s).numpy()

    def both():
        orc.forward(cfg, npin)
        orc.backward(cfg, npin, dy)
    return both


def time_oracle(w, T_s, reps=1, backward=False):
    fn = oracle_step(w, T_s, backward)
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    return time.perf_counter() - t0


def cpu_baseline(w, budget_s=12.0, backward=False):
    """The oracle (single-threaded C, as it stands) on the first tokens of the
    workload: calibrate on 8 tokens, then run a sample of about budget_s."""
    t8 = time_oracle(w, 8, backward=backward)
    T_s = int(max(8, min(w.T, budget_s / max(t8 / 8, 1e-6))))
    t = time_oracle(w, T_s, backward=backward)
    what = "forward + backward" if backward else "forward"
    return {"value": round(T_s / t, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{what} of the first {T_s} tokens of {w.name} as one batch "
                      f"(same weights), {t:.1f} s"}


def run_reference(args, w):
    """The reference arm: the oracle itself, each step a bounded sample of the
    workload sized so the whole run stays within about two minutes."""
    t8 = time_oracle(w, 8, backward=args.backward)
    per_tok = max(t8 / 8, 1e-6)
    budget = 90.0 / max(args.steps + args.warmup, 1)
    T_s = int(max(1, min(w.T, budget / per_tok)))
    fn = oracle_step(w, T_s, args.backward)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    t = time.perf_counter() - t0
    value = T_s * args.steps / t
    sample = f"first {T_s} tokens of {w.name} per step (same weights)"
    return {"impl": "reference", "metric": METRIC_TRAIN if args.backward else METRIC,
            "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "T": w.T, "d_model": w.d, "experts": w.n, "k": w.k, "d_ff": w.f,
                       "sample_tokens_per_step": T_s},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="lm-flat")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--gate", default="fp32", choices=["fp32", "tf32x3"],
                    help="gate projections: fp32 multiply-adds or the 3-pass TF32 tensor-core split")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time direct library calls instead of a CUDA graph replay of the forward")
    ap.add_argument("--backward", action="store_true",
                    help="time forward + backward (training step) instead of the forward pass")
    ap.add_argument("--no-alt-gate", dest="alt_gate", action="store_false",
                    help="skip the short run of the other gate mode")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    from sparsely_gated_mixture_gate_b200 import synth
    w = (synth.WORKLOADS.get(args.workload) or synth.VARIANTS[args.workload]).with_(
        gate_precision=1 if args.gate == "tf32x3" else 0)
    world, rank, local = dist_info()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    import datetime

    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_ours(args, w, world, rank, local)
        if rank == 0 and line is not None:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(w, backward=args.backward)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
