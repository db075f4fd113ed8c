"""Benchmark of the Sparsely-Gated MoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload hierarchical]
                    [--impl ours|reference] [--backward] [--no-per-config]

One step = one full forward pass (gate, dispatch, experts, combine, balancing
statistics) of one batch of the workload through the fused C-ABI call
``moe_forward``, its launches replayed from a CUDA graph captured from that
call (``MoELayer.forward_graph_``; ``--no-graph`` times direct calls).  The
default workload is the hierarchical layer (65536 tokens, 64 groups x 128
experts, 8.6 B expert parameters), the largest that fits one GPU.  Inputs
are resident in HBM; L2 is flushed (256 MiB write) before every timed step,
and every step is timed on the device with CUDA events on the launching
stream; the total is the max over ranks.  The gate's noise is redrawn every
step (the layer advances its noise key on the device).  With N > 1 (launched
by torchrun) every rank runs its own independent batch on its own GPU
(replicas, weak scaling; the layer has no cross-batch exchange).

The JSON line also carries: e2e (same metric through the Python/C-ABI call
with pinned host buffers, copies inside the timed region), the roofline of the
dominant kernel and of every kernel (per-kernel CUDA-event times recorded by
the library around its own launches, against the algorithmic work per step:
expert weight bytes or FLOPs, gate FP32 FLOPs, routing bytes), the FP32 FMA
peak measured in the same run, the expert-FFN TFLOP/s and routing GB/s of the
metric, clocks sampled during the timed region, the count of library kernel
launches, the oracle's CPU baseline on a bounded sample, and ``per_config``:
a short run of each of the five workloads.  ``--impl reference`` times the
oracle itself (the reference arm of this comparison).

``--backward``: one step is the forward pass followed by the backward pass
(``moe_backward``: dx and every parameter's gradient for an upstream gradient
dy plus the weighted balancing losses); the metric is then training tokens/s
(default workload: hierarchical, as for the forward pass).
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
    """Algorithmic work of all of one step's launches of a kernel, in the
    units of the layer's measurement table: (bound, flops, bytes).

    The expert FFN streams every expert's two weight matrices once: its
    bytes are the weight bytes n*2*d*f*esz (the activations it reads and
    writes are counted by the dispatch and the combine); its FLOPs are
    4*S*d*f.  The fp32 gate GEMM is counted in FLOPs (primary and secondary
    gates of the hierarchical layer together), the routing, dispatch and
    combine kernels in the bytes they must move."""
    T, d, n, k, f = w.T, w.d, w.n, w.k, w.f
    S = T * k
    esz = 2 if w.expert_bf16 else 4
    npj = 2 if w.noise else 1          # projections: clean (+ noise)
    if w.hier_a:
        k1 = w.hier_k1
        gate_flops = 2.0 * T * d * w.hier_a * npj + 2.0 * T * k1 * d * w.hier_b * npj
        gate_cols = T * w.hier_a + T * k1 * w.hier_b        # (row, column) pairs of c and s
        route_extra = 8 * T * k1 + 8 * T * k
        place_extra = 28 * T * k1                              # the group pass moves indices only
    else:
        gate_flops = 2.0 * T * d * n * npj
        gate_cols = T * n
        route_extra = 8 * T * k
        place_extra = 0
    if name == "expert_ffn_tcgen05":
        return "tensor", 4.0 * S_kept * d * f, n * 2 * d * f * esz
    if name == "shared_expert_ffn_tcgen05":
        return "tensor", 4.0 * T * d * f, 2 * d * f * esz
    if name == "gate_gemm_fp32":
        return "alu", gate_flops, 4 * (T * d + 4 * gate_cols)
    if name == "gate_gemm_tf32x3":
        # the fp32-equivalent contraction; three tf32 MMAs carry it
        return "tensor_tf32x3", gate_flops, 4 * (2 * T * d + 4 * gate_cols)
    if name == "expert_ffn_fp32":
        return "hbm", 4.0 * S_kept * d * f, n * 2 * d * f * 4
    # ---- backward pass
    if name == "expert_bwd_tcgen05":
        return "tensor", 4.0 * S_kept * d * f, \
            n * 2 * d * f * esz + S_kept * (2 * d + 2 * f) * esz
    if name == "wgrad_tcgen05":
        return "tensor", 4.0 * S_kept * d * f, S_kept * 2 * (d + f) * esz + n * 2 * d * f * 4
    if name == "combine_bwd":
        return "hbm", 0.0, T * d * 4 + 2 * S_kept * d * esz + 12 * T * k
    if name == "dx_gather":
        return "hbm", 0.0, S_kept * d * esz + T * d * 4 + 4 * T * k
    if name == "bias_grad":
        return "hbm", 0.0, S_kept * (d + f) * esz + n * (d + f) * 4
    ng = w.hier_a if w.hier_a else n   # the flat (or primary) gate's width
    if name == "gate_bwd":
        # c, s read and dc, dz written per (row, column): the flat / primary
        # gate's T rows and, hierarchical, the T k1 secondary rows of width b
        return "hbm", 0.0, 4 * gate_cols * npj * 2 + 16 * T * k + 16 * T
    if name in ("gate_wgrad_fp32", "gate_dgrad_fp32"):
        return "alu", npj * 2.0 * T * d * ng, 4 * (T * d + npj * (d * ng + T * ng))
    if w.hier_a and name in ("hier_gate_wgrad", "hier_gate_dgrad"):
        # the secondary gates' contractions over the T k1 gathered rows
        R2, b = T * w.hier_k1, w.hier_b
        return "alu", npj * 2.0 * R2 * d * b, 4 * (R2 * d + npj * (w.hier_a * d * b + R2 * b))
    if name == "route_topk":
        return "hbm", 0.0, 4 * gate_cols * npj + route_extra
    if name == "combine":
        return "hbm", 0.0, S_kept * d * esz + T * d * 4 + 8 * T * k
    if name == "dispatch_place":
        # x read, kept rows written; per pair: id, gate, block rank and base
        # read, row and sorted gate written; per kept row its token
        return "hbm", 0.0, T * d * 4 + S_kept * d * esz + 24 * S + 4 * S_kept + place_extra
    return None, 0.0, 0.0


def fp32_fma_peak(dev, pk):
    """The FP32 FMA throughput of this GPU, measured: scalar fma.rn.f32 and
    packed fma.rn.f32x2 probe kernels (8 blocks of 256 threads per SM,
    16 independent chains per thread), best of three runs each, CUDA events
    on the launching stream.  Falls back to SMs x 128 lanes x 2 x max clock."""
    import ctypes as C

    import torch

    from sparsely_gated_mixture_gate_b200 import _lib
    derived = SMS * FP32_LANES * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    try:
        L = _lib.load()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        blocks, iters = sms * 8, 4096
        out = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
        st = torch.cuda.current_stream()
        res = {}
        for packed in (0, 1):
            best = 0.0
            for rep in range(4):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                rc = L.moe_fma_probe(C.c_void_p(out.data_ptr()), blocks, iters, packed,
                                     C.c_void_p(st.cuda_stream))
                e1.record(st)
                torch.cuda.synchronize()
                if rc != 0:
                    raise RuntimeError(f"moe_fma_probe: {rc}")
                if rep:  # the first run warms up
                    best = max(best, blocks * 256.0 * iters * 256.0 / (e0.elapsed_time(e1) / 1e3) / 1e12)
            res["f32x2" if packed else "f32"] = round(best, 2)
        return {"tflops": max(res.values()), "source": "measured (FMA probe in this run)", **res,
                "derived": round(derived, 1)}
    except Exception as e:  # pragma: no cover - reported, not hidden
        return {"tflops": derived, "source": f"derived (probe failed: {e})", "derived": round(derived, 1)}


# ------------------------------------------------------------------ arms
def run_ours(args, w, world, rank, local, steps=None, warmup=None, alt_gate=None, fp32_peak=None,
             cpu_sample=False):
    """One workload through the fused forward (or the training step): the
    device-timed value, the per-kernel trace, e2e, the roofline of the
    dominant kernel; with cpu_sample also the oracle's CPU baseline on a
    sample of the same inputs."""
    import torch
    import torch.distributed as dist

    from sparsely_gated_mixture_gate_b200 import moe as M
    from sparsely_gated_mixture_gate_b200 import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    steps = args.steps if steps is None else steps
    warmup = args.warmup if warmup is None else warmup
    alt_gate = args.alt_gate if alt_gate is None else alt_gate
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

    for _ in range(warmup):
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
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches0 = M.launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    launches = per_step_launches * steps if use_graph else M.launch_count() - launches0
    clk = clocks.stop()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms, value = aggregate(total_ms, w.T, steps, world)

    # ---- second timed pass for the roofline: CUDA events recorded by the
    # library around each of its launches, on the launching stream (the
    # events add a little time per launch, so this pass is not the value;
    # direct calls, so it times every kernel without the graph's tighter gaps)
    t_steps = max(3, min(steps, 300))
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
    # consecutive steps overlap copies with compute on separate streams.  The
    # first step's copy in and the last step's copy out are not overlapped
    # (pipeline fill and drain, included); at least 50 steps amortise them.
    e_steps = max(50, min(steps, 200))
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
    if alt_gate and world == 1 and dy is None:
        other = 0 if w.gate_precision else 1
        alt_layer = M.MoELayer(M.Config.from_workload(w.with_(gate_precision=other)), inp, dev)
        alt_step = alt_layer.forward_graph_ if use_graph else alt_layer.forward_
        for _ in range(3):
            flush.fill_(1.0)
            alt_step(x)
        torch.cuda.synchronize()
        a_steps = max(3, min(steps, 300))
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

    cpu = None
    if cpu_sample and rank == 0 and world == 1:
        cpu = cpu_baseline(w, inp=inp, backward=dy is not None)
    layer.release_graph()
    if rank != 0:
        return None

    # ---- per kernel: the step's launches of each kernel against its
    # algorithmic work per step (see kernel_work)
    burst = pk["bf16_tflops"]
    if fp32_peak is None:
        fp32_peak = fp32_fma_peak(dev, pk)
    kstats = {}
    # launches on the library's side stream run beside the main chain; their
    # event spans include waits for SMs the main chain holds, so they take no
    # share of the step and cannot be the dominant kernel
    main_chain = {k: v for k, v in per_kernel.items() if not k.endswith("[side stream]")}
    main_ms = max(sum(r["ms"] for r in main_chain.values()), 1e-9)

    def roof_of(name):
        bound, flops, nbytes = kernel_work(w, name, S_kept)
        step_ms = per_kernel[name]["ms"] / t_steps
        if bound == "tensor":
            ai = flops / max(nbytes, 1)
            ridge = burst * 1e12 / (pk["hbm_gbs"] * 1e9)
            if ai < ridge:  # the weights stream from HBM: bandwidth bound
                r = {"bound": "hbm", "achieved": nbytes / (step_ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "work": "expert weight bytes streamed"}
            else:
                r = {"bound": "tensor", "achieved": flops / (step_ms / 1e3) / 1e12, "peak": burst,
                     "unit": "TFLOP/s", "work": "expert FLOPs (bf16)"}
        elif bound == "tensor_tf32x3":
            # tf32 dense peak = bf16 peak / 2 (nominal ratio); three MMAs per product
            r = {"bound": "tensor", "achieved": 3 * flops / (step_ms / 1e3) / 1e12, "peak": burst / 2.0,
                 "unit": "TFLOP/s (tf32, 3 MMAs per fp32 product)", "work": "gate FLOPs"}
        elif bound == "alu":
            r = {"bound": "alu", "achieved": flops / (step_ms / 1e3) / 1e12,
                 "peak": round(fp32_peak["tflops"], 2), "unit": "TFLOP/s", "work": "gate FLOPs (fp32)"}
        elif bound == "hbm":
            r = {"bound": "hbm", "achieved": nbytes / (step_ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                 "unit": "GB/s", "work": "bytes moved"}
        else:
            return None
        r["achieved"] = round(r["achieved"], 2)
        r["frac"] = round(r["achieved"] / r["peak"], 4)
        return r

    for name, rec in per_kernel.items():
        e = {"launches_per_step": round(rec["launches"] / t_steps, 2),
             "ms_per_step": round(rec["ms"] / t_steps, 5)}
        if name in main_chain:
            e["share"] = round(rec["ms"] / main_ms, 4)
            r = roof_of(name)
            if r:
                e["roofline"] = {k2: r[k2] for k2 in ("bound", "achieved", "unit", "frac")}
        else:
            e["overlapped"] = True
        kstats[name] = e
    dom = max(main_chain, key=lambda k: main_chain[k]["ms"])
    roof = roof_of(dom) or {"bound": None, "achieved": None, "peak": None, "unit": None, "frac": None}
    roof["kernel"] = dom
    roof["peak_source"] = fp32_peak["source"] if roof["bound"] == "alu" else \
        (pk["source"] + (" (burst)" if roof["bound"] == "tensor" else ""))
    trf = ncu_traffic(dom, w.name)
    roof["traffic"] = trf
    if trf is not None and roof["bound"] == "hbm":
        # the capture's DRAM bytes per launch against the algorithmic bytes of one launch
        lps = per_kernel[dom]["launches"] / t_steps
        roof["traffic_over_algorithmic"] = round(trf * lps / kernel_work(w, dom, S_kept)[2], 3)

    ffn_ms = sum(per_kernel[k]["ms"] / t_steps for k in per_kernel if k.startswith("expert_ffn_tcgen05"))
    ffn_flops = 4.0 * S_kept * w.d * w.f
    route_names = [k for k in main_chain if k.startswith(("route", "dispatch", "combine"))]
    route_ms = sum(per_kernel[k]["ms"] / t_steps for k in route_names)
    route_bytes = sum(kernel_work(w, k, S_kept)[2] for k in route_names)

    routing = routing_report(w, layer)

    line = {
        "metric": METRIC_TRAIN if dy is not None else METRIC, "value": round(value, 1),
        "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms / steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp32",
        "data": "synthetic (seeded; random-init weights of the workload's shapes)",
        "config": {"workload": w.name + (" (forward + backward)" if dy is not None else ""),
                   "T": w.T, "d_model": w.d, "experts": w.n, "k": w.k,
                   "d_ff": w.f, "hier": [w.hier_a, w.hier_b] if w.hier_a else None,
                   "router": {0: "noisy-top-k", 1: "switch-top1", 2: "sigmoid"}[w.router],
                   "gate": "3-pass TF32 on tensor cores (fp32-level)" if w.gate_precision
                   else "fp32 multiply-adds",
                   "capacity_factor": w.capacity_factor or None,
                   "l2": "flushed before every timed step (256 MiB write)",
                   "noise": "redrawn every step (noise key advanced on the device)" if w.noise else None,
                   "launch": (("one CUDA graph replay per step (captured from moe_forward"
                               + (" and moe_backward)" if dy is not None else ")"))
                              if use_graph else "direct C-ABI calls"),
                   "parallelism": f"replicas x{world}"},
        "expert_ffn_tflops": round(ffn_flops / (ffn_ms / 1e3) / 1e12, 2) if ffn_ms else None,
        "expert_ffn_frac_bf16_peak": round(ffn_flops / (ffn_ms / 1e3) / 1e12 / burst, 4) if ffn_ms else None,
        "routing_hbm_gbs": round(route_bytes / (route_ms / 1e3) / 1e9, 1) if route_ms else None,
        "routing_frac_hbm": round(route_bytes / (route_ms / 1e3) / 1e9 / pk["hbm_gbs"], 4)
        if route_ms else None,
        "roofline": roof,
        "fp32_fma_peak": fp32_peak,
        "kernels": kstats,
        "kernel_timing": f"second pass of {t_steps} steps, CUDA events around every library launch; "
                         "work and time per step",
        "gpu_launches": int(launches),
        "gpu_launches_per_step": int(per_step_launches),
        "e2e": {"value": round(e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes, "steps": e_steps,
                "how": ("pinned host x in, y and losses out every step; copies of neighbouring "
                        "steps overlap compute on two copy streams; pipeline fill and drain "
                        "included"
                        + ("; each step's forward replayed from a CUDA graph" if use_graph else ""))
                       if dy is None else
                       ("pinned host x and dy in, y, losses and dx out every step; copies of "
                        "neighbouring steps overlap compute on two copy streams (parameter "
                        "gradients stay on the device); pipeline fill and drain included")},
        "clocks": clk,
        "alt_gate_mode": alt,
        "wall_s": round(wall, 3),
        "device_status": st,
        "routing": routing,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def routing_report(w, layer):
    """The last step's routing outcome, read back after the timed region: the
    per-expert slot counts (the load histogram, summarised), the balancing
    losses and the drop rate, from the layer's own outputs."""
    counts = layer.counts.double().cpu()
    losses = layer.losses.double().cpu().tolist()
    mean = float(counts.mean())
    hist = {"experts": int(counts.numel()), "min": int(counts.min()), "max": int(counts.max()),
            "mean": round(mean, 3), "std": round(float(counts.std(unbiased=False)), 3),
            "max_over_mean": round(float(counts.max()) / mean, 3) if mean > 0 else None,
            "empty_experts": int((counts == 0).sum())}
    rep = {"counts": hist, "L_importance": losses[0], "L_load": losses[1],
           "cv2_importance": losses[5], "cv2_load": losses[6],
           "drop_rate": losses[4], "dropped_slots": int(losses[7])}
    if w.router == 1:  # Switch: N * sum f_i P_i and its alpha-weighted loss
        rep["switch_aux"] = losses[2]
        rep["L_aux"] = losses[3]
    return rep


def per_config_summary(line):
    """The per-workload figures kept in the headline line's per_config."""
    roof = line["roofline"]
    out = {"value": line["value"], "unit": "tokens/s", "ms_per_step": line["ms_per_step"],
           "e2e_value": line["e2e"]["value"], "steps": line["steps"],
           "dominant": {k: roof.get(k) for k in ("kernel", "bound", "achieved", "peak", "unit", "frac")},
           "expert_ffn_tflops": line["expert_ffn_tflops"],
           "expert_ffn_frac_bf16_peak": line["expert_ffn_frac_bf16_peak"],
           "routing_frac_hbm": line["routing_frac_hbm"], "clocks": line["clocks"],
           "device_status": line["device_status"], "routing": line["routing"]}
    ks = {}
    for name in ("gate_gemm_fp32", "route_topk", "dispatch_place", "combine", "expert_ffn_tcgen05"):
        if name in line["kernels"] and "roofline" in line["kernels"][name]:
            r = line["kernels"][name]["roofline"]
            ks[name] = {"ms_per_step": line["kernels"][name]["ms_per_step"],
                        "share": line["kernels"][name].get("share"), "achieved": r["achieved"],
                        "unit": r["unit"], "frac": r["frac"]}
    out["kernels"] = ks
    return out


def oracle_sample_inputs(w, T_s, inp=None):
    """The oracle's inputs for the first T_s tokens of the workload, as numpy
    arrays (bf16 weights as uint16 bit patterns).  The expert weight arrays
    keep their full [n][...] shapes but only the experts that the sample's
    tokens reach (found by the oracle's own gate, untimed) are filled: the
    arrays start as lazily zeroed pages, so the 8192-expert layer does not
    need its 17 GB of weights in host memory.  inp: the workload's tensors
    already made (on any device); else they are made here, on the GPU when
    there is one (the same generator the GPU path uses)."""
    import numpy as np
    import torch

    from oracle import oracle as orc
    from sparsely_gated_mixture_gate_b200 import synth
    if inp is None:
        inp = synth.make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")

    def host(t):
        if t is None:
            return None
        return synth.bf16_bits(t) if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()

    expert_keys = ("W1", "W2", "b1", "b2")
    out = {key: host(v[:T_s] if key == "x" else v) for key, v in inp.items() if key not in expert_keys}
    used = np.unique(orc.gate_batch(dict(w.cfg(), T=T_s), out)["topk_idx"])
    for key in expert_keys:
        v = inp[key]
        arr = np.zeros(tuple(v.shape), np.uint16 if v.dtype == torch.bfloat16 else np.float32)
        if used.size:
            arr[used] = host(v.index_select(0, torch.from_numpy(used.astype(np.int64)).to(v.device)))
        out[key] = arr
    return out


def oracle_step(w, T_s, backward=False, inp=None):
    """One oracle step on the first T_s tokens: the forward pass, and with
    backward the backward pass too (as a function of no arguments)."""
    from oracle import oracle as orc
    orc.build()
    npin = oracle_sample_inputs(w, T_s, inp)
    cfg = dict(w.cfg(), T=T_s)
    if not backward:
        return lambda: orc.forward(cfg, npin)
    from sparsely_gated_mixture_gate_b200 import synth
    dy = synth.make_dy(w, T=T_s).numpy()

    def both():
        orc.forward(cfg, npin)
        orc.backward(cfg, npin, dy)
    return both


def time_oracle(w, T_s, reps=1, backward=False, inp=None):
    fn = oracle_step(w, T_s, backward, inp)
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    return time.perf_counter() - t0


def cpu_baseline(w, budget_s=12.0, backward=False, inp=None):
    """The oracle (single-threaded C, as it stands) on the first tokens of the
    workload: calibrate on 8 tokens, then run a sample of about budget_s."""
    t8 = time_oracle(w, 8, backward=backward, inp=inp)
    T_s = int(max(8, min(w.T, budget_s / max(t8 / 8, 1e-6))))
    t = time_oracle(w, T_s, backward=backward, inp=inp)
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


def run_stage(args, w):
    """One stage of the layer through its own C-ABI call, timed alone on a
    workload's shapes (optionally with fewer tokens, so that a profiler
    capture stays small): gate (moe_gate), dispatch (moe_dispatch on the
    gate's routing), experts (moe_expert_ffn on a dispatched batch), combine
    (moe_combine).  Prints the mean device time per call; not a bench line."""
    import torch

    from sparsely_gated_mixture_gate_b200 import moe as M
    from sparsely_gated_mixture_gate_b200 import synth
    if args.tokens:
        w = w.with_(T=args.tokens)
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.make_inputs(w, device=dev, experts=args.stage == "experts")
    cfg = M.Config.from_workload(w)
    ws = M.workspace(cfg, dev)
    status = M.new_status(dev)
    x = inp["x"]
    if args.stage == "gate":
        def step():
            return M.gate(cfg, x, inp, ws=ws, status=status)
    else:
        g = M.gate(cfg, x, inp, ws=ws, status=status)
        d = M.dispatch(cfg, x, g["topk_idx"], ws=ws, status=status)
        if args.stage == "dispatch":
            def step():
                return M.dispatch(cfg, x, g["topk_idx"], ws=ws, status=status)
        elif args.stage == "experts":
            def step():
                return M.expert_ffn(cfg, d["x_perm"], d["offsets"], inp, ws=ws, status=status)
        else:
            y_perm = d["x_perm"]  # any expert-row buffer of the right shape

            def step():
                return M.combine(cfg, y_perm, g["topk_gate"], d["row_of"], x, status=status)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    return {"stage": args.stage, "workload": w.name, "T": w.T, "gate": args.gate,
            "ms_per_call": e0.elapsed_time(e1) / args.steps, "calls": args.steps,
            "device_status": M.status_bits(status)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None,
                    help="default: hierarchical (the largest single-GPU workload), also with "
                         "--backward")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--gate", default="fp32", choices=["fp32", "tf32x3"],
                    help="gate projections: fp32 multiply-adds or the 3-pass TF32 tensor-core split")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the short runs of the other workloads (per_config)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time direct library calls instead of a CUDA graph replay of the forward")
    ap.add_argument("--backward", action="store_true",
                    help="time forward + backward (training step) instead of the forward pass")
    ap.add_argument("--no-alt-gate", dest="alt_gate", action="store_false",
                    help="skip the short run of the other gate mode")
    ap.add_argument("--stage", default=None, choices=["gate", "dispatch", "experts", "combine"],
                    help="time one stage's C-ABI call alone (for profiler captures); no bench line")
    ap.add_argument("--tokens", type=int, default=None, help="with --stage: tokens of the batch")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    from sparsely_gated_mixture_gate_b200 import synth
    name = args.workload or "hierarchical"
    w = (synth.WORKLOADS.get(name) or synth.VARIANTS[name]).with_(
        gate_precision=1 if args.gate == "tf32x3" else 0)
    world, rank, local = dist_info()

    if args.stage:
        print(json.dumps(run_stage(args, w)), flush=True)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        cpu = world == 1 and not args.no_cpu_baseline
        line = run_ours(args, w, world, rank, local, cpu_sample=cpu)
        if rank == 0 and line is not None and world == 1 and args.per_config and not args.backward:
            # the five workloads, each a short run of its own (the headline's own figures reused)
            per = {}
            for other, wo in synth.WORKLOADS.items():
                if other == w.name and not w.gate_precision:
                    per[other] = per_config_summary(line)
                    continue
                torch.cuda.empty_cache()
                o = run_ours(args, wo, world, rank, local, steps=min(args.steps, 20), warmup=3,
                             alt_gate=False, fp32_peak=line["fp32_fma_peak"])
                per[other] = per_config_summary(o)
            line["per_config"] = per
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
