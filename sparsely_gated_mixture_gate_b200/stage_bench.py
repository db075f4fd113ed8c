"""Time one step of the layer through its own C-ABI call on a workload's
shapes (optionally with fewer tokens), e.g. to profile a single kernel family
without holding the whole layer on the device.

    python -m sparsely_gated_mixture_gate_b200.stage_bench --workload many-expert \
        --stage gate --tokens 16384 [--gate tf32x3] [--steps 20]

Stages: gate (moe_gate), dispatch (moe_dispatch on the gate's routing),
experts (moe_expert_ffn on a dispatched batch), combine (moe_combine).
Prints one JSON line with the mean device time per call.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import moe as M
from . import synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="lm-flat")
    ap.add_argument("--stage", default="gate", choices=["gate", "dispatch", "experts", "combine"])
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--gate", default="fp32", choices=["fp32", "tf32x3"])
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()

    w = synth.WORKLOADS.get(args.workload) or synth.VARIANTS[args.workload]
    w = w.with_(gate_precision=1 if args.gate == "tf32x3" else 0)
    if args.tokens:
        w = w.with_(T=args.tokens)
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = synth.make_inputs(w, device=dev, experts=args.stage in ("experts",))
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
    print(json.dumps({"workload": w.name, "T": w.T, "stage": args.stage, "gate": args.gate,
                      "ms_per_call": e0.elapsed_time(e1) / args.steps,
                      "device_status": M.status_bits(status)}))


if __name__ == "__main__":
    main()
