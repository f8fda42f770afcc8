"""Run the layer on one of the synthetic workloads, untimed: a fixed number of steps of
moe_plan + moe_forward (or moe_plan alone) through the C ABI, then a check of the device
status word. Meant as the command line under a profiler (each kernel of the path then
appears a known number of times) or as a quick check that a shape runs on this GPU.

    python -m dropless_moe_layer_b200.run_layer --workload 16k-uniform --steps 2
    python -m dropless_moe_layer_b200.run_layer --workload 32k-zipf1.2-router-gemm \
        --tokens 4096 --plan-only --steps 1

--tokens N replaces the workload's token count (the other sizes, the routing recipe and the
seed stay), so a kernel can be profiled on a case that holds less device memory.
--plan-only skips the expert weights and runs only the router and the planner.
--backward also runs the backward pass (moe_backward) after each forward.
--per-step runs the rounds through moe_round_dispatch / gate_up / down / combine, each its own
kernel, so that every step of a large round can be profiled on its own.
"""
from __future__ import annotations

import argparse
import dataclasses
import json

import torch

from . import moe
from . import workloads as wl


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="4k-zipf1", choices=[w.name for w in wl.WORKLOADS])
    ap.add_argument("--steps", type=int, default=1)
    ap.add_argument("--tokens", type=int, default=0, help="replace the workload's token count")
    ap.add_argument("--plan-only", action="store_true", help="router + planner only (no expert weights)")
    ap.add_argument("--schedule", default="auto", choices=sorted(moe.SCHEDULES))
    ap.add_argument("--borrow", action="store_true")
    ap.add_argument("--backward", action="store_true", help="also run the backward pass after each forward")
    ap.add_argument("--per-step", action="store_true",
                    help="run the rounds through the per-round step calls (stand-alone dispatch, gate/up, "
                         "down and combine kernels) instead of moe_forward")
    args = ap.parse_args()
    w = wl.BY_NAME[args.workload]
    if args.tokens > 0:
        w = dataclasses.replace(w, name=f"{w.name}-T{args.tokens}", T=args.tokens)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    moe.load_library()
    inp = wl.generate(w, dev, routing_only=args.plan_only)
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, device=dev, schedule=args.schedule,
                            borrow=args.borrow)
    y = None if args.plan_only else torch.empty(w.T, w.d, dtype=torch.float32, device=dev)
    dy = wl.generate_dy(w, dev) if args.backward and not args.plan_only else None
    before = moe.launch_count()
    for _ in range(args.steps):
        layer.plan(logits=inp["logits"], x=inp["x"] if w.router == "gemm" else None,
                   w_router=inp["w_router"], bias=inp["bias"])
        if not args.plan_only and args.per_step:
            for r in range(layer.info.R):
                layer.round_step("dispatch", r, inp["x"])
                layer.round_step("gate_up", r, inp["w_gate_up"])
                layer.round_step("down", r, inp["w_down"])
                layer.round_step("combine", r, y)
        elif not args.plan_only:
            layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"], y=y)
        if dy is not None:
            layer.backward(inp["x"], inp["w_gate_up"], inp["w_down"], dy)
    torch.cuda.synchronize(dev)
    status = layer.device_status()
    print(json.dumps({"workload": w.name, "T": w.T, "steps": args.steps, "rounds": layer.info.R,
                      "launches": moe.launch_count() - before, "device_status": status}))
    if status != 0:
        raise SystemExit(f"device status {status}: a kernel wait timed out")


if __name__ == "__main__":
    main()
