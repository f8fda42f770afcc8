"""Benchmark: routed tokens/s of one multi-round dropless MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
                    [--schedule auto|per_round|pipeline] [--borrow]

One step = moe_plan (router top-k + round planner) + moe_forward (all rounds of dispatch ->
gate/up GEMM -> down GEMM -> combine) on one batch, inputs resident in HBM. L2 is flushed
(a 256 MiB write) between timed steps, outside the timed events. Per-step device time comes
from CUDA events on the launching stream; the job time is the max over ranks. The `e2e` key
times the same calls with each step's inputs copied in from pinned host memory and its result
copied out, the copies of neighbouring steps overlapping the compute (the sequential form is
reported beside it). --borrow turns on capacity borrowing (not the plan the metric is defined
on; reported as such in `config`).

Multi-GPU: the layer's experts all live on one GPU, so N GPUs run N independent replicas
(weak scaling, no collective on the data path); torch.distributed is used only for the
barrier and the max-over-ranks of the timing.

--impl reference times the CPU oracle (float64 numpy) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from dropless_moe_layer_b200 import workloads as wl  # noqa: E402

# the largest single-GPU workload of the benchmark (the router GEMM form, 16 rounds)
DEFAULT_WORKLOAD = "32k-zipf1.2-router-gemm"
METRIC = "routed tokens/s per MoE layer fwd (bf16, 1 B200); % of tensor/HBM roofline"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic per launch of a kernel, from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum per launch; summaries in profiles/), valid only while the kernel's
# sources, with comments and blank space taken out, hash to the recorded value.
GEMM_SOURCES = ["sm100.cuh", "gemm_sm100.cuh", "copy_phases.cuh", "kernels.h", "grouped_gemm.cu"]
TRAFFIC = {
    # 16 gate/up launches of one step, dram__bytes_read.sum + dram__bytes_write.sum by ncu on the
    # full workload (one-pass counters), averaged per launch
    ("32k-zipf1.2-router-gemm", "gate_up"): {
        "bytes_per_launch": 43.50506675e9 / 16,
        "sources": GEMM_SOURCES,
        "sources_sha1": "9f976955032251e8e0d5019f3419301efade9e77"},
}


def code_tokens(src):
    """C++ source without its comments, each line's blank space collapsed, blank lines dropped:
    an edit to comments or layout leaves it unchanged, an edit to code does not."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif src[i] in "\"'":
            q, j = src[i], i + 1
            while j < n and src[j] != q:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return "\n".join(" ".join(l.split()) for l in "".join(out).splitlines() if l.strip())


def sources_sha1(files):
    import hashlib
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "dropless_moe_layer_b200", "csrc", f)) as fh:
            h.update(code_tokens(fh.read()).encode())
    return h.hexdigest()


def measured_traffic(workload, kernel):
    rec = TRAFFIC.get((workload, kernel))
    if rec is None or rec["sources_sha1"] != sources_sha1(rec["sources"]):
        return None
    return rec["bytes_per_launch"]


# B200 datasheet figures, for the fractions reported beside the measured ones: dense bf16 tensor
# throughput and HBM3e bandwidth.
DATASHEET = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_config(w, schedule="auto", borrow=False):
    """The `config` dict of the JSON line; both arms (GPU and reference) emit the same one."""
    desc = {"tiny-zipf1": "Zipf(1.0) expert popularity", "4k-zipf1": "Zipf(1.0) expert popularity",
            "16k-uniform": "near-uniform routing", "16k-hot-expert": "one expert picked by ~50% of tokens",
            "32k-zipf1.2-router-gemm": "Zipf(1.2) popularity, logits from the router GEMM"}.get(w.name, "")
    return {"workload": f"{w.name}: T={w.T} d={w.d} E={w.E} top-{w.k} SwiGLU d_ff={w.F} C={w.C}; {desc}",
            "T": w.T, "d": w.d, "E": w.E, "k": w.k, "d_ff": w.F, "C": w.C,
            "router": "fp32 logits given" if w.router == "logits" else "bf16 router GEMM x W_r^T + b",
            "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
            "schedule": schedule, "capacity_borrowing": bool(borrow)}


# ----------------------------------------------------------------------------- CPU oracle timing

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_step(w, host, tokens=None):
    import oracle
    out = oracle.layer(host["x"], host["w_gate_up"], host["w_down"], k=w.k, C=w.C,
                       logits=host["logits"], w_router_bits=host["w_router"], bias=host["bias"],
                       tokens=tokens)
    return out


def host_inputs(w, inp=None):
    """The workload's inputs as host arrays for the oracle: drawn on the CPU, or, when `inp`
    (the device tensors the GPU arm times) is given, copied from there, so that the CPU
    baseline runs on the very inputs of the GPU run."""
    if inp is None:
        inp = wl.generate(w, "cpu")
    return {"x": wl.bf16_bits(inp["x"]), "w_gate_up": wl.bf16_bits(inp["w_gate_up"]),
            "w_down": wl.bf16_bits(inp["w_down"]), "logits": wl.f32_host(inp["logits"]),
            "w_router": wl.bf16_bits(inp["w_router"]), "bias": wl.f32_host(inp["bias"])}


def oracle_sample_plan(w, host, budget_s):
    """Pick a token sample so one oracle step takes about `budget_s` seconds: time a probe
    on 64 tokens (plus the full-T router and plan) and scale."""
    probe = np.arange(min(64, w.T))
    t0 = time.perf_counter()
    oracle_step(w, host, tokens=probe)
    dt = time.perf_counter() - t0
    per_token = dt / len(probe)
    n = w.T if per_token * w.T <= budget_s else max(64, int(budget_s / per_token))
    if n >= w.T:
        return None, f"full workload ({w.T} tokens), router + plan + forward"
    rng = np.random.default_rng(12345)
    tok = np.sort(rng.choice(w.T, size=n, replace=False))
    return tok, (f"seeded sample of {n} of {w.T} tokens (all their top-{w.k} pairs) + the full "
                 f"router/top-k/plan; throughput counts the sampled tokens")


def cpu_baseline(w, min_seconds=10.0, budget_s=15.0, max_steps=50, inp=None):
    """The oracle as it stands on the host cores: repeated steps (each the full workload, or
    a seeded token sample when the full workload would exceed `budget_s`) until at least
    `min_seconds` of CPU work has been timed."""
    host = host_inputs(w, inp)
    tok, sample = oracle_sample_plan(w, host, budget_s)
    n_tok = w.T if tok is None else len(tok)
    times = []
    while sum(times) < min_seconds and len(times) < max_steps:
        t0 = time.perf_counter()
        oracle_step(w, host, tokens=tok)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    return {"value": n_tok * len(times) / total, "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle", "sample": f"{sample}; {len(times)} steps, {total:.1f} s",
            "seconds_per_step": total / len(times)}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    host = host_inputs(w)
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    tok, sample = oracle_sample_plan(w, host, budget)
    n_tok = w.T if tok is None else len(tok)
    for _ in range(args.warmup):
        oracle_step(w, host, tokens=tok)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, host, tokens=tok)
    dt = time.perf_counter() - t0
    value = n_tok * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args.schedule, args.borrow),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
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
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- algorithmic work

def round_rows(w, info, n_plan=None):
    """n[r][e]: rows of expert e in round r (the device plan's when given, else from the loads
    by the no-borrowing rule)."""
    if n_plan is not None:
        return np.asarray(n_plan, dtype=np.int64)
    load = np.array(info.load[:w.E], dtype=np.int64)
    return np.clip(load[None, :] - w.C * np.arange(info.R)[:, None], 0, w.C)


def combine_bytes(w, round_np, rounds=None):
    """combine reads every pair's expert row once (d bf16), writes each token's y row on every
    round it has a pair in, and reads it back on every such round but the first. `rounds`
    restricts the count to a set of rounds."""
    T, d = w.T, w.d
    total = 0
    for t_rounds in round_np.tolist():
        seen = sorted(set(t_rounds))
        for i, r in enumerate(seen):
            if rounds is not None and r not in rounds:
                continue
            total += t_rounds.count(r) * d * 2 + d * 4 + (d * 4 if i > 0 else 0)
    return total


# The library's rule for which copy steps ride on a neighbouring GEMM launch (moe_api.cu,
# moe_forward): small steps always; larger ones when their bytes at the copy warps' rate stay
# below the GEMM's flops at its rate. Mirrored here only to split the work between kernel kinds.
FUSE_COPY_BYTES = 32 << 20
SIDE_COPY_GBS = 2000.0
GEMM_TFLOPS = 1100.0


def ride_plan(w, n, r0):
    """For per-round rounds [0, r0): sets of rounds whose combine rides on the next gate/up launch
    and whose dispatch rides on the previous down launch (n: rows per (round, expert))."""
    rows = [int(v) for v in np.asarray(n).sum(axis=1)]
    R = len(rows)

    def small(r):
        return rows[r] * w.d * 2 <= FUSE_COPY_BYTES

    def combine_rides(rc, rg):
        if small(rc):
            return True
        tokens = min(rows[rc], w.T)
        return (2.0 * rows[rc] + 8.0 * tokens) * w.d / (SIDE_COPY_GBS * 1e9) <= \
            4.0 * rows[rg] * w.d * w.F / (GEMM_TFLOPS * 1e12)

    def dispatch_rides(rd, rg):
        if small(rd):
            return True
        return 4.0 * rows[rd] * w.d / (SIDE_COPY_GBS * 1e9) <= 2.0 * rows[rg] * w.d * w.F / (GEMM_TFLOPS * 1e12)

    comb = {r for r in range(r0) if r + 1 < r0 and combine_rides(r, r + 1)}
    disp = {r + 1 for r in range(r0) if r + 1 < R and dispatch_rides(r + 1, r)}
    return comb, disp


def algorithmic_work(w, info, r0, round_np, n_plan=None):
    """Per kernel kind, the algorithmic units of one step, from the plan alone (padding rows
    C - n never count). Per-round kernels cover rounds [0, r0), the pipelined launch [r0, R).
    GEMMs: flops (tensor-bound). Copies: bytes (HBM-bound). The pipelined launch runs all four
    steps of its rounds; its bound is the larger of its tensor time (6 n d F flops per
    (round, expert)) and its HBM time (the weights, 6 d F bytes per active (round, expert),
    plus its copies' and its GEMM operands' bytes), each at the measured peak."""
    n = round_rows(w, info, n_plan)
    per = n[:r0].sum()
    pipe = n[r0:]
    prow = int(pipe.sum())
    d, F = w.d, w.F
    rode_comb, rode_disp = ride_plan(w, n, r0)
    # stand-alone copy kernels: round 0's dispatch, and the per-round steps that do not ride
    disp_rounds = [r for r in range(min(r0 + 1, info.R)) if r == 0 or r not in rode_disp]
    comb_rounds = {r for r in range(r0) if r not in rode_comb}
    work = {
        "router_gemm": ("hbm", (w.T * w.d * 2 + w.E * w.d * 2 + w.T * w.E * 4) if w.router == "gemm" else 0),
        "topk": ("hbm", w.T * w.E * 4 + w.T * w.k * 8),
        "plan": ("hbm", w.T * w.k * 4 * 6),
        # copy steps that ride on a GEMM launch are done inside that launch (its kind's time)
        "dispatch": ("hbm", 2 * int(sum(n[r].sum() for r in disp_rounds)) * d * 2),
        "gate_up": ("tensor", 4 * int(per) * d * F),
        "down": ("tensor", 2 * int(per) * F * d),
        "combine": ("hbm", combine_bytes(w, round_np, comb_rounds) if comb_rounds else 0),
    }
    if prow:
        flops = 6 * prow * d * F
        active = int((pipe > 0).sum())
        bytes_ = (active * 6 * d * F                  # weights of each active (round, expert)
                  + 2 * prow * d * 2                  # dispatch: x rows in, buf rows out
                  + prow * (d + F) * 2 * 2            # GEMM operands: buf, h (twice), out
                  + combine_bytes(w, round_np, set(range(r0, info.R))))
        work["pipeline"] = ("mixed", (flops, bytes_))
    return work


def layer_roofline_s(w, info, round_np, peaks, tensor_tflops, n_plan=None):
    """Lower bound on one step's time from the layer's algorithmic work alone:
    the bytes of the router GEMM, top-k, plan, the reads of the pairs' x rows and the combine at
    the HBM peak, plus,
    for every expert that has rows in a round, the larger of its GEMM time (6 n d d_ff flops
    at the tensor peak) and the time to stream its weights once (6 d d_ff bytes at the HBM
    peak). Returns (seconds, parts)."""
    n = round_rows(w, info, n_plan)
    d, F = w.d, w.F
    bw = peaks["hbm_gbs"] * 1e9
    pt = tensor_tflops * 1e12
    copy_bytes = ((w.T * w.d * 2 + w.E * w.d * 2 + w.T * w.E * 4) if w.router == "gemm" else 0)
    copy_bytes += w.T * w.E * 4 + w.T * w.k * 8 + w.T * w.k * 4 * 6
    # every pair's x row is read once (the gate/up GEMM gathers it; no dispatch buffer is needed)
    copy_bytes += int(n.sum()) * d * 2 + combine_bytes(w, round_np)
    t_copy = copy_bytes / bw
    n = np.asarray(n)
    active = n[n > 0].astype(np.float64)
    t_expert = float(np.maximum(6.0 * active * d * F / pt, 6.0 * d * F / bw).sum())
    return t_copy + t_expert, {"copy_bytes": int(copy_bytes), "copies_ms": t_copy * 1e3,
                               "experts_ms": t_expert * 1e3, "active_expert_rounds": int(active.size)}


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(value, dist=None, device="cpu"):
    """The job's time: the maximum of `value` over all ranks (identity on one rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, steps, world, job_ms):
    """Whole-job tokens/s: the tokens all ranks processed divided by the job time."""
    return tokens_per_rank * world * steps / (job_ms / 1e3)


# ----------------------------------------------------------------------------- backward pass

BWD_METRIC = ("routed tokens/s per MoE layer backward with per-round recompute (bf16, 1 B200); "
              "% of tensor roofline")


# Tensor-core flops per routed pair, in units of d * d_ff, of each backward GEMM launch kind. The
# recompute and dh run as two launches in rounds whose GEMMs use the CTA-pair form and as one
# (backward_recompute_dh) in the others, so they are rated together ("front" GEMMs).
BWD_KIND_FLOPS = {"backward_recompute": 4, "backward_dh": 2, "backward_recompute_dh": 6, "backward_dx_wgrad": 10}
BWD_FRONT_KINDS = ("backward_recompute", "backward_dh", "backward_recompute_dh")


def backward_flops(w):
    """Tensor-core work of one backward pass: per routed pair the recompute of a and b (4 d d_ff),
    W2^T dy (2 d d_ff), dx = [da | db] W13 (4 d d_ff), dW2 (2 d d_ff) and dW1, dW3 (4 d d_ff)."""
    return 16 * w.T * w.k * w.d * w.F


def backward_roofline_s(w, info, round_np, peaks, tensor_tflops, n_plan=None):
    """Lower bound on one backward pass from its algorithmic work, per round and launch kind
    the larger of its tensor-core time and its DRAM time (the copies at the DRAM peak alone).
    Bytes counted: the round's x and dy rows read once and kept as bf16 rows, the expert
    weights each GEMM reads once per active expert, the recomputed a, b and gate*h written once
    and read where used, [da | db] likewise, the per-pair dx rows, every token's dx read-add-write
    in each round it has pairs in, and the fp32 weight gradients stored (round 0) or
    read-added (later rounds) per active expert. Returns (seconds, parts)."""
    n = round_rows(w, info, n_plan)
    d, F = w.d, w.F
    bw = peaks["hbm_gbs"] * 1e9
    pt = tensor_tflops * 1e12
    parts = {"recompute": 0.0, "dh": 0.0, "dx_wgrad": 0.0, "copies": 0.0}
    rnd = np.asarray(round_np)
    for r in range(n.shape[0]):
        P = int(n[r].sum())
        A = int((n[r] > 0).sum())
        tokens = int((rnd == r).any(axis=1).sum())
        first = int(((rnd == r).any(axis=1) & ~(rnd < r).any(axis=1)).sum())   # tokens whose dx starts here
        w13, w2 = A * 2 * F * d * 2, A * d * F * 2
        grads = A * 3 * d * F * 4 * (1 if r == 0 else 2)
        kinds = {
            "recompute": (4 * P * d * F, P * d * 2 + w13 + P * 2 * F * 2 + P * F * 2),
            "dh": (2 * P * d * F, P * d * 2 + w2 + P * 2 * F * 2 + P * 2 * F * 2),
            "dx_wgrad": (10 * P * d * F,
                         2 * P * 2 * F * 2 + w13 + P * d * 2 + P * F * 2 + P * d * 2 + P * d * 2 + grads),
        }
        for k, (fl, by) in kinds.items():
            parts[k] += max(fl / pt, by / bw)
        parts["copies"] += (P * d * (2 + 4) + P * d * 4 + P * d * 2 + tokens * d * 8 - first * d * 4) / bw
    parts["copies"] += (w.T * w.E * 8 + w.T * w.k * 8) / bw      # dz from the logits and dgate
    return sum(parts.values()), {k: v * 1e3 for k, v in parts.items()}


def backward_cpu_baseline(w, budget_s=12.0):
    """The oracle's backward on the host cores, on a seeded token sample (all the sampled tokens'
    pairs), scaled to tokens/s."""

    import oracle
    host = host_inputs(w)
    z = host["logits"] if host["logits"] is not None else oracle.router_logits(host["x"], host["w_router"],
                                                                              host["bias"])
    dy = wl.generate_dy(w, "cpu").numpy().astype(np.float64)
    rng = np.random.default_rng(12345)

    def run(n):
        tok = np.sort(rng.choice(w.T, size=min(n, w.T), replace=False))
        zs = z[tok]
        t0 = time.perf_counter()
        oracle.backward(host["x"][tok], host["w_gate_up"], host["w_down"], zs, oracle.select_topk(zs, w.k),
                        dy[tok])
        return len(tok), time.perf_counter() - t0

    n, dt = run(64)
    n_tok = w.T if dt / n * w.T <= budget_s else max(64, int(budget_s / (dt / n)))
    n, dt = run(n_tok)
    return {"value": n / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"seeded sample of {n} of {w.T} tokens (all their top-{w.k} pairs), oracle.backward, "
                      f"{dt:.1f} s"}


def bench_backward(args, w):
    import torch

    from dropless_moe_layer_b200 import moe

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    moe.load_library()
    inp = wl.generate(w, dev)
    dy = wl.generate_dy(w, dev)
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, device=dev)
    layer.plan(logits=inp["logits"], x=inp["x"] if w.router == "gemm" else None,
               w_router=inp["w_router"], bias=inp["bias"])
    layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    info = layer.info
    bws_bytes = moe.backward_workspace_bytes(layer.shape)
    bws = torch.empty(bws_bytes, dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = dict(dx=torch.empty(w.T, w.d, **f32), dw_gate_up=torch.empty(w.E, 2 * w.F, w.d, **f32),
             dw_down=torch.empty(w.E, w.d, w.F, **f32), dz=torch.empty(w.T, w.E, **f32))
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        moe.backward(layer.shape, info, layer.ws, layer.ws_bytes, int(bws.data_ptr()), bws_bytes,
                     int(inp["x"].data_ptr()), int(inp["w_gate_up"].data_ptr()), int(inp["w_down"].data_ptr()),
                     int(dy.data_ptr()), int(g["dx"].data_ptr()), int(g["dw_gate_up"].data_ptr()),
                     int(g["dw_down"].data_ptr()), int(g["dz"].data_ptr()), int(stream.cuda_stream))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = "0"
    clocks = ClockSampler(gpu_id)
    clocks.start()
    t_end = time.perf_counter() + 0.6       # the clock record covers the timed steps (100 ms samples)
    while time.perf_counter() < t_end:
        step()
    torch.cuda.synchronize(dev)
    launches0 = moe.launch_count()
    host_s = 0.0   # host time to enqueue the calls (their launches, events and waits)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        h0 = time.perf_counter()
        step()
        host_s += time.perf_counter() - h0
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    launches = moe.launch_count() - launches0
    t_end = time.perf_counter() + 0.4
    while time.perf_counter() < t_end:
        step()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    total_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends))
    # one more pass with per-launch events, for the per-kernel split
    moe.profile_enable(True)
    flush.fill_(1)
    step()
    torch.cuda.synchronize(dev)
    prof = {k: v for k, v in moe.profile_read().items() if v[0] > 0}
    moe.profile_enable(False)
    status = layer.device_status()
    peaks, peak_src = load_peaks()
    flops = backward_flops(w)
    gemm_ms = sum(prof[k][1] for k in moe.BACKWARD_GEMM_KINDS if k in prof)
    front_ms = sum(prof[k][1] for k in BWD_FRONT_KINDS if k in prof)
    achieved = flops / (gemm_ms / 1e3) / 1e12
    power_capped = bool(clk and "sw_power_cap" in clk.get("reasons", []))
    tensor_key = "bf16_tflops_sustained" if power_capped and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    peak = peaks[tensor_key]
    ms = total_ms / args.steps
    pass_s, pass_parts = backward_roofline_s(w, info, layer.plan_tensors()["round"].cpu().numpy(), peaks, peak,
                                             layer.plan_tensors()["n"].cpu().numpy())
    line = {
        "metric": BWD_METRIC, "pass": "backward", "value": w.T / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w), "rounds": info.R,
        "roofline": {"kernel": "backward GEMMs (" + ", ".join(moe.BACKWARD_GEMM_KINDS) + ")", "bound": "tensor",
                     "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} ({tensor_key})", "traffic": None,
                     "frac_vs_burst": achieved / peaks["bf16_tflops"],
                     "frac_vs_datasheet": achieved / DATASHEET["bf16_tflops"], "flops_per_step": flops},
        "whole_pass_tflops": flops / (ms / 1e3) / 1e12,
        "host_enqueue_ms_per_call": host_s * 1e3 / args.steps,
        "pass_frac": pass_s * 1e3 / ms,
        "pass_roofline": {"ms": pass_s * 1e3, **{k + "_ms": round(v, 4) for k, v in pass_parts.items()},
                          "peaks": f"{peak_src}: hbm_gbs {peaks['hbm_gbs']}, {tensor_key} {peak}",
                          "formula": "per round and launch kind max(tensor flops at the peak, algorithmic DRAM "
                                     "bytes at the copy peak); copies at the copy peak"},
        "kernels": {k: dict({"launches": c, "ms": round(t, 4)},
                            **({"TFLOP/s": round(BWD_KIND_FLOPS[k] * w.T * w.k * w.d * w.F / (t / 1e3) / 1e12, 1)}
                               if k == "backward_dx_wgrad" else {}))
                    for k, (c, t) in prof.items()},
        "front_gemms_TFLOP/s": round(6 * w.T * w.k * w.d * w.F / (front_ms / 1e3) / 1e12, 1) if front_ms > 0 else None,
        "cpu_baseline": None if args.no_cpu_baseline else backward_cpu_baseline(w),
        "gpu_launches": launches,
        "clocks": clk,
        "device_status": status,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU benchmark

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=[x.name for x in wl.WORKLOADS])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", default="auto", choices=["auto", "per_round", "pipeline"],
                    help="moe_forward launch schedule (the layer's results are identical)")
    ap.add_argument("--borrow", action="store_true",
                    help="capacity borrowing between experts (fewer rounds; not the default plan)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (moe_backward) instead of the forward step; prints "
                         "its own line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = wl.BY_NAME[args.workload]
    if args.backward:
        bench_backward(args, w)
        return
    if args.impl == "reference":
        run_reference(args, w)
        return

    import torch

    from dropless_moe_layer_b200 import moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    moe.load_library()
    inp = wl.generate(w, dev)
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, device=dev, schedule=args.schedule,
                            borrow=args.borrow)
    y = torch.empty(w.T, w.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        layer.plan(logits=inp["logits"], x=inp["x"] if w.router == "gemm" else None,
                   w_router=inp["w_router"], bias=inp["bias"])
        layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"], y=y)

    def timed(K, profile=False):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        if profile:
            moe.profile_enable(True)
        launches0 = moe.launch_count()
        for i in range(K):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        launches = moe.launch_count() - launches0
        prof = moe.profile_read() if profile else None
        if profile:
            moe.profile_enable(False)
        if dist is not None:
            dist.barrier()
        ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
        return ms, launches, prof

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if layer.device_status() != 0:
        raise SystemExit("kernel wait timed out during warm-up")

    # nvidia-smi samples every 100 ms, longer than a short timed region: keep the GPU under
    # the same load (untimed steps) for ~0.5 s on each side so the clock record covers it.
    def load_for(seconds):
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            step()
        torch.cuda.synchronize(dev)

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    load_for(0.6)
    total_ms, launches, _ = timed(args.steps)
    load_for(0.4)
    clk = clocks.stop()
    total_ms = max_over_ranks(total_ms, dist, dev)
    value = job_throughput(w.T, args.steps, world, total_ms)

    # second timed pass with per-kernel events (for the roofline of the dominant kernel)
    _, _, prof = timed(args.steps, profile=True)
    info = layer.info
    rnd = layer.plan_tensors()["round"].cpu().numpy()
    peaks, peak_src = load_peaks()
    kinds = {k: v for k, v in prof.items() if v[0] > 0}
    # per-round launches cover rounds [0, r0): one gate/up launch per round and step
    r0 = kinds["gate_up"][0] // args.steps if "gate_up" in kinds else 0
    if "pipeline" not in kinds:
        r0 = info.R
    work = algorithmic_work(w, info, r0, rnd, layer.plan_tensors()["n"].cpu().numpy())

    def resolve(kind):
        """(bound, units per step) of a kind; a mixed launch takes its slower roofline."""
        b, u = work[kind]
        if b != "mixed":
            return b, u
        flops, bytes_ = u
        t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
        t_hbm = bytes_ / (peaks["hbm_gbs"] * 1e9)
        return ("tensor", flops) if t_tensor >= t_hbm else ("hbm", bytes_)

    dom = max(kinds, key=lambda k: kinds[k][1])
    bound, units_per_step = resolve(dom)
    cnt, ms = kinds[dom]
    per_launch_units = units_per_step * args.steps / cnt
    avg_launch_s = ms / cnt / 1e3
    # A GEMM timed inside a long run of steps that holds the GPU at its power cap is compared
    # with the sustained bf16 peak (a cuBLAS loop under the same cap); otherwise with the burst
    # peak. The fraction against the burst peak is reported beside it either way.
    power_capped = bool(clk and "sw_power_cap" in clk.get("reasons", []))
    tensor_key = "bf16_tflops_sustained" if power_capped and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    if bound == "tensor":
        achieved, peak, unit = per_launch_units / avg_launch_s / 1e12, peaks[tensor_key], "TFLOP/s"
    else:
        achieved, peak, unit = per_launch_units / avg_launch_s / 1e9, peaks["hbm_gbs"], "GB/s"
    layer_s, layer_parts = layer_roofline_s(w, info, rnd, peaks, peaks[tensor_key],
                                            layer.plan_tensors()["n"].cpu().numpy())
    # the same bound with the datasheet's peaks (dense bf16 2.25 PFLOP/s, HBM3e 8 TB/s)
    layer_ds_s, _ = layer_roofline_s(w, info, rnd, {"hbm_gbs": DATASHEET["hbm_gbs"]}, DATASHEET["bf16_tflops"],
                                     layer.plan_tensors()["n"].cpu().numpy())
    per_kernel = {}
    for k, (c, t) in kinds.items():
        b, u = resolve(k)
        rate = u * args.steps / (t / 1e3)
        per_kernel[k] = {"launches": c, "ms_total": round(t, 4), "share": round(t / sum(v[1] for v in kinds.values()), 4),
                         "bound": b, ("TFLOP/s" if b == "tensor" else "GB/s"): round(rate / (1e12 if b == "tensor" else 1e9), 2)}
    if "pipeline" in work:
        flops, bytes_ = work["pipeline"][1]
        per_kernel.setdefault("pipeline", {}).update(
            {"rounds": [r0, info.R], "flops_per_step": flops, "bytes_per_step": bytes_})

    # end to end through the public API from pinned host buffers
    host_x = inp["x"].cpu().pin_memory()
    host_z = inp["logits"].cpu().pin_memory() if inp["logits"] is not None else None
    host_y = torch.empty(w.T, w.d, dtype=torch.float32).pin_memory()
    dx = torch.empty_like(inp["x"])
    dz = torch.empty_like(inp["logits"]) if host_z is not None else None
    h2d = host_x.numel() * 2 + (host_z.numel() * 4 if host_z is not None else 0)
    d2h = host_y.numel() * 4

    def e2e_step():
        dx.copy_(host_x, non_blocking=True)
        if dz is not None:
            dz.copy_(host_z, non_blocking=True)
        layer.plan(logits=dz, x=dx if w.router == "gemm" else None, w_router=inp["w_router"], bias=inp["bias"])
        layer.forward(dx, inp["w_gate_up"], inp["w_down"], y=y)
        host_y.copy_(y, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev0.record(stream)
        e2e_step()
        ev1.record(stream)
        ev1.synchronize()
        e2e_ms += ev0.elapsed_time(ev1)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    e2e_seq_value = job_throughput(w.T, args.steps, world, e2e_ms)

    # Pipelined end to end, as a server would run the layer: step i+1's inputs go host->device
    # and step i-1's result device->host while step i computes (a stream per direction,
    # device tensors double-buffered, events ordering every reuse). Every step's copies are
    # inside the timed region, which runs from before the first input copy to after the last
    # result copy. No L2 flush here: the weights alone (E x 6 d d_ff bytes) exceed the L2.
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dxs = [torch.empty_like(inp["x"]) for _ in range(2)]
    dzs = [torch.empty_like(inp["logits"]) if host_z is not None else None for _ in range(2)]
    ys = [torch.empty(w.T, w.d, dtype=torch.float32, device=dev) for _ in range(2)]
    host_ys = [torch.empty(w.T, w.d, dtype=torch.float32).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]     # slot's inputs on the device
    ev_used = [torch.cuda.Event() for _ in range(2)]   # slot's step computed (inputs free, y ready)
    ev_out = [torch.cuda.Event() for _ in range(2)]    # slot's y on the host

    def p_h2d(i):
        sl = i & 1
        h2d_stream.wait_event(ev_used[sl])
        with torch.cuda.stream(h2d_stream):
            dxs[sl].copy_(host_x, non_blocking=True)
            if dzs[sl] is not None:
                dzs[sl].copy_(host_z, non_blocking=True)
        ev_in[sl].record(h2d_stream)

    def p_compute(i):
        sl = i & 1
        stream.wait_event(ev_in[sl])
        stream.wait_event(ev_out[sl])
        layer.plan(logits=dzs[sl], x=dxs[sl] if w.router == "gemm" else None, w_router=inp["w_router"],
                   bias=inp["bias"], stream=stream)
        layer.forward(dxs[sl], inp["w_gate_up"], inp["w_down"], y=ys[sl], stream=stream)
        ev_used[sl].record(stream)

    def p_d2h(i):
        sl = i & 1
        d2h_stream.wait_event(ev_used[sl])
        with torch.cuda.stream(d2h_stream):
            host_ys[sl].copy_(ys[sl], non_blocking=True)
        ev_out[sl].record(d2h_stream)

    def pipelined(K):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        h2d_stream.wait_event(start)
        d2h_stream.wait_event(start)
        p_h2d(0)
        for i in range(K):
            if i + 1 < K:
                p_h2d(i + 1)
            p_compute(i)
            p_d2h(i)
        stream.wait_event(ev_out[(K - 1) & 1])
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end)

    pipelined(3)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e2e_pipe_ms = max_over_ranks(pipelined(args.steps), dist, dev)
    e2e_value = job_throughput(w.T, args.steps, world, e2e_pipe_ms)
    torch.cuda.synchronize(dev)
    status = layer.device_status()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inp=inp)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, args.schedule, args.borrow),
            "rounds": info.R, "pipelined_rounds": [r0, info.R], "routed_pairs_per_s": value * w.k,
            "roofline": dict({"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                              "frac": achieved / peak,
                              "peak_source": f"{peak_src} ({tensor_key if bound == 'tensor' else 'hbm_gbs copy'})",
                              "traffic": measured_traffic(w.name, dom)},
                             **({"frac_vs_burst": achieved / peaks["bf16_tflops"]} if bound == "tensor" else {}),
                             frac_vs_datasheet=achieved / (DATASHEET["bf16_tflops"] if bound == "tensor"
                                                           else DATASHEET["hbm_gbs"])),
            "layer_frac": layer_s * 1e3 / (total_ms / args.steps),
            "layer_frac_vs_datasheet": layer_ds_s * 1e3 / (total_ms / args.steps),
            "layer_roofline": dict(layer_parts, ms=layer_s * 1e3,
                                   peaks=f"{peak_src}: hbm_gbs {peaks['hbm_gbs']}, {tensor_key} {peaks[tensor_key]}",
                                   formula="router/top-k/plan/dispatch/combine bytes at HBM + sum over active "
                                           "(round, expert) of max(6 n d d_ff flops at tensor, 6 d d_ff weight "
                                           "bytes at HBM)"),
            "kernels": per_kernel,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_pipe_ms / args.steps,
                    "overlap": "step i+1's inputs and step i-1's result cross the bus while step i computes",
                    "l2": "not flushed between these steps; each step streams all expert weights "
                          f"({w.E * 6 * w.d * w.F / 1e6:.0f} MB), more than the 126 MB L2",
                    "sequential": {"value": e2e_seq_value, "ms_per_step": e2e_ms / args.steps}},
            "gpu_launches": launches,
            "clocks": clk,
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
