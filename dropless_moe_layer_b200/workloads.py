"""Seeded synthetic workloads for the multi-round dropless MoE layer (forward and backward).

This module only draws random inputs. It holds none of the layer's arithmetic:
no routing, no planning, no expert math. Both the CUDA path and the CPU oracle
are fed from here, so that they see bit-identical inputs.

The workloads follow the shapes of the MoE layer described in "Frontier
Pre-training at Microsoft AI (MAI-Base-2)" (Key claims, the multi-round
dropless MoE item under "Scaling MoE") and "Microsoft AI's MAI-Base-2 trained
on 16K GPUs with Muon" (section "Expert groups keep memory fixed when tokens
pile up"): T tokens, hidden size d, E experts, top-k routing, SwiGLU experts
with inner size d_ff, and a fixed per-expert capacity C per round. The pages
give no concrete layer shapes; the five sizes below are synthetic.

Draw order per workload (one generator, seeded with the workload's seed):
router logits (or router weights), expert-bias permutation, x, w_gate_up, w_down.
Every floating-point draw is fp32 and is rounded to bf16 (round-to-nearest-even)
where the tensor is bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    d: int          # hidden size
    E: int          # experts
    k: int          # experts per token
    F: int          # SwiGLU inner size (d_ff)
    C: int          # per-expert token capacity of one round
    router: str     # "logits": fp32 logits are given; "gemm": logits = x @ w_router^T + bias
    bias: str       # "none", "zipf" (expert-popularity bias), "hot" (one expert picked by ~half the tokens)
    zipf_s: float = 0.0
    seed: int = 0

    @property
    def pairs(self) -> int:
        return self.T * self.k


WORKLOADS = [
    Workload("tiny-zipf1", T=256, d=128, E=8, k=2, F=256, C=32,
             router="logits", bias="zipf", zipf_s=1.0, seed=0),
    Workload("4k-zipf1", T=4096, d=1024, E=32, k=4, F=512, C=256,
             router="logits", bias="zipf", zipf_s=1.0, seed=1),
    Workload("16k-uniform", T=16384, d=4096, E=64, k=8, F=1536, C=1024,
             router="logits", bias="none", seed=2),
    Workload("16k-hot-expert", T=16384, d=4096, E=64, k=8, F=1536, C=512,
             router="logits", bias="hot", seed=3),
    Workload("32k-zipf1.2-router-gemm", T=32768, d=7168, E=128, k=8, F=2048, C=2048,
             router="gemm", bias="zipf", zipf_s=1.2, seed=4),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def custom(name: str = "custom", **kw) -> Workload:
    """A workload of arbitrary shape (used by tests for ragged and edge cases)."""
    base = dict(router="logits", bias="none", zipf_s=0.0, seed=0)
    base.update(kw)
    return Workload(name=name, **base)


def _randn(gen: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def _zipf_bias(gen: torch.Generator, E: int, s: float, device) -> torch.Tensor:
    """Expert-popularity bias: expert e gets -s * ln(rank(e) + 1), where rank is a
    seeded permutation of 0..E-1. Before noise, expert popularity then falls off as
    a power of its rank with exponent s (a Zipf(s) law)."""
    perm = torch.randperm(E, generator=gen, device=device)
    return (-s * torch.log(perm.to(torch.float64) + 1.0)).to(torch.float32)


def _hot_expert_bias(gen: torch.Generator, z: torch.Tensor, k: int) -> torch.Tensor:
    """Bias that puts one seeded expert into the top-k of about half of the tokens.

    For token t let gap[t] = (k-th largest logit among the other experts) - z[t, hot].
    The hot expert is selected by t when z[t, hot] + b > that k-th largest logit,
    i.e. when b > gap[t]; b = median(gap) selects it for about half of the tokens.
    """
    T, E = z.shape
    perm = torch.randperm(E, generator=gen, device=z.device)
    hot = int(perm[0])
    others = torch.cat([z[:, :hot], z[:, hot + 1:]], dim=1).to(torch.float64)
    kth = torch.topk(others, k, dim=1).values[:, k - 1]
    gap = kth - z[:, hot].to(torch.float64)
    b = torch.quantile(gap.cpu(), 0.5).item()
    bias = torch.zeros(E, dtype=torch.float32, device=z.device)
    bias[hot] = b
    return bias


def generate(w: Workload, device: str | torch.device = "cpu",
             routing_only: bool = False) -> dict:
    """Draw the inputs of workload `w` on `device`.

    Returns a dict with:
      logits   [T, E] fp32 (router == "logits"; already includes the expert bias), else None
      w_router [E, d] bf16 (router == "gemm"), else None
      bias     [E]    fp32 (router == "gemm"; added to x @ w_router^T), else None
      x        [T, d] bf16
      w_gate_up [E, 2F, d] bf16: rows 0..F-1 are the gate projection W1, rows F..2F-1 the up projection W3
      w_down   [E, d, F] bf16 (W2)
    With routing_only the expert weights and x are skipped (routing-only tests).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    out = dict(logits=None, w_router=None, bias=None, x=None, w_gate_up=None, w_down=None)
    if w.router == "logits":
        z = _randn(gen, (w.T, w.E), device)
        if w.bias == "zipf":
            z = z + _zipf_bias(gen, w.E, w.zipf_s, device)[None, :]
        elif w.bias == "hot":
            z = z + _hot_expert_bias(gen, z, w.k)[None, :]
        elif w.bias != "none":
            raise ValueError(f"unknown bias kind {w.bias!r}")
        out["logits"] = z.contiguous()
    elif w.router == "gemm":
        out["w_router"] = (_randn(gen, (w.E, w.d), device) * (1.0 / math.sqrt(w.d))).to(torch.bfloat16)
        if w.bias == "zipf":
            out["bias"] = _zipf_bias(gen, w.E, w.zipf_s, device)
        elif w.bias == "none":
            out["bias"] = torch.zeros(w.E, dtype=torch.float32, device=device)
        else:
            raise ValueError(f"bias kind {w.bias!r} is not drawn for the router-GEMM form")
    else:
        raise ValueError(f"unknown router kind {w.router!r}")
    if routing_only and w.router == "logits":
        return out
    out["x"] = _randn(gen, (w.T, w.d), device).to(torch.bfloat16)
    if routing_only:
        return out
    out["w_gate_up"] = (_randn(gen, (w.E, 2 * w.F, w.d), device) * 0.02).to(torch.bfloat16)
    out["w_down"] = (_randn(gen, (w.E, w.d, w.F), device) * 0.02).to(torch.bfloat16)
    return out


def generate_dy(w: Workload, device: str | torch.device = "cpu") -> torch.Tensor:
    """The output gradient dy [T, d] fp32 of a backward pass over workload `w`: N(0, 1) drawn
    from its own generator, seeded with the workload's seed + 1000, so that the forward inputs
    above are the same with or without it."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 1000)
    return _randn(gen, (w.T, w.d), device).contiguous()


def bf16_bits(t: Optional[torch.Tensor]):
    """bf16 tensor -> numpy uint16 array of its bit patterns (host copy)."""
    if t is None:
        return None
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def f32_host(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return t.detach().contiguous().cpu().numpy()
