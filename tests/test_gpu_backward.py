"""GPU parity of the backward pass with per-round recompute (through the C ABI) against the
CPU oracle's backward.

Bars: every gradient is built from bf16 operands with fp32 accumulation (dy, the recomputed
a and b, gate * h, da and db are rounded to bf16, 2^-9 relative each) and fp32 reductions, so
each gradient is compared as max|g - g_ref| / max|g_ref| <= 2e-2, the bar of the forward's y.
The oracle takes the same seeded inputs and the logits the GPU's plan used.
"""
import numpy as np
import pytest
import torch

import oracle
from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

pytestmark = pytest.mark.gpu

G_TOL = 2e-2
NAMES = ("dx", "dw_gate_up", "dw_down", "dz")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def rel_err(got, ref):
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def run_backward(w, inp, dy, renorm=False, borrow=False):
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, renorm=renorm, borrow=borrow)
    layer(inp["x"], inp["w_gate_up"], inp["w_down"], logits=inp["logits"])
    g = layer.backward(inp["x"], inp["w_gate_up"], inp["w_down"], dy)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, g


def check(w, inp, dy, g, renorm=False):
    z = inp["logits"].cpu().numpy()
    idx = oracle.select_topk(z, w.k)
    ref = oracle.backward(wl.bf16_bits(inp["x"]), wl.bf16_bits(inp["w_gate_up"]), wl.bf16_bits(inp["w_down"]),
                          z, idx, dy.cpu().numpy().astype(np.float64), renorm=renorm)
    errs = {n: rel_err(g[n].cpu().numpy().astype(np.float64), ref[n]) for n in NAMES}
    assert all(e <= G_TOL for e in errs.values()), errs
    return errs


@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_backward_full_parity(name):
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g = run_backward(w, inp, dy)
    assert layer.info.R >= 2
    check(w, inp, dy, g)


EDGE = [
    dict(T=1000, d=192, E=6, k=2, F=320, C=100),       # ragged T, d and d_ff not multiples of 128
    dict(T=40, d=64, E=4, k=2, F=64, C=1),             # C = 1: many rounds of one row
    dict(T=300, d=128, E=5, k=3, F=128, C=1000),       # C > T: one round
    dict(T=257, d=128, E=1, k=1, F=192, C=64),         # one expert: dz = 0
    dict(T=200, d=256, E=8, k=8, F=128, C=77),         # k = E
    dict(T=512, d=128, E=256, k=16, F=64, C=40),       # widest routing
    dict(T=1, d=128, E=8, k=2, F=128, C=3),            # one token
    dict(T=700, d=64, E=16, k=4, F=256, C=130),        # C not a multiple of the 128-row tile
]


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: "T{T}-d{d}-E{E}-k{k}-F{F}-C{C}".format(**c))
def test_backward_edge_shapes(cfg):
    w = wl.custom(name="edge", T=cfg["T"], d=cfg["d"], E=cfg["E"], k=cfg["k"], F=cfg["F"], C=cfg["C"],
                  bias="zipf", zipf_s=1.0, seed=cfg["T"])
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g = run_backward(w, inp, dy)
    if w.E == 1:
        assert torch.count_nonzero(g["dz"]) == 0
    check(w, inp, dy, g)


def test_backward_renormalised_gates():
    w = wl.custom(name="renorm", T=333, d=128, E=12, k=3, F=128, C=50, bias="zipf", zipf_s=1.0, seed=5)
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g = run_backward(w, inp, dy, renorm=True)
    check(w, inp, dy, g, renorm=True)


def test_backward_is_deterministic():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g1 = run_backward(w, inp, dy)
    g2 = layer.backward(inp["x"], inp["w_gate_up"], inp["w_down"], dy)
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(g1[n], g2[n]), n


OVERLAP_CASES = ["4k-zipf1", "16k-hot-expert", "C1", "C130"]


@pytest.mark.parametrize("name", OVERLAP_CASES)
def test_backward_overlapped_rounds_equal_one_at_a_time(name):
    """Rounds in the second buffer set overlap the round before (two streams); the per-round
    schedule runs every round in the first set, one after another. The gradients are bitwise
    equal: the weight gradients and dx are accumulated in round order either way, and a round's
    arithmetic does not depend on which set its rows live in."""
    if name in wl.BY_NAME:
        w = wl.BY_NAME[name]
    else:
        cfg = {"C1": EDGE[1], "C130": EDGE[7]}[name]
        w = wl.custom(name="edge", T=cfg["T"], d=cfg["d"], E=cfg["E"], k=cfg["k"], F=cfg["F"], C=cfg["C"],
                      bias="zipf", zipf_s=1.0, seed=cfg["T"])
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    out = {}
    for sched in ("auto", "per_round"):
        layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, schedule=sched)
        layer(inp["x"], inp["w_gate_up"], inp["w_down"], logits=inp["logits"])
        assert layer.info.R >= 3
        out[sched] = layer.backward(inp["x"], inp["w_gate_up"], inp["w_down"], dy)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        del layer
    for n in NAMES:
        assert torch.equal(out["auto"][n], out["per_round"][n]), n


def test_backward_empty_batch():
    """No tokens: no rounds; the weight gradients are all zero."""
    layer = moe.DroplessMoE(0, 128, 8, 2, 128, 16)
    layer.plan(logits=torch.empty(0, 8, dtype=torch.float32, device="cuda"))
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    w13 = torch.randn(8, 256, 128, device="cuda").to(torch.bfloat16)
    w2 = torch.randn(8, 128, 128, device="cuda").to(torch.bfloat16)
    layer.forward(x, w13, w2)
    g = layer.backward(x, w13, w2, torch.empty(0, 128, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert g["dx"].shape == (0, 128) and g["dz"].shape == (0, 8)
    assert torch.count_nonzero(g["dw_gate_up"]) == 0 and torch.count_nonzero(g["dw_down"]) == 0


@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_backward_borrow_full_parity(name):
    """With capacity borrowing the rounds hold pooled rows; the gradients do not depend on the
    plan."""
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g = run_backward(w, inp, dy, borrow=True)
    assert layer.info.R < (max(layer.info.load[:w.E]) + w.C - 1) // w.C    # borrowing saved rounds
    check(w, inp, dy, g)


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: "T{T}-d{d}-E{E}-k{k}-F{F}-C{C}".format(**c))
def test_backward_borrow_edge_shapes(cfg):
    w = wl.custom(name="edge", T=cfg["T"], d=cfg["d"], E=cfg["E"], k=cfg["k"], F=cfg["F"], C=cfg["C"],
                  bias="zipf", zipf_s=1.0, seed=cfg["T"])
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g = run_backward(w, inp, dy, borrow=True)
    check(w, inp, dy, g)


# Round 0 of this shape holds 16 experts x ~512 rows: 32 row blocks of 256 times 4 to 8 column
# tiles, enough for every SM pair, so its GEMMs run in the CTA-pair form (256-row tiles, ragged
# where an expert has fewer than 512 rows); the short later rounds run in the single-CTA form.
PAIR_SHAPE = dict(T=4096, d=1024, E=16, k=2, F=1024, C=512)


@pytest.mark.parametrize("borrow", [False, True], ids=["per-expert", "borrow"])
def test_backward_pair_form_full_parity(borrow):
    w = wl.custom(name="pair", bias="none", seed=11, **PAIR_SHAPE)
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    layer, g = run_backward(w, inp, dy, borrow=borrow)
    check(w, inp, dy, g)
    g2 = layer.backward(inp["x"], inp["w_gate_up"], inp["w_down"], dy)
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(g[n], g2[n]), n


class _LazyExperts:
    """Expert weights fetched from the GPU one expert at a time, as bf16 bits."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, e):
        return wl.bf16_bits(self.t[e])


def _sampled_backward_check(w, pick_experts):
    """Full-size backward on the GPU; dx and dz of 16 sampled tokens and the weight gradients of
    the experts `pick_experts(load)` names, against the oracle's entries (each token's and each
    expert's pairs alone)."""
    inp = wl.generate(w, "cuda")
    dy = wl.generate_dy(w, "cuda")
    if w.router == "gemm":
        layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C)
        layer(inp["x"], inp["w_gate_up"], inp["w_down"], w_router=inp["w_router"], bias=inp["bias"])
        g = layer.backward(inp["x"], inp["w_gate_up"], inp["w_down"], dy)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        z = layer.plan_tensors()["logits"].cpu().numpy()     # the logits the GPU routed on
    else:
        layer, g = run_backward(w, inp, dy)
        z = inp["logits"].cpu().numpy()
    assert layer.info.R >= 2
    idx = oracle.select_topk(z, w.k)
    load = np.bincount(idx.ravel(), minlength=w.E)
    experts = pick_experts(load)
    rng = np.random.default_rng(0)
    tokens = np.concatenate([[0, w.T - 1], rng.choice(w.T, 14, replace=False)])
    ref = oracle.backward_sampled(wl.bf16_bits(inp["x"]), _LazyExperts(inp["w_gate_up"]),
                                  _LazyExperts(inp["w_down"]), z, idx, dy.cpu().numpy().astype(np.float64),
                                  tokens, experts)
    got = {"dx": g["dx"][tokens], "dz": g["dz"][tokens],
           "dw_gate_up": g["dw_gate_up"][experts], "dw_down": g["dw_down"][experts]}
    errs = {n: rel_err(got[n].cpu().numpy().astype(np.float64), ref[n]) for n in got}
    assert all(e <= G_TOL for e in errs.values()), errs


def test_backward_16k_uniform_sampled_parity():
    """16k-uniform at full size: the experts with the most and the fewest pairs."""
    _sampled_backward_check(wl.BY_NAME["16k-uniform"], lambda load: [int(np.argmax(load)), int(np.argmin(load))])


def test_backward_32k_sampled_parity():
    """The bench's default workload at full size (router-GEMM logits, 16 rounds, round 0 in the
    pair form with most experts' rows in one short block): the experts with the fewest pairs and
    with the median count (the hottest expert's 32k rows would take the float64 oracle minutes)."""
    def pick(load):
        order = np.argsort(load, kind="stable")
        return [int(order[0]), int(order[len(order) // 2])]
    _sampled_backward_check(wl.BY_NAME["32k-zipf1.2-router-gemm"], pick)
