"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars (from the arithmetic of each step):
  * routing (selected experts, rounds, slots, loads, R, n) is integer work decided by
    fp32 comparisons of the same fp32 logits on both sides: bit-exact;
  * gates: fp32 softmax on the GPU vs float64 in the oracle; relative error bounded by
    about E * 2^-24 + a few ulp of expf: rtol 1e-5;
  * the dispatch buffer is a copy: bit-exact;
  * expert outputs and y: bf16 weights with fp32 accumulation and bf16 rounding of the
    SwiGLU activations and of each expert output (2^-9 relative each):
    max|y - y_ref| / max|y_ref| <= 2e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

pytestmark = pytest.mark.gpu

Y_TOL = 2e-2
GATE_RTOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def bits(t):
    return wl.bf16_bits(t)


class LazyExperts:
    """Expert weights fetched from the GPU one expert at a time, as bf16 bits."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, e):
        return bits(self.t[e])


class LazyRows:
    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, rows):
        return bits(self.t[torch.as_tensor(np.asarray(rows), device=self.t.device)])


def rel_err(got, ref):
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


SCHEDULES = ["auto", "per_round", "pipeline"]


def run_gpu(w, inp, C=None, renorm=False, schedule="auto", borrow=False):
    C = C or w.C
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, C, renorm=renorm, schedule=schedule, borrow=borrow)
    y = layer(inp["x"], inp["w_gate_up"], inp["w_down"], logits=inp["logits"],
              w_router=inp["w_router"], bias=inp["bias"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, y


def check_plan(layer, w, C, z, renorm=False, borrow=False):
    """Routing and plan bit-exact against the oracle on the logits the GPU used."""
    pt = layer.plan_tensors()
    idx_ref = oracle.select_topk(z, w.k)
    np.testing.assert_array_equal(pt["topk_idx"].cpu().numpy(), idx_ref)
    g_ref = oracle.gates(z, idx_ref, renorm)
    np.testing.assert_allclose(pt["gate"].cpu().numpy(), g_ref, rtol=GATE_RTOL, atol=1e-12)
    p = oracle.plan_borrow(idx_ref, w.E, C) if borrow else oracle.plan(idx_ref, w.E, C)
    info = layer.info
    assert info.R == p["R"] and info.max_load == p["max_load"]
    assert list(info.load)[:w.E] == list(p["load"])
    np.testing.assert_array_equal(pt["round"].cpu().numpy(), p["round"])
    np.testing.assert_array_equal(pt["slot"].cpu().numpy(), p["slot"])
    np.testing.assert_array_equal(pt["load"].cpu().numpy(), p["load"])
    np.testing.assert_array_equal(pt["offsets"].cpu().numpy(), p["offsets"])
    np.testing.assert_array_equal(pt["n"].cpu().numpy(), p["n"])
    return idx_ref, g_ref, p


def sample_tokens(T, p, count, seed):
    rng = np.random.default_rng(seed)
    tok = set(rng.choice(T, size=min(count, T), replace=False).tolist()) | {0, T - 1}
    last = np.nonzero((p["round"] == p["R"] - 1).any(axis=1))[0]       # tokens in the last round
    tok |= set(last[:8].tolist())
    spread = np.nonzero((p["round"].max(1) - p["round"].min(1)) >= 2)[0]  # pairs several rounds apart
    tok |= set(spread[:8].tolist())
    return np.array(sorted(tok), dtype=np.int64)


# ----------------------------------------------------------------------------- workloads

@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_workload_full_parity(name, schedule):
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, schedule=schedule)
    z = inp["logits"].cpu().numpy()
    idx, g, p = check_plan(layer, w, w.C, z)
    assert p["R"] >= 2
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


@pytest.mark.parametrize("name", ["16k-uniform", "16k-hot-expert", "32k-zipf1.2-router-gemm"])
def test_workload_sampled_parity(name):
    """Full-size workloads in the benchmark's launch configuration; the plan is checked on
    every token, y on a seeded token sample (each token's output depends on its row only)."""
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp)
    if w.router == "gemm":
        z = layer.plan_tensors()["logits"].cpu().numpy()
    else:
        z = inp["logits"].cpu().numpy()
    idx, g, p = check_plan(layer, w, w.C, z)
    tok = sample_tokens(w.T, p, 48 if w.router == "gemm" else 96, seed=w.seed)
    if w.router == "gemm":
        xs = bits(inp["x"][torch.as_tensor(tok, device="cuda")])
        z_ref = oracle.router_logits(xs, bits(inp["w_router"]), inp["bias"].cpu().numpy())
        assert np.max(np.abs(z[tok] - z_ref)) <= 1e-4 * np.max(np.abs(z_ref))
    x_rows = LazyRows(inp["x"])
    ref = oracle.forward(x_rows, LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g,
                         tokens=tok)
    got = y[torch.as_tensor(tok, device="cuda")].cpu().numpy().astype(np.float64)
    assert rel_err(got, ref) <= Y_TOL
    assert np.all(np.isfinite(y.cpu().numpy()))


# ----------------------------------------------------------------------------- per-step parity

@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_round_steps_against_oracle(name):
    """dispatch bit-exact, then each expert GEMM on the GPU's own inputs, round by round."""
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C)
    info = layer.plan(logits=inp["logits"])
    z = inp["logits"].cpu().numpy()
    idx, g, p = check_plan(layer, w, w.C, z)
    xb = bits(inp["x"])
    y = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    W13, W2 = LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"])
    for r in range(info.R):
        layer.round_step("dispatch", r, inp["x"])
        buf = bits(layer.round_buffer())
        rows = oracle.round_rows(p, idx, r)
        for (e, s, t, j) in rows:
            assert np.array_equal(buf[e, s], xb[t]), (r, e, s, t)
        layer.round_step("gate_up", r, inp["w_gate_up"])
        h = bits(layer.hidden_buffer())
        layer.round_step("down", r, inp["w_down"])
        out = bits(layer.output_buffer())
        for e in range(w.E):
            n = int(p["n"][r, e])
            if n == 0:
                continue
            a = oracle.bf16_to_f64(buf[e, :n])
            h_ref = oracle.expert_hidden(a, oracle.bf16_to_f64(W13[e]))
            assert rel_err(oracle.bf16_to_f64(h[e, :n]), h_ref) <= 1e-2, (r, e)
            o_ref = oracle.bf16_to_f64(h[e, :n]) @ oracle.bf16_to_f64(W2[e]).T
            assert rel_err(oracle.bf16_to_f64(out[e, :n]), o_ref) <= 1e-2, (r, e)
        layer.round_step("combine", r, y)
    torch.cuda.synchronize()
    ref = oracle.forward(xb, W13, W2, idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


# ----------------------------------------------------------------------------- edge cases

EDGE = [
    dict(T=1000, d=192, E=6, k=2, F=320, C=100),       # ragged T, d % 128 != 0, d_ff % 128 != 0
    dict(T=40, d=64, E=4, k=2, F=64, C=1),             # C = 1: one round per token of the busiest expert
    dict(T=300, d=128, E=5, k=3, F=128, C=1000),       # C > T: a single round
    dict(T=257, d=128, E=1, k=1, F=192, C=64),         # one expert: a dense MLP in rounds
    dict(T=200, d=256, E=8, k=8, F=128, C=77),         # k = E
    dict(T=512, d=128, E=256, k=16, F=64, C=40),       # widest routing
    dict(T=1, d=128, E=8, k=2, F=128, C=3),            # one token
    dict(T=700, d=64, E=16, k=4, F=256, C=130),        # C not a multiple of the 128-row tile
]


@pytest.mark.parametrize("schedule", ["per_round", "pipeline"])
@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: "T{T}-d{d}-E{E}-k{k}-F{F}-C{C}".format(**c))
def test_edge_shapes(cfg, schedule):
    w = wl.custom(name="edge", T=cfg["T"], d=cfg["d"], E=cfg["E"], k=cfg["k"], F=cfg["F"], C=cfg["C"],
                  bias="zipf", zipf_s=1.0, seed=cfg["T"])
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, schedule=schedule)
    idx, g, p = check_plan(layer, w, w.C, inp["logits"].cpu().numpy())
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


def test_renormalised_gates():
    w = wl.custom(name="renorm", T=333, d=128, E=12, k=3, F=128, C=50, bias="zipf", zipf_s=1.0, seed=5)
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, renorm=True)
    idx, g, p = check_plan(layer, w, w.C, inp["logits"].cpu().numpy(), renorm=True)
    np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-12)
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


def test_ties_in_logits_are_bit_exact():
    """Logits drawn from a handful of values (many exact ties, +0 and -0)."""
    T, E, k = 2000, 16, 4
    rng = np.random.default_rng(0)
    pool = np.array([-1.0, -0.0, 0.0, 0.5, 1.0], dtype=np.float32)
    z = pool[rng.integers(0, len(pool), size=(T, E))]
    w = wl.custom(name="ties", T=T, d=64, E=E, k=k, F=64, C=300)
    layer = moe.DroplessMoE(T, 64, E, k, 64, 300)
    layer.plan(logits=torch.from_numpy(z).cuda())
    check_plan(layer, w, 300, z)


def test_empty_batch():
    layer = moe.DroplessMoE(0, 128, 8, 2, 128, 16)
    z = torch.empty(0, 8, dtype=torch.float32, device="cuda")
    info = layer.plan(logits=z)
    assert info.R == 0 and info.max_load == 0
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    w13 = torch.zeros(8, 256, 128, dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros(8, 128, 128, dtype=torch.bfloat16, device="cuda")
    y = layer.forward(x, w13, w2)
    torch.cuda.synchronize()
    assert y.shape == (0, 128)


def test_router_gemm_small():
    """logits = x W_r^T + b on tensor cores (E not a power of two), then a bit-exact plan."""
    w = wl.custom(name="router", T=300, d=256, E=40, k=4, F=128, C=37, router="gemm", bias="zipf",
                  zipf_s=1.2, seed=9)
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp)
    z = layer.plan_tensors()["logits"].cpu().numpy()
    z_ref = oracle.router_logits(bits(inp["x"]), bits(inp["w_router"]), inp["bias"].cpu().numpy())
    assert np.max(np.abs(z - z_ref)) <= 1e-4 * np.max(np.abs(z_ref))
    idx, g, p = check_plan(layer, w, w.C, z)
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


# ----------------------------------------------------------------------------- properties

def test_deterministic_bits():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")
    _, y1 = run_gpu(w, inp)
    _, y2 = run_gpu(w, inp)
    assert torch.equal(y1, y2)


def test_capacity_changes_rounds_not_result():
    """Dropless: for every C the output is the same layer output (up to the fp32 order in
    which a token's pairs are summed across rounds); the round count follows ceil(max/C)."""
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")
    ys = {}
    for C in (64, 256, 1000, 4096):
        layer, y = run_gpu(w, inp, C=C)
        assert layer.info.R == math.ceil(layer.info.max_load / C)
        ys[C] = y.cpu().numpy().astype(np.float64)
    base = ys[4096]
    for C, y in ys.items():
        assert rel_err(y, base) <= 1e-5, C
    assert layer.info.R == 1


def test_schedules_give_identical_bits():
    """The launch schedule changes which rounds overlap, never the arithmetic: every output
    element is the same K-ordered fp32 sum and every token's pairs are combined in the same
    (round, j) order, whatever the tile widths and the launch boundaries."""
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")
    ys = {sch: run_gpu(w, inp, schedule=sch)[1] for sch in SCHEDULES}
    assert torch.equal(ys["per_round"], ys["pipeline"])
    assert torch.equal(ys["auto"], ys["pipeline"])


def test_pipeline_counters_return_to_zero_and_repeat():
    """One plan, two pipelined forwards: the dependency counters are zero after each launch
    (the last CTA clears them), so the second call starts clean and gives the same bits."""
    w = wl.BY_NAME["tiny-zipf1"]
    inp = wl.generate(w, "cuda")
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, schedule="pipeline")
    layer.plan(logits=inp["logits"])
    assert int(layer.sync_counters().abs().sum()) == 0
    y1 = layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert int(layer.sync_counters().abs().sum()) == 0
    y2 = layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(y1, y2)


# ----------------------------------------------------------------------------- capacity borrowing

@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_borrow_full_parity(name):
    """Capacity borrowing: the plan bit-exact against the oracle's borrowing plan (fewer
    rounds on skewed routing), y the same layer output."""
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, borrow=True)
    z = inp["logits"].cpu().numpy()
    idx, g, p = check_plan(layer, w, w.C, z, borrow=True)
    assert p["R"] < oracle.plan(idx, w.E, w.C)["R"]
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: "T{T}-d{d}-E{E}-k{k}-F{F}-C{C}".format(**c))
def test_borrow_edge_shapes(cfg):
    w = wl.custom(name="edge", T=cfg["T"], d=cfg["d"], E=cfg["E"], k=cfg["k"], F=cfg["F"], C=cfg["C"],
                  bias="zipf", zipf_s=1.0, seed=cfg["T"])
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, borrow=True)
    idx, g, p = check_plan(layer, w, w.C, inp["logits"].cpu().numpy(), borrow=True)
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


def test_borrow_sampled_parity_hot_expert():
    """16k-hot-expert with borrowing: the hot expert's overflow fills the other experts'
    unused rows; plan on every token, y on a token sample."""
    w = wl.BY_NAME["16k-hot-expert"]
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, borrow=True)
    z = inp["logits"].cpu().numpy()
    idx, g, p = check_plan(layer, w, w.C, z, borrow=True)
    assert p["R"] < oracle.plan(idx, w.E, w.C)["R"]
    tok = sample_tokens(w.T, p, 64, seed=w.seed)
    ref = oracle.forward(LazyRows(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g,
                         tokens=tok)
    got = y[torch.as_tensor(tok, device="cuda")].cpu().numpy().astype(np.float64)
    assert rel_err(got, ref) <= Y_TOL


# Round 0 of this shape gives each expert C = 1100 rows: four 256-row tiles of the CTA-pair
# GEMMs and a last tile with 76 rows; later rounds leave ragged last tiles of other sizes. The
# per-round GEMMs of round 0 run in the pair form (their 256-row tiles cover at most 15 % more
# rows than 128-row tiles).
RAGGED_SHAPE = dict(T=16384, d=512, E=32, k=4, F=512, C=1100)


@pytest.mark.parametrize("borrow", [False, True], ids=["per-expert", "borrow"])
@pytest.mark.parametrize("bias", ["none", "zipf"])
def test_ragged_pair_tiles_full_parity(bias, borrow):
    w = wl.custom(name="ragged", bias=bias, zipf_s=0.5, seed=21, **RAGGED_SHAPE)
    inp = wl.generate(w, "cuda")
    layer, y = run_gpu(w, inp, schedule="per_round", borrow=borrow)
    z = inp["logits"].cpu().numpy()
    idx, g, p = check_plan(layer, w, w.C, z, borrow=borrow)
    assert p["R"] >= 2
    ref = oracle.forward(bits(inp["x"]), LazyExperts(inp["w_gate_up"]), LazyExperts(inp["w_down"]), idx, g)
    assert rel_err(y.cpu().numpy().astype(np.float64), ref) <= Y_TOL


def test_ragged_pair_tiles_match_the_pipelined_bits():
    """The CTA-pair tiles of the per-round launches and the 128-row tiles of the single-CTA
    kernel that runs the pipelined rounds compute each output as the same K-ordered fp32 sum,
    so the two schedules agree bit for bit on a shape whose per-round GEMMs run in the pair
    form with ragged last row blocks."""
    w = wl.custom(name="ragged", bias="none", seed=21, **RAGGED_SHAPE)
    inp = wl.generate(w, "cuda")
    _, y_round = run_gpu(w, inp, schedule="per_round")
    _, y_pipe = run_gpu(w, inp, schedule="pipeline")
    assert torch.equal(y_round, y_pipe)
