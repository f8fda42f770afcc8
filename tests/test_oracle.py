"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute the same way:
a hand-derived worked example (tests/golden), brute-force enumeration, a closed
form, a library routine (torch float64 on the CPU), or an exact invariant that
the pages state (no token dropped, rounds change nothing but the schedule,
R = ceil(max load / C), a single round once C covers the largest load).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from dropless_moe_layer_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_bf16_bits(rng, shape, scale=1.0):
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *rest = line.split()
            vals[key] = rest
    return vals


# ----------------------------------------------------------------------------- formats

def test_bf16_widening_known_patterns():
    # values from the binary format: sign | 8-bit exponent (bias 127) | 7-bit fraction
    cases = {
        0x3F80: 1.0,
        0xC000: -2.0,
        0x3FC0: 1.5,
        0x0000: 0.0,
        0x0001: math.ldexp(1.0, -133),                  # smallest subnormal
        0x7F7F: math.ldexp(2.0 - 2.0 ** -7, 127),       # largest finite
        0x3E80: 0.25,
    }
    bits = np.array(list(cases.keys()), dtype=np.uint16)
    got = oracle.bf16_to_f64(bits)
    assert list(got) == list(cases.values())
    assert math.copysign(1.0, oracle.bf16_to_f64(np.array([0x8000], np.uint16))[0]) == -1.0


def test_bf16_widening_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    bits = bits[exp != 0xFF]                                   # finite only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.bf16_to_f64(bits), ref)


# ----------------------------------------------------------------------------- selection

def _brute_topk(zrow, k):
    """Best ordered k-tuple of distinct experts, compared position by position on
    (logit, -index): the largest logit first, equal logits to the lower index."""
    E = len(zrow)
    best = None
    for tup in itertools.permutations(range(E), k):
        key = [(float(zrow[e]) + 0.0, -e) for e in tup]   # +0.0 folds -0 into +0
        if best is None or key > best[0]:
            best = (key, tup)
    return list(best[1])


@pytest.mark.parametrize("E", [1, 2, 3, 5, 6])
def test_select_topk_brute_force_with_ties(E):
    rng = np.random.default_rng(E)
    pool = np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 2.0], dtype=np.float32)   # many ties
    z = pool[rng.integers(0, len(pool), size=(40, E))]
    for k in range(1, E + 1):
        idx = oracle.select_topk(z, k)
        for t in range(z.shape[0]):
            assert list(idx[t]) == _brute_topk(z[t], k), (t, k, z[t])


def test_select_topk_rejects_nonfinite_and_bad_k():
    with pytest.raises(ValueError):
        oracle.select_topk(np.array([[0.0, np.inf]], np.float32), 1)
    with pytest.raises(ValueError):
        oracle.select_topk(np.zeros((2, 3), np.float32), 4)


# ----------------------------------------------------------------------------- gates

def test_gates_two_experts_logistic_closed_form():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((64, 2)).astype(np.float32) * 3
    idx = oracle.select_topk(z, 1)
    g = oracle.gates(z, idx)
    zd = z.astype(np.float64)
    for t in range(64):
        e = idx[t, 0]
        other = 1 - e
        logistic = 1.0 / (1.0 + math.exp(zd[t, other] - zd[t, e]))
        assert g[t, 0] == pytest.approx(logistic, rel=1e-14)


def test_gates_sum_and_renorm():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((50, 6)).astype(np.float32)
    full = oracle.gates(z, oracle.select_topk(z, 6))
    np.testing.assert_allclose(full.sum(1), 1.0, rtol=1e-14)
    part = oracle.gates(z, oracle.select_topk(z, 3))
    assert np.all(part.sum(1) < 1.0)
    assert np.all(np.diff(part, axis=1) <= 0)          # best first
    ren = oracle.gates(z, oracle.select_topk(z, 3), renorm=True)
    np.testing.assert_allclose(ren.sum(1), 1.0, rtol=1e-14)


# ----------------------------------------------------------------------------- plan

def test_plan_worked_example():
    g = _read_golden("plan_worked_example.txt")
    T, E, k, C = (int(g[key][0]) for key in ("T", "E", "k", "C"))
    z = np.array([float(v) for v in g["logits"]], dtype=np.float32).reshape(T, E)
    assert math.copysign(1.0, z[5, 2]) == -1.0                 # the -0.0 survived parsing
    idx = oracle.select_topk(z, k)
    np.testing.assert_array_equal(idx, np.array(g["idx"], int).reshape(T, k))
    p = oracle.plan(idx, E, C)
    np.testing.assert_array_equal(p["round"], np.array(g["round"], int).reshape(T, k))
    np.testing.assert_array_equal(p["slot"], np.array(g["slot"], int).reshape(T, k))
    np.testing.assert_array_equal(p["load"], np.array(g["load"], int))
    assert p["R"] == int(g["R"][0])
    np.testing.assert_array_equal(p["n"], np.array(g["n"], int).reshape(p["R"], E))
    for r in range(p["R"]):
        want = []
        for item in g[f"round{r}"]:
            es, t = item.split("=")
            e, s = es.split(":")
            want.append((int(e), int(s), int(t)))
        got = [(e, s, t) for (e, s, t, j) in oracle.round_rows(p, idx, r)]
        assert got == sorted(want)


def _check_plan_invariants(idx, p, E, C):
    T, k = idx.shape
    assert p["load"].sum() == T * k                              # no pair dropped
    assert p["R"] == math.ceil(p["load"].max() / C)
    assert np.all(p["round"] < max(p["R"], 1)) and np.all(p["slot"] < C)
    assert np.all(p["slot"] >= 0)
    for e in range(E):
        ts, js = np.nonzero(idx == e)                            # ts ascending
        rk = p["round"][ts, js] * C + p["slot"][ts, js]
        np.testing.assert_array_equal(rk, np.arange(ts.size))   # stable token order
    for r in range(p["R"]):
        for e in range(E):
            sl = np.sort(p["slot"][(p["round"] == r) & (idx == e)])
            np.testing.assert_array_equal(sl, np.arange(p["n"][r, e]))
    np.testing.assert_array_equal(p["n"].sum(0), p["load"])


@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_plan_invariants_on_workloads(name):
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cpu", routing_only=True)
    z = inp["logits"].numpy()
    idx = oracle.select_topk(z, w.k)
    p = oracle.plan(idx, w.E, w.C)
    _check_plan_invariants(idx, p, w.E, w.C)
    assert p["R"] >= 2                                           # skewed: several rounds


def test_plan_special_cases():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((300, 7)).astype(np.float32)
    idx = oracle.select_topk(z, 3)
    big = oracle.plan(idx, 7, C=10_000)
    assert big["R"] == 1 and not big["round"].any()             # C >= max load: one round
    assert np.array_equal(big["slot"], big["rank"])
    one = oracle.plan(idx, 7, C=1)
    assert one["R"] == one["max_load"]                           # C = 1: a round per token of the busiest expert
    assert not one["slot"].any()
    exact = oracle.plan(idx, 7, C=int(big["max_load"]))
    assert exact["R"] == 1
    over = oracle.plan(idx, 7, C=int(big["max_load"]) - 1)
    assert over["R"] == 2
    empty = oracle.plan(np.zeros((0, 3), np.int32), 7, C=4)
    assert empty["R"] == 0 and empty["load"].sum() == 0


# ----------------------------------------------------------------------------- capacity borrowing

def test_plan_borrow_worked_example():
    g = _read_golden("plan_borrow_worked_example.txt")
    T, E, k, C = (int(g[key][0]) for key in ("T", "E", "k", "C"))
    z = np.array([float(v) for v in g["logits"]], dtype=np.float32).reshape(T, E)
    idx = oracle.select_topk(z, k)
    np.testing.assert_array_equal(idx, np.array(g["idx"], int).reshape(T, k))
    p = oracle.plan_borrow(idx, E, C)
    np.testing.assert_array_equal(p["round"], np.array(g["round"], int).reshape(T, k))
    np.testing.assert_array_equal(p["slot"], np.array(g["slot"], int).reshape(T, k))
    np.testing.assert_array_equal(p["load"], np.array(g["load"], int))
    assert p["R"] == int(g["R"][0])
    np.testing.assert_array_equal(p["n"], np.array(g["n"], int).reshape(p["R"], E))
    for r in range(p["R"]):
        want = []
        for item in g[f"round{r}"]:
            es, t = item.split("=")
            e, s = es.split(":")
            want.append((int(e), int(s), int(t)))
        got = [(e, s, t) for (e, s, t, j) in oracle.round_rows(p, idx, r)]
        assert got == sorted(want)


def _check_borrow_invariants(idx, p, E, C):
    """What the borrowing rule fixes, whatever order spare rows are lent in."""
    T, k = idx.shape
    load = p["load"]
    assert load.sum() == T * k
    np.testing.assert_array_equal(p["n"].sum(0), load)                  # every pair once
    assert np.all(p["n"].sum(1) <= E * C)                                # fixed round buffer
    pending = load.copy()
    for r in range(p["R"]):
        n_r = p["n"][r]
        assert np.all(n_r >= np.minimum(pending, C))                      # own capacity first
        if n_r.sum() < E * C:                                            # spare left over:
            assert np.array_equal(n_r, pending)                           # nothing was waiting
        pending = pending - n_r
    assert not pending.any()
    total = T * k
    assert p["R"] >= math.ceil(total / (E * C))                           # pool bound
    assert p["R"] <= math.ceil(load.max() / C) if total else p["R"] == 0  # never worse
    for e in range(E):                                                    # stable token order
        ts, js = np.nonzero(idx == e)
        start = np.concatenate([[0], np.cumsum(p["n"][:, e])])
        rk = start[p["round"][ts, js]] + p["slot"][ts, js]
        np.testing.assert_array_equal(rk, np.arange(ts.size))


@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_plan_borrow_invariants_on_workloads(name):
    w = wl.BY_NAME[name]
    z = wl.generate(w, "cpu", routing_only=True)["logits"].numpy()
    idx = oracle.select_topk(z, w.k)
    p = oracle.plan_borrow(idx, w.E, w.C)
    _check_borrow_invariants(idx, p, w.E, w.C)
    assert p["R"] < oracle.plan(idx, w.E, w.C)["R"]                      # skewed: fewer rounds


def test_plan_borrow_special_cases():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((300, 7)).astype(np.float32)
    idx = oracle.select_topk(z, 3)
    # one round exactly when all pairs fit the pool: R = 1 iff T*k <= E*C
    for C in (128, 129, 130, 200):
        p = oracle.plan_borrow(idx, 7, C)
        _check_borrow_invariants(idx, p, 7, C)
        assert (p["R"] == 1) == (900 <= 7 * C)
    # nobody over capacity: borrowing changes nothing
    base = oracle.plan(idx, 7, C=10_000)
    bor = oracle.plan_borrow(idx, 7, C=10_000)
    for key in ("round", "slot", "n"):
        np.testing.assert_array_equal(base[key], bor[key])
    # a single expert has nobody to borrow from
    one = np.zeros((50, 1), np.int64)
    for key in ("round", "slot", "n"):
        np.testing.assert_array_equal(oracle.plan(one, 1, 7)[key], oracle.plan_borrow(one, 1, 7)[key])
    # every pair on one expert of eight: the whole pool each round
    hot = np.zeros((100, 1), np.int64)
    p = oracle.plan_borrow(hot, 8, 4)
    assert p["R"] == math.ceil(100 / 32) and list(p["n"][:, 0]) == [32, 32, 32, 4]
    empty = oracle.plan_borrow(np.zeros((0, 2), np.int64), 5, 3)
    assert empty["R"] == 0
    # two overloaded experts, two spare rows: the lower expert index takes them (the reading)
    two = np.array([[0]] * 4 + [[1]] * 4, np.int64)
    p = oracle.plan_borrow(two, 3, 2)
    np.testing.assert_array_equal(p["n"], [[4, 2, 0], [0, 2, 0]])
    np.testing.assert_array_equal(p["round"][:, 0], [0, 0, 0, 0, 0, 0, 1, 1])
    np.testing.assert_array_equal(p["slot"][:, 0], [0, 1, 2, 3, 0, 1, 0, 1])


@pytest.mark.parametrize("seed", [0, 1])
def test_borrowing_rounds_do_not_change_the_output(seed):
    """The pooled round executor with borrowing gives the capacity-free output."""
    rng = np.random.default_rng(40 + seed)
    T, E, k, d, F = 24, 5, 2, 8, 16
    z = rng.standard_normal((T, E)).astype(np.float32)
    z[:, 0] += 3.0                                                        # one hot expert
    x = _rand_bf16_bits(rng, (T, d))
    w13 = _rand_bf16_bits(rng, (E, 2 * F, d), 0.3)
    w2 = _rand_bf16_bits(rng, (E, d, F), 0.3)
    idx = oracle.select_topk(z, k)
    g = oracle.gates(z, idx)
    y_free = oracle.forward(x, w13, w2, idx, g)
    for C in (1, 2, 3, 5, 24):
        y, p, peak = oracle.forward_rounds(x, w13, w2, idx, g, C, borrow=True)
        assert p["R"] <= oracle.plan(idx, E, C)["R"]
        assert peak <= E * C
        np.testing.assert_allclose(y, y_free, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- expert math

def _torch_swiglu(x, w1, w3, w2):
    """Dense SwiGLU MLP with torch float64 CPU ops (a library routine)."""
    return torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(x, w1)) * torch.nn.functional.linear(x, w3), w2)


def _bits_to_torch64(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64)


def test_single_expert_is_dense_swiglu_mlp():
    rng = np.random.default_rng(4)
    T, d, F = 37, 24, 40
    x = _rand_bf16_bits(rng, (T, d))
    w13 = _rand_bf16_bits(rng, (1, 2 * F, d), 0.2)
    w2 = _rand_bf16_bits(rng, (1, d, F), 0.2)
    z = rng.standard_normal((T, 1)).astype(np.float32)
    out = oracle.layer(x, w13, w2, k=1, C=5, logits=z)
    assert np.all(out["gate"] == 1.0)
    X, W13, W2 = _bits_to_torch64(x), _bits_to_torch64(w13)[0], _bits_to_torch64(w2)[0]
    ref = _torch_swiglu(X, W13[:F], W13[F:], W2).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def test_two_expert_mixture_closed_form():
    rng = np.random.default_rng(5)
    T, d, F = 29, 16, 32
    x = _rand_bf16_bits(rng, (T, d))
    w13 = _rand_bf16_bits(rng, (2, 2 * F, d), 0.2)
    w2 = _rand_bf16_bits(rng, (2, d, F), 0.2)
    z = (rng.standard_normal((T, 2)) * 2).astype(np.float32)
    out = oracle.layer(x, w13, w2, k=2, C=3, logits=z)
    X, W13, W2 = _bits_to_torch64(x), _bits_to_torch64(w13), _bits_to_torch64(w2)
    f = [_torch_swiglu(X, W13[e, :F], W13[e, F:], W2[e]).numpy() for e in range(2)]
    zd = z.astype(np.float64)
    g0 = 1.0 / (1.0 + np.exp(zd[:, 1] - zd[:, 0]))               # logistic form of the 2-way softmax
    ref = g0[:, None] * f[0] + (1.0 - g0)[:, None] * f[1]
    np.testing.assert_allclose(out["y"], ref, rtol=1e-10, atol=1e-12)


def _small_layer_inputs(seed, T=40, d=16, F=24, E=5):
    rng = np.random.default_rng(seed)
    x = _rand_bf16_bits(rng, (T, d))
    w13 = _rand_bf16_bits(rng, (E, 2 * F, d), 0.3)
    w2 = _rand_bf16_bits(rng, (E, d, F), 0.3)
    z = rng.standard_normal((T, E)).astype(np.float32)
    z[:, 0] += 1.5                                                # skew towards expert 0
    return x, w13, w2, z


def test_output_scales_exactly_with_w_down():
    x, w13, w2, z = _small_layer_inputs(6)
    y1 = oracle.layer(x, w13, w2, k=2, C=4, logits=z)["y"]
    w2x2 = (w2.astype(np.uint32) + (1 << 7)).astype(np.uint16)   # exponent + 1: exactly 2 * w2
    assert np.all(oracle.bf16_to_f64(w2x2) == 2 * oracle.bf16_to_f64(w2))
    y2 = oracle.layer(x, w13, w2x2, k=2, C=4, logits=z)["y"]
    np.testing.assert_array_equal(y2, 2 * y1)


def test_expert_relabelling_leaves_output_unchanged():
    x, w13, w2, z = _small_layer_inputs(7)
    perm = np.array([3, 0, 4, 1, 2])
    y = oracle.layer(x, w13, w2, k=2, C=3, logits=z)["y"]
    yp = oracle.layer(x, w13[perm], w2[perm], k=2, C=3, logits=z[:, perm])["y"]
    np.testing.assert_allclose(yp, y, rtol=1e-13, atol=1e-15)


def test_token_permutation_permutes_output():
    x, w13, w2, z = _small_layer_inputs(8)
    perm = np.random.default_rng(0).permutation(x.shape[0])
    y = oracle.layer(x, w13, w2, k=3, C=2, logits=z)["y"]
    yp = oracle.layer(x[perm], w13, w2, k=3, C=2, logits=z[perm])["y"]
    np.testing.assert_allclose(yp, y[perm], rtol=1e-12, atol=1e-14)


def test_sampled_tokens_equal_full_rows():
    x, w13, w2, z = _small_layer_inputs(9)
    full = oracle.layer(x, w13, w2, k=2, C=3, logits=z)
    tok = np.array([0, 5, 7, 39])
    part = oracle.forward(x, w13, w2, full["idx"], full["gate"], tokens=tok)
    np.testing.assert_allclose(part, full["y"][tok], rtol=1e-13, atol=1e-15)


def test_router_logits_match_torch_matmul():
    rng = np.random.default_rng(10)
    x = _rand_bf16_bits(rng, (33, 64))
    wr = _rand_bf16_bits(rng, (8, 64), 1 / 8)
    b = rng.standard_normal(8).astype(np.float32)
    z = oracle.router_logits(x, wr, b)
    ref = (_bits_to_torch64(x) @ _bits_to_torch64(wr).T + torch.from_numpy(b).double()).float().numpy()
    np.testing.assert_allclose(z, ref, rtol=2e-7, atol=1e-7)


# ----------------------------------------------------------------------------- rounds

@pytest.mark.parametrize("seed", [11, 12])
def test_rounds_do_not_change_the_output(seed):
    """Dropless: for every capacity the round-by-round executor gives the
    capacity-free output; memory per round never exceeds C rows per expert."""
    x, w13, w2, z = _small_layer_inputs(seed, T=48)
    k = 2
    idx = oracle.select_topk(z, k)
    g = oracle.gates(z, idx)
    y_free = oracle.forward(x, w13, w2, idx, g)
    max_load = int(oracle.plan(idx, 5, 1)["max_load"])
    for C in (1, 2, 3, 7, max_load, 48):
        y, p, peak = oracle.forward_rounds(x, w13, w2, idx, g, C)
        assert peak <= C
        assert p["R"] == math.ceil(max_load / C)
        np.testing.assert_allclose(y, y_free, rtol=1e-12, atol=1e-14)


def test_rounds_golden_dispatch_contents():
    g = _read_golden("plan_worked_example.txt")
    T, E, k, C = (int(g[key][0]) for key in ("T", "E", "k", "C"))
    z = np.array([float(v) for v in g["logits"]], dtype=np.float32).reshape(T, E)
    rng = np.random.default_rng(13)
    x = _rand_bf16_bits(rng, (T, 8))
    w13 = _rand_bf16_bits(rng, (E, 16, 8), 0.3)
    w2 = _rand_bf16_bits(rng, (E, 8, 8), 0.3)
    idx = oracle.select_topk(z, k)
    gt = oracle.gates(z, idx)
    y, p, peak = oracle.forward_rounds(x, w13, w2, idx, gt, C)
    assert p["R"] == 3 and peak == 2
    np.testing.assert_allclose(y, oracle.forward(x, w13, w2, idx, gt), rtol=1e-12, atol=1e-14)
