"""Pins of the expert-parallel oracle (oracle/moe_ep.py) against what does not depend on it:
a hand-derived worked example, the single-GPU plan of the ranks' batches concatenated in rank
order (itself pinned in test_oracle.py), invariants of the exchange that hold for any input,
and the capacity-free dropless output, which the literal expert-parallel executor must
reproduce for any capacity and any number of ranks."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ep_plan_worked_example.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *rest = line.split()
                vals[key] = rest
    return vals


def _ints(v):
    return np.array([int(x) for x in v], dtype=np.int64)


def test_worked_example():
    g = _golden()
    G, E, k, C = (int(g[n][0]) for n in ("G", "E", "k", "C"))
    idx = [_ints(g[f"idx{s}"]).reshape(-1, k) for s in range(G)]
    p = oracle.ep_plan(idx, E, C, G)
    for s in range(G):
        assert np.array_equal(p["round"][s], _ints(g[f"round{s}"]).reshape(-1, k))
        assert np.array_equal(p["slot"][s], _ints(g[f"slot{s}"]).reshape(-1, k))
    assert np.array_equal(p["load"], _ints(g["load"]).reshape(G, E))
    assert np.array_equal(p["base"], _ints(g["base"]).reshape(G, E))
    assert p["R"] == int(g["R"][0])
    assert np.array_equal(p["n"], _ints(g["n"]).reshape(-1, E))
    assert np.array_equal(p["send"], _ints(g["send"]).reshape(-1, G, G))
    # owner 0's round-0 buffer: (local expert, slot) -> (source rank, token)
    buf = {}
    for s in range(G):
        for (e, slot, t, j) in p["rows"][0][s]:
            if oracle.owner(e, E, G) == 0:
                buf[(e, slot)] = (s, t)
    want = {}
    for item in g["owner0_round0"]:
        key, val = item.split("=")
        e, slot = (int(x) for x in key.split(":"))
        s, t = (int(x) for x in val.split("/"))
        want[(e, slot)] = (s, t)
    assert buf == want


def _random_idx(rng, G, T, E, k, skew):
    out = []
    for _ in range(G):
        z = rng.standard_normal((T, E)) - skew * np.log1p(np.arange(E))[None, :]
        out.append(oracle.select_topk(z.astype(np.float32), k))
    return out


@pytest.mark.parametrize("G,E,k,C,T", [(1, 8, 2, 3, 20), (2, 8, 2, 3, 20), (4, 8, 3, 5, 17), (2, 6, 1, 1, 9),
                                       (4, 16, 4, 64, 30), (3, 9, 2, 4, 0)])
def test_plan_is_the_single_gpu_plan_of_the_concatenated_batch(G, E, k, C, T):
    rng = np.random.default_rng(G * 100 + C)
    idx = _random_idx(rng, G, T, E, k, skew=1.0)
    p = oracle.ep_plan(idx, E, C, G)
    q = oracle.plan(np.concatenate(idx, axis=0).reshape(-1, k), E, C)
    assert p["R"] == q["R"]
    assert np.array_equal(p["total"], q["load"])
    assert np.array_equal(p["n"], q["n"])
    off = 0
    for s in range(G):
        assert np.array_equal(p["round"][s], q["round"][off:off + T])
        assert np.array_equal(p["slot"][s], q["slot"][off:off + T])
        off += T


@pytest.mark.parametrize("G,E,k,C,T", [(2, 8, 2, 3, 40), (4, 8, 3, 5, 33), (4, 16, 4, 7, 50)])
def test_exchange_invariants(G, E, k, C, T):
    rng = np.random.default_rng(7 + G)
    idx = _random_idx(rng, G, T, E, k, skew=1.5)
    p = oracle.ep_plan(idx, E, C, G)
    per = E // G
    send = p["send"]
    # every pair is sent exactly once, in its own round, to the owner of its expert
    for s in range(G):
        assert send[:, s, :].sum() == T * k
        for r in range(p["R"]):
            assert send[r, s, :].sum() == int((p["round"][s] == r).sum())
            assert len(p["rows"][r][s]) == send[r, s, :].sum()
    # what an owner receives in a round fills exactly its experts' rows of that round
    for r in range(p["R"]):
        for g in range(G):
            assert send[r, :, g].sum() == p["n"][r, g * per:(g + 1) * per].sum() <= per * C
    # the offsets are the exclusive prefix sums of the counts
    assert np.array_equal(p["send_off"][:, :, 1:], np.cumsum(send, axis=2)[:, :, :-1])
    assert np.array_equal(p["recv_off"][:, :, 1:], np.cumsum(send.transpose(0, 2, 1), axis=2)[:, :, :-1])
    # base is the exclusive prefix over ranks of the loads; the total is what one GPU would see
    assert np.array_equal(p["base"][1:], np.cumsum(p["load"], axis=0)[:-1])
    assert p["R"] == -(-int(p["total"].max()) // C)


def test_one_rank_is_the_single_gpu_plan():
    rng = np.random.default_rng(3)
    idx = _random_idx(rng, 1, 64, 8, 2, skew=2.0)
    p = oracle.ep_plan(idx, 8, 5, 1)
    q = oracle.plan(idx[0], 8, 5)
    assert np.array_equal(p["round"][0], q["round"]) and np.array_equal(p["slot"][0], q["slot"])
    assert np.array_equal(p["send"][:, 0, 0], q["n"].sum(axis=1))


def _bits(rng, shape, scale):
    import torch
    return (torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
            .to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("C", [1, 2, 5, 1000])
def test_executor_equals_capacity_free_output(G, C):
    """The literal expert-parallel executor gives every rank the capacity-free dropless output of
    its own tokens, for any capacity and rank count, and never holds more than C rows of an
    expert in a round."""
    rng = np.random.default_rng(11 * G + C)
    E, k, T, d, F = 8, 2, 12, 16, 24
    idx = _random_idx(rng, G, T, E, k, skew=1.0)
    zs = [rng.standard_normal((T, E)).astype(np.float32) for _ in range(G)]
    gts = [oracle.gates(z, i) for z, i in zip(zs, idx)]
    xs = [_bits(rng, (T, d), 1.0) for _ in range(G)]
    w13 = _bits(rng, (E, 2 * F, d), 0.1)
    w2 = _bits(rng, (E, d, F), 0.1)
    ys, p, peak = oracle.ep_forward(xs, w13, w2, idx, gts, C, G)
    assert peak <= C
    for s in range(G):
        ref = oracle.forward(xs[s], w13, w2, idx[s], gts[s])
        np.testing.assert_allclose(ys[s], ref, rtol=1e-12, atol=1e-12)
