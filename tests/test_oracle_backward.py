"""Pins of the backward oracle against facts it does not compute the same way.

The backward's arithmetic is checked against (1) central finite differences of the forward
oracle's own definitions (`gates`, `expert_ffn`), entry by entry; (2) torch float64 autograd
of the same forward written with torch ops; (3) exact identities of the forward's structure
(y is linear in the gates, in W2 and in W3, and the gates do not change when a constant is
added to all of a token's logits); (4) special cases with a closed form. The round-by-round
executor with recompute is then checked against the schedule-free definition.
"""
import numpy as np
import pytest
import torch

import oracle


def _bits(rng, shape, scale=1.0):
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _problem(seed=0, T=12, d=8, E=4, k=2, F=6, wscale=0.4):
    rng = np.random.default_rng(seed)
    x = _bits(rng, (T, d))
    w13 = _bits(rng, (E, 2 * F, d), wscale)
    w2 = _bits(rng, (E, d, F), wscale)
    # logits on a 2^-12 grid with |z| < 4: z +- 2^-10 is exact in fp32, so finite differences
    # through the oracle's fp32 view of z see exactly the intended step
    z = (np.round(rng.standard_normal((T, E)) * 4096.0) / 4096.0).clip(-3.9, 3.9).astype(np.float32)
    idx = oracle.select_topk(z, k)
    dy = rng.standard_normal((T, d))
    return x, w13, w2, z, idx, dy


def _loss(x, w13, w2, z, idx, dy, renorm):
    """L = sum_t <dy[t], y[t]> from the forward oracle's pieces, float64 inputs."""
    g = oracle.gates(z, idx, renorm)
    L = 0.0
    for t in range(idx.shape[0]):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            L += g[t, j] * float(dy[t] @ oracle.expert_ffn(x[t:t + 1], w13[e], w2[e])[0])
    return L


@pytest.mark.parametrize("renorm", [False, True])
def test_gradients_match_central_differences(renorm):
    xb, w13b, w2b, z, idx, dy = _problem(seed=1)
    grad = oracle.backward(xb, w13b, w2b, z, idx, dy, renorm=renorm)
    x, w13, w2 = (oracle.bf16_to_f64(a) for a in (xb, w13b, w2b))
    h = 1e-4

    def check(arr, g_analytic, name):
        flat = arr.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = _loss(x, w13, w2, z, idx, dy, renorm)
            flat[i] = keep - h
            lm = _loss(x, w13, w2, z, idx, dy, renorm)
            flat[i] = keep
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g_analytic.reshape(-1)[i]) <= 1e-6 * (1 + abs(fd)), (name, i, fd)

    check(x, grad["dx"], "dx")
    check(w13, grad["dw_gate_up"], "dw_gate_up")
    check(w2, grad["dw_down"], "dw_down")
    # logits: exact fp32 steps of 2^-10
    hz = 2.0 ** -10
    for t in range(z.shape[0]):
        for e in range(z.shape[1]):
            zp, zm = z.copy(), z.copy()
            zp[t, e] += np.float32(hz)
            zm[t, e] -= np.float32(hz)
            fd = (_loss(x, w13, w2, zp, idx, dy, renorm) - _loss(x, w13, w2, zm, idx, dy, renorm)) / (2 * hz)
            assert abs(fd - grad["dz"][t, e]) <= 2e-6 * (1 + abs(fd)), (t, e, fd, grad["dz"][t, e])


@pytest.mark.parametrize("renorm", [False, True])
def test_gradients_match_torch_autograd(renorm):
    xb, w13b, w2b, z, idx, dy = _problem(seed=2, T=20, d=16, E=6, k=3, F=12)
    grad = oracle.backward(xb, w13b, w2b, z, idx, dy, renorm=renorm)
    x = torch.tensor(oracle.bf16_to_f64(xb), requires_grad=True)
    w13 = torch.tensor(oracle.bf16_to_f64(w13b), requires_grad=True)
    w2 = torch.tensor(oracle.bf16_to_f64(w2b), requires_grad=True)
    zt = torch.tensor(z.astype(np.float64), requires_grad=True)
    it = torch.from_numpy(idx.astype(np.int64))
    g = torch.softmax(zt, dim=1).gather(1, it)
    if renorm:
        g = g / g.sum(dim=1, keepdim=True)
    F = w13.shape[1] // 2
    y = torch.zeros_like(x)
    for j in range(idx.shape[1]):
        a = torch.einsum("td,tfd->tf", x, w13[it[:, j], :F])
        b = torch.einsum("td,tfd->tf", x, w13[it[:, j], F:])
        hid = torch.nn.functional.silu(a) * b
        y = y + g[:, j:j + 1] * torch.einsum("tf,tdf->td", hid, w2[it[:, j]])
    (y * torch.from_numpy(dy)).sum().backward()
    for name, ref in (("dx", x.grad), ("dw_gate_up", w13.grad), ("dw_down", w2.grad), ("dz", zt.grad)):
        ref = ref.numpy()
        assert np.abs(grad[name] - ref).max() <= 1e-12 * (1 + np.abs(ref).max()), name


def test_structure_identities():
    """y is linear in the gates, in W2_e and in W3_e, so by Euler's theorem for degree-one
    homogeneous maps <gate, dgate> = <W2, dW2> = <W3, dW3> = <dy, y>; every token's dz sums to
    zero because the gates ignore a common shift of its logits."""
    xb, w13b, w2b, z, idx, dy = _problem(seed=3, T=30, d=16, E=5, k=2, F=8)
    g = oracle.gates(z, idx)
    grad = oracle.backward(xb, w13b, w2b, z, idx, dy)
    y = oracle.forward(xb, w13b, w2b, idx, g)
    dyy = float((dy * y).sum())
    assert abs(float((g * grad["dgate"]).sum()) - dyy) <= 1e-12 * (1 + abs(dyy))
    F = w13b.shape[1] // 2
    w13, w2 = oracle.bf16_to_f64(w13b), oracle.bf16_to_f64(w2b)
    for e in range(w13.shape[0]):
        tt, jj = np.nonzero(idx == e)
        part = float((g[tt, jj][:, None] * dy[tt] * oracle.expert_ffn(oracle.bf16_to_f64(xb[tt]), w13[e], w2[e])).sum())
        assert abs(float((w2[e] * grad["dw_down"][e]).sum()) - part) <= 1e-12 * (1 + abs(part))
        assert abs(float((w13[e, F:] * grad["dw_gate_up"][e, F:]).sum()) - part) <= 1e-12 * (1 + abs(part))
    assert np.abs(grad["dz"].sum(axis=1)).max() <= 1e-14


def test_gate_gradient_special_cases():
    rng = np.random.default_rng(4)
    z = rng.standard_normal((7, 5)).astype(np.float32)
    # k = E: renormalising divides by a sum that is already one, and changes nothing
    idx = oracle.select_topk(z, 5)
    dg = rng.standard_normal((7, 5))
    assert np.allclose(oracle.gates_backward(z, idx, dg, renorm=True),
                       oracle.gates_backward(z, idx, dg, renorm=False), rtol=0, atol=1e-15)
    # renormalised gates sum to one: a gradient equal on all of a token's pairs moves nothing
    idx2 = oracle.select_topk(z, 2)
    flat = np.repeat(rng.standard_normal((7, 1)), 2, axis=1)
    assert np.abs(oracle.gates_backward(z, idx2, flat, renorm=True)).max() <= 1e-15
    # one expert: the softmax is identically one
    assert np.all(oracle.gates_backward(z[:, :1], np.zeros((7, 1), np.int32), dg[:, :1]) == 0.0)
    # top-1 without renorm: dz = p * (dg * onehot - p_e * dg)
    idx1 = oracle.select_topk(z, 1)
    p = np.exp(z.astype(np.float64) - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    want = -p * (p[np.arange(7), idx1[:, 0]] * dg[:, 0])[:, None]
    want[np.arange(7), idx1[:, 0]] += p[np.arange(7), idx1[:, 0]] * dg[:, 0]
    assert np.allclose(oracle.gates_backward(z, idx1, dg[:, :1]), want, rtol=0, atol=1e-15)


def test_silu_grad_special_points():
    assert oracle.silu_grad(np.array([0.0]))[0] == 0.5
    assert abs(oracle.silu_grad(np.array([40.0]))[0] - 1.0) <= 1e-15
    assert abs(oracle.silu_grad(np.array([-40.0]))[0]) <= 1e-15
    # minimum of silu at the root of silu' (u* ~ -1.2784645, the solution of
    # 1 + e^u = -u): silu' changes sign there
    u = np.array([-1.2784645 - 1e-6, -1.2784645 + 1e-6])
    g = oracle.silu_grad(u)
    assert g[0] < 0 < g[1]
    uu = np.linspace(-6, 6, 25)
    h = 1e-5
    fd = (oracle.silu(uu + h) - oracle.silu(uu - h)) / (2 * h)
    assert np.abs(fd - oracle.silu_grad(uu)).max() <= 1e-9


def test_router_gradients_match_autograd():
    rng = np.random.default_rng(5)
    xb, wb = _bits(rng, (9, 16)), _bits(rng, (6, 16), 0.25)
    dz = rng.standard_normal((9, 6))
    got = oracle.router_backward(xb, wb, dz)
    x = torch.tensor(oracle.bf16_to_f64(xb), requires_grad=True)
    w = torch.tensor(oracle.bf16_to_f64(wb), requires_grad=True)
    b = torch.zeros(6, dtype=torch.float64, requires_grad=True)
    ((x @ w.T + b) * torch.from_numpy(dz)).sum().backward()
    for name, ref in (("dx", x.grad), ("dw_router", w.grad), ("dbias", b.grad)):
        assert np.abs(got[name] - ref.numpy()).max() <= 1e-12, name


def test_backward_is_linear_in_dy():
    xb, w13b, w2b, z, idx, dy = _problem(seed=6)
    dy2 = np.random.default_rng(7).standard_normal(dy.shape)
    a = oracle.backward(xb, w13b, w2b, z, idx, dy)
    b = oracle.backward(xb, w13b, w2b, z, idx, dy2)
    c = oracle.backward(xb, w13b, w2b, z, idx, dy + 2.0 * dy2)
    for name in ("dx", "dw_gate_up", "dw_down", "dgate", "dz"):
        assert np.allclose(c[name], a[name] + 2.0 * b[name], rtol=1e-12, atol=1e-12), name


@pytest.mark.parametrize("C,borrow", [(1, False), (2, False), (5, False), (64, False),
                                      (1, True), (3, True)])
def test_rounds_with_recompute_equal_the_definition(C, borrow):
    """The round schedule changes where and when each pair's gradients are computed, never
    what: every round recomputes its rows' forward from x, and the weight gradients add up
    over rounds to the schedule-free sums."""
    rng = np.random.default_rng(8)
    T, d, E, k, F = 40, 8, 4, 2, 6
    xb, w13b, w2b = _bits(rng, (T, d)), _bits(rng, (E, 2 * F, d), 0.3), _bits(rng, (E, d, F), 0.3)
    bias = -np.log(np.arange(1, E + 1))                  # skewed popularity: several rounds
    z = (rng.standard_normal((T, E)) + 2.0 * bias).astype(np.float32)
    idx = oracle.select_topk(z, k)
    dy = rng.standard_normal((T, d))
    ref = oracle.backward(xb, w13b, w2b, z, idx, dy)
    got = oracle.backward_rounds(xb, w13b, w2b, z, idx, dy, C, borrow=borrow)
    want_plan = oracle.plan_borrow(idx, E, C) if borrow else oracle.plan(idx, E, C)
    assert got["plan"]["R"] == want_plan["R"]
    if C == 1 and not borrow:
        assert got["plan"]["R"] == max(np.bincount(idx.ravel(), minlength=E))
    for name in ("dx", "dw_gate_up", "dw_down", "dgate", "dz"):
        scale = 1 + np.abs(ref[name]).max()
        assert np.abs(got[name] - ref[name]).max() <= 1e-12 * scale, name


@pytest.mark.parametrize("renorm", [False, True])
def test_sampled_entries_equal_the_definition(renorm):
    """The sampled evaluation takes each token's and each expert's pairs alone; the entries it
    returns must be the full backward's, for any choice of tokens (repeats, unsorted) and of
    experts (one with no pairs included)."""
    rng = np.random.default_rng(9)
    T, d, E, k, F = 30, 8, 5, 2, 6
    xb, w13b, w2b = _bits(rng, (T, d)), _bits(rng, (E, 2 * F, d), 0.3), _bits(rng, (E, d, F), 0.3)
    z = (rng.standard_normal((T, E)) - 8.0 * (np.arange(E) == 4)).astype(np.float32)   # expert 4 unused
    idx = oracle.select_topk(z, k)
    assert not np.any(idx == 4)
    dy = rng.standard_normal((T, d))
    ref = oracle.backward(xb, w13b, w2b, z, idx, dy, renorm=renorm)
    tokens = [7, 0, 29, 7, 13]
    experts = [3, 4, 0]
    got = oracle.backward_sampled(xb, w13b, w2b, z, idx, dy, tokens, experts, renorm=renorm)
    for name in ("dx", "dgate", "dz"):
        scale = 1 + np.abs(ref[name]).max()
        assert np.abs(got[name] - ref[name][tokens]).max() <= 1e-12 * scale, name
    for name in ("dw_gate_up", "dw_down"):
        scale = 1 + np.abs(ref[name]).max()
        assert np.abs(got[name] - ref[name][experts]).max() <= 1e-12 * scale, name
    assert np.count_nonzero(got["dw_gate_up"][1]) == 0 and np.count_nonzero(got["dw_down"][1]) == 0
