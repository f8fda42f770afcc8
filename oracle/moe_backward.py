"""CPU oracle for the backward pass of the multi-round dropless MoE layer.

TEST INFRASTRUCTURE, like the forward oracle beside it: only the test suite, the smoke check
and the benchmark's CPU-baseline leg may import it; the library shares no code with it.
Arithmetic is float64 (numpy); bf16 inputs are widened exactly.

What the pages say about the backward pass:
  * "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups keep
    memory fixed when tokens pile up": the backward pass recomputes each expert group on
    the same round schedule as the forward, so its memory is as static as the forward's.
  * "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless
    MoE item [section "Scaling MoE", Fig. 6]: the backward uses fine-grained per-expert-group
    recompute.

The pages give no formulas; the gradients are those of the forward the oracle defines (the
derivative of a function is fixed by the function). Notation, per expert e and row x:
    a = W1 x,  b = W3 x,  s = silu(a),  h = s * b,  out = W2 h
and per pair (t, j) with e = idx[t, j]: y[t] += gate[t, j] * out_e(x_t). Given dy = dL/dy:
    dgate[t, j] = <dy[t], out_e(x_t)>
    dout        = gate[t, j] * dy[t]
    dW2_e      += dout h^T                 dh = W2^T dout
    db = dh * s                            da = dh * b * silu'(a),
    silu'(a) = sig(a) (1 + a (1 - sig(a)))
    dW1_e      += da x^T,  dW3_e += db x^T,  dx[t] += W1^T da + W3^T db
and through the gates (softmax over all E logits, then the k selected; the selection itself is
piecewise constant in z and contributes nothing):
    dp_e = sum_{j: idx[t, j] = e} dgate[t, j]    (renormalised gates: dp_{e_j} = (dgate_j -
                                                   sum_i gate_i dgate_i) / sum_i p_{e_i})
    dz[t, e] = p_e (dp_e - sum_e' p_e' dp_e')
Router (logits z = x W_r^T + b): dW_r = dz^T x, db = sum_t dz[t], dx[t] += W_r^T dz[t].
The gate function is the forward oracle's reading (softmax over all E, then top-k), which the
pages never name: "parity unpinned" for that choice, as in the forward; the gradients of the
chosen function are pinned (finite differences, autograd, exact identities).

`backward` is that definition, pair by pair, with no schedule; `backward_sampled` is the same
definition evaluated only for some tokens and some experts (every gradient entry depends on a
token's own pairs or on one expert's pairs alone), for sizes where the whole is too slow;
`backward_rounds` is the
literal round-by-round form with recompute: each round re-dispatches its rows of x and of
gate * dy into fixed buffers of E*C rows, recomputes a, b and h for them, and adds the
round's weight gradients into per-expert accumulators, so nothing it keeps grows with the
routing. The two agree up to the order of float64 additions.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import bf16_to_f64, gates, plan, plan_borrow, round_rows, silu


def silu_grad(u):
    """d silu(u) / du = sig(u) + u sig(u) (1 - sig(u)), sig(u) = 1 / (1 + e^-u)."""
    sig = 1.0 / (1.0 + np.exp(-u))
    return sig * (1.0 + u * (1.0 - sig))


def expert_backward(xrows, w_gate_up_e, w_down_e, dout) -> dict:
    """Gradients of one expert's SwiGLU FFN for rows x (float64 [n, d]) given dout [n, d].

    w_gate_up_e: [2F, d] (rows 0..F-1 = W1, gate; rows F..2F-1 = W3, up); w_down_e: [d, F].
    Returns out [n, d] (the recomputed forward), dx [n, d], dw_gate_up [2F, d], dw_down [d, F].
    """
    F = w_gate_up_e.shape[0] // 2
    w1, w3 = w_gate_up_e[:F], w_gate_up_e[F:]
    a = xrows @ w1.T
    b = xrows @ w3.T
    s = silu(a)
    h = s * b
    out = h @ w_down_e.T
    dh = dout @ w_down_e
    dw_down = dout.T @ h
    db = dh * s
    da = dh * b * silu_grad(a)
    dw_gate_up = np.concatenate([da.T @ xrows, db.T @ xrows], axis=0)
    dx = da @ w1 + db @ w3
    return dict(out=out, dx=dx, dw_gate_up=dw_gate_up, dw_down=dw_down)


def gates_backward(z, idx, dgate, renorm: bool = False) -> np.ndarray:
    """dL/dz [T, E] (float64) given dL/dgate [T, k], for the gates of `gates` (softmax over all
    E fp32 logits, the k selected, optionally divided by their sum)."""
    zd = np.asarray(z, dtype=np.float32).astype(np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    dgate = np.asarray(dgate, dtype=np.float64)
    T, E = zd.shape
    m = zd.max(axis=1, keepdims=True)
    p = np.exp(zd - m)
    p = p / p.sum(axis=1, keepdims=True)
    psel = np.take_along_axis(p, idx, axis=1)                 # p of the selected experts
    if renorm:
        S = psel.sum(axis=1, keepdims=True)
        g = psel / S
        dpsel = (dgate - (g * dgate).sum(axis=1, keepdims=True)) / S
    else:
        dpsel = dgate
    dp = np.zeros((T, E), dtype=np.float64)
    rows = np.arange(T)
    for j in range(idx.shape[1]):                             # distinct experts per token
        dp[rows, idx[:, j]] += dpsel[:, j]
    return p * (dp - (p * dp).sum(axis=1, keepdims=True))


def router_backward(x_bits, w_router_bits, dz) -> dict:
    """Gradients of z = x W_r^T + b: dx [T, d], dw_router [E, d], dbias [E] (float64)."""
    x = bf16_to_f64(x_bits)
    w = bf16_to_f64(w_router_bits)
    dz = np.asarray(dz, dtype=np.float64)
    return dict(dx=dz @ w, dw_router=dz.T @ x, dbias=dz.sum(axis=0))


def backward(x_bits, w_gate_up_bits, w_down_bits, z, idx, dy, renorm: bool = False,
             gate=None) -> dict:
    """Gradients of the capacity-free layer output y[t] = sum_j gate[t, j] f_{idx[t, j]}(x_t)
    with respect to x (through the experts only), the expert weights, the gates and the
    logits, given dy [T, d]. `gate` defaults to the float64 gates of z; a caller that ran the
    forward with other gate values (fp32, say) passes those, and dz is still taken through
    the softmax of z. Per-pair contributions to dx are added in j order."""
    idx = np.asarray(idx)
    T, k = idx.shape
    E = w_gate_up_bits.shape[0]
    d = w_down_bits.shape[1]
    g = gates(z, idx, renorm) if gate is None else np.asarray(gate, dtype=np.float64)
    dyd = np.asarray(dy, dtype=np.float64)
    x = bf16_to_f64(x_bits)
    dx_terms = np.zeros((T, k, d), dtype=np.float64)
    dgate = np.zeros((T, k), dtype=np.float64)
    dw_gate_up = np.zeros(w_gate_up_bits.shape, dtype=np.float64)
    dw_down = np.zeros(w_down_bits.shape, dtype=np.float64)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        gr = expert_backward(x[tt], bf16_to_f64(w_gate_up_bits[e]), bf16_to_f64(w_down_bits[e]),
                             g[tt, jj][:, None] * dyd[tt])
        dgate[tt, jj] = (dyd[tt] * gr["out"]).sum(axis=1)
        dx_terms[tt, jj, :] = gr["dx"]
        dw_gate_up[e] = gr["dw_gate_up"]
        dw_down[e] = gr["dw_down"]
    dx = np.zeros((T, d), dtype=np.float64)
    for j in range(k):
        dx = dx + dx_terms[:, j, :]
    return dict(dx=dx, dw_gate_up=dw_gate_up, dw_down=dw_down, dgate=dgate,
                dz=gates_backward(z, idx, dgate, renorm))


def backward_sampled(x_bits, w_gate_up_bits, w_down_bits, z, idx, dy, tokens, experts,
                     renorm: bool = False, gate=None) -> dict:
    """Entries of `backward` at sizes where computing all of them is too slow.

    dx, dgate and dz of token t depend only on token t's own k pairs (its row through each of
    its experts), and expert e's weight gradients only on the pairs routed to e. So this takes
    the same definition over those pairs alone: for each sampled token, its k pairs; for each
    sampled expert, all of its pairs in one `expert_backward`. Returns dx [len(tokens), d],
    dgate and dz of those tokens, dw_gate_up [len(experts), 2F, d], dw_down [len(experts), d, F].
    `gate` (full [T, k]) as in `backward`."""
    idx = np.asarray(idx)
    z = np.asarray(z)
    tokens = np.asarray(tokens, dtype=np.int64)
    T, k = idx.shape
    d = w_down_bits.shape[1]
    g = gates(z, idx, renorm) if gate is None else np.asarray(gate, dtype=np.float64)
    dyd = np.asarray(dy, dtype=np.float64)
    dx = np.zeros((tokens.size, d), dtype=np.float64)
    dgate = np.zeros((tokens.size, k), dtype=np.float64)
    for i, t in enumerate(tokens):
        xt = bf16_to_f64(x_bits[t:t + 1])
        for j in range(k):
            e = int(idx[t, j])
            gr = expert_backward(xt, bf16_to_f64(w_gate_up_bits[e]), bf16_to_f64(w_down_bits[e]),
                                 g[t, j] * dyd[t:t + 1])
            dx[i] += gr["dx"][0]
            dgate[i, j] = float(np.dot(dyd[t], gr["out"][0]))
    dz = gates_backward(z[tokens], idx[tokens], dgate, renorm)
    dw_gate_up = np.zeros((len(experts),) + tuple(w_gate_up_bits.shape[1:]), dtype=np.float64)
    dw_down = np.zeros((len(experts),) + tuple(w_down_bits.shape[1:]), dtype=np.float64)
    for i, e in enumerate(experts):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        gr = expert_backward(bf16_to_f64(x_bits[tt]), bf16_to_f64(w_gate_up_bits[e]),
                             bf16_to_f64(w_down_bits[e]), g[tt, jj][:, None] * dyd[tt])
        dw_gate_up[i] = gr["dw_gate_up"]
        dw_down[i] = gr["dw_down"]
    return dict(dx=dx, dgate=dgate, dz=dz, dw_gate_up=dw_gate_up, dw_down=dw_down)


def backward_rounds(x_bits, w_gate_up_bits, w_down_bits, z, idx, dy, C: int,
                    renorm: bool = False, borrow: bool = False, gate=None) -> dict:
    """Literal round-by-round backward with recompute (tiny inputs only).

    For r = 0 .. R-1 of the forward's plan: dispatch copies the round's x rows and its
    gate * dy rows into two fixed buffers of E*C rows (per-expert rows e*C + slot, or packed
    expert after expert when borrowing, as in the forward executor); each expert with
    n[r, e] rows recomputes its forward on them and adds the round's dW1, dW3, dW2 into its
    accumulators; collect scatters each row's dx and dgate back to its pair. Nothing but
    the accumulators and the fixed buffers outlives a round. Returns the same dict as
    `backward` plus the plan."""
    idx = np.asarray(idx)
    T, k = idx.shape
    E = w_gate_up_bits.shape[0]
    d = w_down_bits.shape[1]
    g = gates(z, idx, renorm) if gate is None else np.asarray(gate, dtype=np.float64)
    dyd = np.asarray(dy, dtype=np.float64)
    x = bf16_to_f64(x_bits)
    p = plan_borrow(idx, E, C) if borrow else plan(idx, E, C)
    xbuf = np.zeros((E * C, d), dtype=np.float64)
    dbuf = np.zeros((E * C, d), dtype=np.float64)
    dx_terms = np.zeros((T, k, d), dtype=np.float64)
    dgate = np.zeros((T, k), dtype=np.float64)
    dw_gate_up = np.zeros(w_gate_up_bits.shape, dtype=np.float64)
    dw_down = np.zeros(w_down_bits.shape, dtype=np.float64)
    for r in range(p["R"]):
        n_r = [int(v) for v in p["n"][r]]
        base = [e * C for e in range(E)] if not borrow else [sum(n_r[:e]) for e in range(E)]
        rows = round_rows(p, idx, r)
        for (e, s, t, j) in rows:                      # dispatch x and gate * dy
            xbuf[base[e] + s] = x[t]
            dbuf[base[e] + s] = g[t, j] * dyd[t]
        grads = {}
        for e in range(E):                             # recompute + expert gradients
            n = n_r[e]
            if n:
                gr = expert_backward(xbuf[base[e]:base[e] + n], bf16_to_f64(w_gate_up_bits[e]),
                                     bf16_to_f64(w_down_bits[e]), dbuf[base[e]:base[e] + n])
                dw_gate_up[e] += gr["dw_gate_up"]
                dw_down[e] += gr["dw_down"]
                grads[e] = gr
        for (e, s, t, j) in rows:                      # collect dx and dgate
            dx_terms[t, j] = grads[e]["dx"][s]
            dgate[t, j] = float(np.dot(dyd[t], grads[e]["out"][s]))
    dx = np.zeros((T, d), dtype=np.float64)
    for j in range(k):
        dx = dx + dx_terms[:, j, :]
    return dict(dx=dx, dw_gate_up=dw_gate_up, dw_down=dw_down, dgate=dgate,
                dz=gates_backward(z, idx, dgate, renorm), plan=p)
