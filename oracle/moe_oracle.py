"""CPU oracle for the multi-round dropless MoE layer forward.

TEST INFRASTRUCTURE. This module is the plain, slow, obviously-correct statement of
what the layer computes. Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import it; the library itself never does, and it shares no
code with the CUDA path. Arithmetic is float64 (numpy); bf16 inputs are widened
exactly; nothing is blocked, fused or reordered beyond what is written here.

What the method computes, as the pages describe it:
  * "Frontier Pre-training at Microsoft AI (MAI-Base-2)" (wiki summary), Key claims,
    the multi-round dropless MoE item [section "Scaling MoE", Fig. 6]: experts run one
    or more dispatch -> compute -> collect rounds, each with a fixed per-expert token
    capacity; tokens over capacity wait for another round; memory is static whatever
    the imbalance; capacity is tunable.
  * "MAI-Base-2: Microsoft's 2.8T Model is a BREAKTHROUGH" (video transcript, 03:11
    chapter): overflow tokens wait for an extra round and no token is dropped.
  * "MAI-Base-2: Microsoft details its new training infrastructure", section
    "Optimizations to prevent memory loss": tokens beyond capacity are processed in
    further passes instead of being dropped.
  * "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups
    keep memory fixed when tokens pile up": a router sends each token to a few
    experts; raising capacity costs memory, lowering it costs rounds.

Because no token is dropped, the layer's output equals that of a capacity-free
dropless top-k MoE: the rounds change where and when each (token, expert) pair is
computed, never what. The oracle is therefore that plain definition
(`select_topk`, `gates`, `expert_ffn`, `forward`), plus the round plan stated on
its own (`plan`) and a literal round-by-round executor for tiny inputs
(`forward_rounds`) used to show, inside the oracle, that the rounds do not change
the result.

Readings where the pages are silent (each listed in the design notes):
  * gating: softmax over all E logits, then top-k, gates not renormalised unless
    asked (renorm=True). "parity unpinned": the pages never name the gate function.
  * selection order and ties: by logit descending, equal logits (+0 == -0) broken
    by the lower expert index.
  * which pairs go first: in ascending token order within each expert.
  * by default no capacity borrowing between experts: each expert owns C rows per
    round, so the round count is R = ceil(max_e load_e / C). `plan_borrow` states the
    pages' fuller rule (an overloaded expert takes capacity other experts leave unused,
    else an extra round); the order in which spare rows are handed out is not given,
    and the reading taken is "ascending expert index".
  * expert FFN: SwiGLU without biases, f(x) = W2 (silu(W1 x) * (W3 x)).
"""
from __future__ import annotations

import numpy as np


# --------------------------------------------------------------------------- formats

def bf16_to_f64(bits) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to float64.

    A bf16 value is the upper 16 bits of an IEEE binary32 value, so shifting the
    pattern into the top half of a 32-bit word gives that float32 exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- router

def router_logits(x_bits, w_router_bits, bias) -> np.ndarray:
    """Router logits z = x W_r^T + b, accumulated in float64 from the bf16 values and
    stored as float32. x: [T, d] bf16 bits, w_router: [E, d] bf16 bits, bias: [E] fp32.
    (Router weights are replicated on every rank in the pages' system, "Frontier
    Pre-training at Microsoft AI", Key claims, distributed Muon item.)"""
    x = bf16_to_f64(x_bits)
    w = bf16_to_f64(w_router_bits)
    z = x @ w.T
    if bias is not None:
        z = z + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return z.astype(np.float32)


def select_topk(z, k: int) -> np.ndarray:
    """The k experts with the largest logits per token, best first.

    Order: logit descending; equal logits (+0 and -0 compare equal) go to the lower
    expert index. Selection compares the fp32 logits themselves; softmax is
    monotone, so this is also the order of the softmax probabilities.
    Implemented as k passes of "take the first maximum among the not yet taken".
    """
    z = np.asarray(z, dtype=np.float32)
    T, E = z.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    if not np.all(np.isfinite(z)):
        raise ValueError("logits must be finite")
    cand = z.astype(np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    rows = np.arange(T)
    for j in range(k):
        best = np.argmax(cand, axis=1)          # first occurrence of the maximum
        idx[:, j] = best
        cand[rows, best] = -np.inf              # logits are finite, so -inf never wins again
    return idx


def gates(z, idx, renorm: bool = False) -> np.ndarray:
    """Gate of pair (t, j): the softmax probability of expert idx[t, j] over all E
    logits of token t, in float64: exp(z_e - m) / sum_e' exp(z_e' - m), m = max_e z_e.
    With renorm the k selected gates of a token are divided by their sum."""
    zd = np.asarray(z, dtype=np.float32).astype(np.float64)
    m = zd.max(axis=1, keepdims=True)
    p = np.exp(zd - m)
    p = p / p.sum(axis=1, keepdims=True)
    g = np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    if renorm:
        g = g / g.sum(axis=1, keepdims=True)
    return g


# --------------------------------------------------------------------------- round plan

def plan(idx, E: int, C: int) -> dict:
    """Assign every (token, expert) pair a round and a slot.

    rank(t, j)  = number of earlier tokens t' < t that also selected e = idx[t, j]
    round(t, j) = rank // C, slot(t, j) = rank % C
    load[e]     = number of tokens that selected e
    R           = ceil(max_e load[e] / C) rounds (0 if there are no pairs)
    n[r, e]     = rows expert e processes in round r = min(C, max(0, load[e] - r*C))
    offsets[e]  = sum of load[e'] for e' < e (expert-sorted pair order)
    Written as the plain counting loop over tokens in ascending order.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    if C < 1:
        raise ValueError("capacity C must be >= 1")
    count = [0] * E
    rank = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            rank[t, j] = count[e]
            count[e] += 1
    load = np.array(count, dtype=np.int64)
    max_load = int(load.max()) if E > 0 else 0
    R = (max_load + C - 1) // C
    n = np.clip(load[None, :] - C * np.arange(R, dtype=np.int64)[:, None], 0, C)
    offsets = np.concatenate([[0], np.cumsum(load)]).astype(np.int64)
    return dict(rank=rank, round=rank // C, slot=rank % C, load=load, R=R,
                max_load=max_load, n=n, offsets=offsets, C=C)


def plan_borrow(idx, E: int, C: int) -> dict:
    """Round plan with capacity borrowing.

    "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless
    MoE item: overflow tokens use unused capacity of other experts of the same group, and
    only otherwise go to an extra round; "MAI-Base-2: Microsoft details its new training
    infrastructure", section "Optimizations to prevent memory loss": the system can reuse
    capacity other experts leave unallocated. A round holds at most E*C rows (the fixed
    buffer). Reading where the pages are silent: in each round every expert first takes up
    to C of its pending pairs; the rows left unused by that are handed to experts that still
    have pending pairs, in ascending expert index, each taking what it has pending or what is
    left. An expert's pairs still go in ascending token order: its pairs with ranks
    [start[r, e], start[r, e] + n[r, e]) form its rows of round r, at slots 0 .. n[r, e]-1.
    Written as the plain loop over rounds.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    if C < 1:
        raise ValueError("capacity C must be >= 1")
    count = [0] * E
    rank = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            rank[t, j] = count[e]
            count[e] += 1
    load = np.array(count, dtype=np.int64)
    pending = load.copy()
    rounds = []
    while pending.sum() > 0:
        own = np.minimum(pending, C)                 # each expert's own C rows first
        spare = E * C - int(own.sum())               # rows nobody took that way
        extra = np.zeros(E, dtype=np.int64)
        for e in range(E):                           # lent in ascending expert order
            want = int(pending[e] - own[e])
            take = min(want, spare)
            extra[e] = take
            spare -= take
        n_r = own + extra
        rounds.append(n_r)
        pending = pending - n_r
    R = len(rounds)
    n = np.array(rounds, dtype=np.int64).reshape(R, E)
    start = np.zeros((R + 1, E), dtype=np.int64)     # start[r, e]: pairs of e in rounds < r
    for r in range(R):
        start[r + 1] = start[r] + n[r]
    rnd = np.empty((T, k), dtype=np.int64)
    slot = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            r = 0
            while rank[t, j] >= start[r + 1, e]:
                r += 1
            rnd[t, j] = r
            slot[t, j] = rank[t, j] - start[r, e]
    max_load = int(load.max()) if E > 0 else 0
    offsets = np.concatenate([[0], np.cumsum(load)]).astype(np.int64)
    return dict(rank=rank, round=rnd, slot=slot, load=load, R=R, max_load=max_load, n=n,
                offsets=offsets, C=C)


def round_rows(p: dict, idx, r: int) -> list:
    """The rows of round r as (expert, slot, token, j) tuples, ordered by expert then
    slot: the contents of the round's fixed [E, C, d] dispatch buffer."""
    idx = np.asarray(idx)
    rows = []
    T, k = idx.shape
    for t in range(T):
        for j in range(k):
            if p["round"][t, j] == r:
                rows.append((int(idx[t, j]), int(p["slot"][t, j]), t, j))
    rows.sort()
    return rows


# --------------------------------------------------------------------------- experts

def silu(u):
    return u / (1.0 + np.exp(-u))


def expert_hidden(xrows, w_gate_up_e) -> np.ndarray:
    """SwiGLU hidden activations silu(x W1^T) * (x W3^T) for rows x (float64 [n, d]).
    w_gate_up_e: [2F, d] float64, rows 0..F-1 = W1 (gate), rows F..2F-1 = W3 (up)."""
    F = w_gate_up_e.shape[0] // 2
    a = xrows @ w_gate_up_e[:F].T
    b = xrows @ w_gate_up_e[F:].T
    return silu(a) * b


def expert_ffn(xrows, w_gate_up_e, w_down_e) -> np.ndarray:
    """f_e(x) = W2 (silu(W1 x) * (W3 x)) for rows x; w_down_e: [d, F] float64."""
    return expert_hidden(xrows, w_gate_up_e) @ w_down_e.T


def forward(x_bits, w_gate_up_bits, w_down_bits, idx, gate, tokens=None) -> np.ndarray:
    """Capacity-free dropless MoE output y[t] = sum_j gate[t, j] * f_{idx[t, j]}(x_t),
    float64. Per-pair terms are added in j order. `tokens` restricts the output to
    a subset of tokens (each token's output depends only on its own row), which is
    how large workloads are checked on samples."""
    idx = np.asarray(idx)
    gate = np.asarray(gate, dtype=np.float64)
    T, k = idx.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    nt = tok.size
    E = w_gate_up_bits.shape[0]
    d = w_down_bits.shape[1]
    if nt * k * d * 8 > (8 << 30):
        raise MemoryError("oracle forward on this many tokens needs a token sample")
    sub_idx = idx[tok]
    terms = np.zeros((nt, k, d), dtype=np.float64)
    for e in range(E):
        where = np.nonzero(sub_idx == e)              # (rows into tok, j)
        if where[0].size == 0:
            continue
        w13 = bf16_to_f64(w_gate_up_bits[e])
        w2 = bf16_to_f64(w_down_bits[e])
        xe = bf16_to_f64(x_bits[tok[where[0]]])
        out = expert_ffn(xe, w13, w2)
        terms[where[0], where[1], :] = gate[tok[where[0]], where[1]][:, None] * out
    y = np.zeros((nt, d), dtype=np.float64)
    for j in range(k):
        y = y + terms[:, j, :]
    return y


def forward_rounds(x_bits, w_gate_up_bits, w_down_bits, idx, gate, C: int,
                   borrow: bool = False) -> tuple:
    """Literal multi-round executor (tiny inputs only).

    For r = 0 .. R-1: dispatch copies the round's pairs into a fixed buffer of E*C rows;
    compute runs each expert's FFN on its n[r, e] rows; collect writes gate * output back
    to the pair. Without borrowing the buffer is [E, C, d] (expert e's rows at e*C + slot);
    with borrowing (`plan_borrow`) an expert may hold more than C rows of a round, so the
    round's rows are packed expert after expert (expert e's rows at
    sum_{e' < e} n[r, e'] + slot). Either way the buffer never grows with the routing.
    Returns (y, plan, max rows any round held for one expert)."""
    idx = np.asarray(idx)
    gate = np.asarray(gate, dtype=np.float64)
    T, k = idx.shape
    E = w_gate_up_bits.shape[0]
    d = w_down_bits.shape[1]
    p = plan_borrow(idx, E, C) if borrow else plan(idx, E, C)
    x = bf16_to_f64(x_bits)
    buf = np.zeros((E * C, d), dtype=np.float64)
    terms = np.zeros((T, k, d), dtype=np.float64)
    peak = 0
    for r in range(p["R"]):
        n_r = [int(v) for v in p["n"][r]]
        base = [e * C for e in range(E)] if not borrow else [sum(n_r[:e]) for e in range(E)]
        rows = round_rows(p, idx, r)
        for (e, s, t, j) in rows:                      # dispatch
            buf[base[e] + s, :] = x[t]
        outs = {}
        for e in range(E):                             # compute
            n = n_r[e]
            peak = max(peak, n)
            if n:
                outs[e] = expert_ffn(buf[base[e]:base[e] + n], bf16_to_f64(w_gate_up_bits[e]),
                                     bf16_to_f64(w_down_bits[e]))
        for (e, s, t, j) in rows:                      # collect
            terms[t, j, :] = gate[t, j] * outs[e][s]
    y = np.zeros((T, d), dtype=np.float64)
    for j in range(k):
        y = y + terms[:, j, :]
    return y, p, peak


def layer(x_bits, w_gate_up_bits, w_down_bits, k: int, C: int, logits=None,
          w_router_bits=None, bias=None, renorm: bool = False, tokens=None) -> dict:
    """The whole layer forward on the CPU: router -> top-k -> plan -> output."""
    if logits is None:
        logits = router_logits(x_bits, w_router_bits, bias)
    idx = select_topk(logits, k)
    g = gates(logits, idx, renorm)
    E = w_gate_up_bits.shape[0]
    p = plan(idx, E, C)
    y = forward(x_bits, w_gate_up_bits, w_down_bits, idx, g, tokens=tokens)
    return dict(logits=np.asarray(logits, np.float32), idx=idx, gate=g, plan=p, y=y)
