"""CPU oracle for the expert-parallel form of the multi-round dropless MoE layer.

TEST INFRASTRUCTURE, like the rest of `oracle/`: only the test suite, the smoke check and the
benchmark's CPU legs may import it; the library shares no code with it. Arithmetic is float64.

What the pages say about the expert-parallel form:
  * "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, the multi-round dropless
    MoE item [section "Scaling MoE", Fig. 6]: the experts are split into groups, one group per
    expert-parallel rank; each group runs one or more dispatch -> compute -> collect rounds with a
    fixed per-expert token capacity; the token metadata stays on the device and the exchange
    runs as an all-to-all over symmetric memory.
  * "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups keep
    memory fixed when tokens pile up": a router sends each token to a few experts; tokens over
    an expert's capacity wait for another round instead of being dropped.

Readings where the pages are silent (each listed in the design notes):
  * G ranks, E divisible by G; rank g owns the E/G contiguous experts [g E/G, (g+1) E/G).
  * Every rank routes its own tokens (the router is replicated), with the selection rule and
    gates of the single-GPU oracle.
  * An expert's capacity C per round is shared by all the ranks that send to it. The pairs of
    expert e are ranked over the whole job in the order (source rank ascending, token ascending);
    round = rank // C and slot = rank % C, as on one GPU. The plan of the job is therefore the
    single-GPU plan of the ranks' batches concatenated in rank order, split back by rank.
  * Every rank runs the same R = ceil(max_e (total load of e) / C) rounds, because the exchange
    of each round is a collective step.
  * In round r, rank s sends rank g its pairs of round r whose expert g owns, ordered by
    (expert, slot); rank g receives the chunks of the ranks in ascending source order. The
    results come back the same way, and rank s adds them into its outputs in its own
    (round, j) order.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import bf16_to_f64, expert_ffn


def owner(e: int, E: int, G: int) -> int:
    """The rank that holds expert e: experts are split into G contiguous groups of E/G."""
    return e // (E // G)


def ep_plan(idx_list, E: int, C: int, G: int) -> dict:
    """Round plan and exchange tables of an expert-parallel layer over G ranks.

    idx_list[s] is rank s's top-k selection [T_s, k]. Written as the plain counting loop over
    ranks, then tokens, then the token's k pairs. Returns
      rank[s], round[s], slot[s]: [T_s, k] per rank (the global rank of the pair in its expert)
      load [G, E]: pairs of rank s routed to expert e;  total [E] = load summed over ranks
      base [G, E]: pairs of expert e on ranks before s (= where rank s's pairs of e start)
      R: rounds of the job;  n [R, E]: rows of expert e in round r (from all ranks)
      send [R, G, G]: send[r, s, g] = pairs rank s sends rank g in round r
      send_off [R, G, G]: send_off[r, s, g] = sum of send[r, s, g'] for g' < g (position of the
          chunk for g in s's packed round-r rows); recv_off [R, G, G]: recv_off[r, g, s] = sum
          of send[r, s', g] for s' < s (position of s's chunk in g's received rows)
      rows [R][s]: rank s's pairs of round r in packed order, as (e, slot, t, j).
    """
    if E % G != 0:
        raise ValueError("E must be a multiple of G")
    if C < 1:
        raise ValueError("capacity C must be >= 1")
    count = [0] * E
    load = np.zeros((G, E), dtype=np.int64)
    ranks, rounds, slots = [], [], []
    for s in range(G):
        idx = np.asarray(idx_list[s])
        T, k = idx.shape
        rk = np.empty((T, k), dtype=np.int64)
        for t in range(T):
            for j in range(k):
                e = int(idx[t, j])
                rk[t, j] = count[e]
                count[e] += 1
                load[s, e] += 1
        ranks.append(rk)
        rounds.append(rk // C)
        slots.append(rk % C)
    total = load.sum(axis=0)
    base = np.zeros((G, E), dtype=np.int64)
    for s in range(1, G):
        base[s] = base[s - 1] + load[s - 1]
    R = int((int(total.max()) + C - 1) // C) if total.size else 0
    n = np.clip(total[None, :] - C * np.arange(R, dtype=np.int64)[:, None], 0, C)
    send = np.zeros((R, G, G), dtype=np.int64)
    rows = [[[] for _ in range(G)] for _ in range(R)]
    for s in range(G):
        idx = np.asarray(idx_list[s])
        T, k = idx.shape
        for t in range(T):
            for j in range(k):
                e = int(idx[t, j])
                r = int(rounds[s][t, j])
                send[r, s, owner(e, E, G)] += 1
                rows[r][s].append((e, int(slots[s][t, j]), t, j))
    for r in range(R):
        for s in range(G):
            rows[r][s].sort()
    send_off = np.zeros_like(send)
    recv_off = np.zeros_like(send)
    for r in range(R):
        for s in range(G):
            for g in range(1, G):
                send_off[r, s, g] = send_off[r, s, g - 1] + send[r, s, g - 1]
        for g in range(G):
            for s in range(1, G):
                recv_off[r, g, s] = recv_off[r, g, s - 1] + send[r, s - 1, g]
    return dict(rank=ranks, round=rounds, slot=slots, load=load, total=total, base=base, R=R, n=n,
                send=send, send_off=send_off, recv_off=recv_off, rows=rows, C=C, G=G)


def ep_forward(x_list, w_gate_up_bits, w_down_bits, idx_list, gate_list, C: int, G: int) -> tuple:
    """Literal expert-parallel executor (tiny inputs only).

    For every round: each rank packs its pairs of the round by (expert, slot) and cuts them
    into one chunk per owner rank; the chunks are exchanged; each owner places the rows it
    received into its fixed buffer of E/G * C rows (local expert l at rows l*C + slot), runs
    each expert's FFN on its n[r, e] rows, and sends every result row back to where it came
    from; each rank then adds gate * result into its own pair terms. Returns (y_list, plan,
    largest number of rows any expert held in a round), y_list[s] [T_s, d] float64."""
    E = w_gate_up_bits.shape[0]
    d = w_down_bits.shape[1]
    per = E // G
    p = ep_plan(idx_list, E, C, G)
    xs = [bf16_to_f64(x) for x in x_list]
    terms = [np.zeros((np.asarray(i).shape[0], np.asarray(i).shape[1], d)) for i in idx_list]
    peak = 0
    for r in range(p["R"]):
        # pack and cut: chunk[s][g] = rank s's rows of round r owned by g, in (expert, slot) order
        chunk = [[[row for row in p["rows"][r][s] if owner(row[0], E, G) == g] for g in range(G)]
                 for s in range(G)]
        results = {}
        for g in range(G):                                   # on owner rank g
            buf = np.zeros((per * C, d))
            filled = np.zeros(per * C, dtype=bool)
            for s in range(G):                               # received in source order
                for (e, slot, t, j) in chunk[s][g]:
                    row = (e - g * per) * C + slot
                    if filled[row]:
                        raise AssertionError("two pairs in one buffer row")
                    filled[row] = True
                    buf[row] = xs[s][t]
            for l in range(per):
                e = g * per + l
                nr = int(p["n"][r, e])
                peak = max(peak, nr)
                if nr == 0:
                    continue
                if not filled[l * C:l * C + nr].all():
                    raise AssertionError("a row of an expert's round is missing")
                out = expert_ffn(buf[l * C:l * C + nr], bf16_to_f64(w_gate_up_bits[e]),
                                 bf16_to_f64(w_down_bits[e]))
                for s in range(G):                           # results go back to their senders
                    for (ee, slot, t, j) in chunk[s][g]:
                        if ee == e:
                            results[(s, t, j)] = out[slot]
        for s in range(G):                                   # collect on the source rank
            gate = np.asarray(gate_list[s], dtype=np.float64)
            for (e, slot, t, j) in p["rows"][r][s]:
                terms[s][t, j] = gate[t, j] * results[(s, t, j)]
    ys = []
    for s in range(G):
        T, k = terms[s].shape[:2]
        y = np.zeros((T, d))
        for j in range(k):
            y = y + terms[s][:, j, :]
        ys.append(y)
    return ys, p, peak
