"""Expert-parallel data path (moe_ep_*) against the oracle, with G ranks emulated on one GPU.

Each emulated rank has its own tokens, workspace and buffers and holds only its own E/G experts'
weights. The exchange between ranks, which on real ranks is an all-to-all (NCCL), is done here by
plain device copies ordered on the host: every rank packs round r, then each owner's received
rows are assembled from the chunks addressed to it in source order, then every owner runs its
experts, then the results go back the same way, then every rank combines. No kernel waits on
another rank's kernel. Checked: every rank's layer output equals the capacity-free dropless
output of its own tokens (within the forward's 2e-2 bar), the job runs the oracle's number of
rounds, and the exchanged counts are the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl
from dropless_moe_layer_b200.ep import ExpertParallelRank

pytestmark = pytest.mark.gpu

Y_TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def _run(G, T, d, E, k, F, C, seed):
    dev = torch.device("cuda")
    gen = torch.Generator(device="cpu").manual_seed(seed)
    zs = [(torch.randn(T, E, generator=gen) - 1.2 * torch.log1p(torch.randperm(E, generator=gen).double()).float())
          .contiguous() for _ in range(G)]
    xs = [torch.randn(T, d, generator=gen).to(torch.bfloat16) for _ in range(G)]
    w13 = (torch.randn(E, 2 * F, d, generator=gen) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(E, d, F, generator=gen) * 0.02).to(torch.bfloat16)
    per = E // G
    ranks = [ExpertParallelRank(T, d, E, k, F, C, G, s, device=dev) for s in range(G)]
    xd = [x.to(dev) for x in xs]
    loads = np.stack([rk.route(logits=z.to(dev)) for rk, z in zip(ranks, zs)])
    Rs = {rk.plan(loads) for rk in ranks}
    assert len(Rs) == 1
    R = Rs.pop()
    w13_local = [w13[g * per:(g + 1) * per].to(dev).contiguous() for g in range(G)]
    w2_local = [w2[g * per:(g + 1) * per].to(dev).contiguous() for g in range(G)]
    ys = [torch.empty(T, d, dtype=torch.float32, device=dev) for _ in range(G)]
    for r in range(R):
        sends = [rk.pack(r, x) for rk, x in zip(ranks, xd)]
        for g, owner in enumerate(ranks):              # all-to-all: chunk g of every rank, source order
            at = 0
            for s, src in enumerate(ranks):
                off, cnt = int(src.tables["send_offsets"][r][g]), int(src.tables["send_counts"][r][g])
                assert int(owner.tables["recv_counts"][r][s]) == cnt
                owner.recvbuf[at:at + cnt].copy_(sends[s][off:off + cnt])
                at += cnt
        outs = [rk.experts(r, w13_local[g], w2_local[g]) for g, rk in enumerate(ranks)]
        for s, src in enumerate(ranks):                # and back
            for g, owner in enumerate(ranks):
                off, cnt = int(owner.tables["recv_offsets"][r][s]), int(owner.tables["recv_counts"][r][s])
                soff = int(src.tables["send_offsets"][r][g])
                src.retbuf[soff:soff + cnt].copy_(outs[g][off:off + cnt])
        for rk, y in zip(ranks, ys):
            rk.combine(r, y)
    torch.cuda.synchronize()
    for rk in ranks:
        assert rk.layer.device_status() == 0
    # oracle: the job's plan over the concatenated batch, and each rank's capacity-free output
    idx = [oracle.select_topk(z.numpy(), k) for z in zs]
    p = oracle.ep_plan(idx, E, C, G)
    assert R == p["R"] and R >= 2
    for s, rk in enumerate(ranks):
        assert np.array_equal(rk.tables["send_counts"], p["send"][:, s, :])
    w13b, w2b = wl.bf16_bits(w13), wl.bf16_bits(w2)
    for s in range(G):
        ref = oracle.forward(wl.bf16_bits(xs[s]), w13b, w2b, idx[s], oracle.gates(zs[s].numpy(), idx[s]))
        got = ys[s].cpu().numpy()
        err = float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))
        assert err <= Y_TOL, (s, err)


@pytest.mark.parametrize("G,T,d,E,k,F,C", [(2, 256, 128, 8, 2, 256, 32), (4, 200, 256, 16, 4, 128, 24),
                                           (2, 1024, 512, 16, 4, 512, 160)],
                         ids=["2ranks-tiny", "4ranks-ragged", "2ranks-1k"])
def test_expert_parallel_layer_matches_oracle(G, T, d, E, k, F, C):
    _run(G, T, d, E, k, F, C, seed=G * 1000 + T)


def test_rejects_bad_counts():
    ranks = ExpertParallelRank(64, 128, 8, 2, 128, 16, 2, 0, device="cuda")
    ranks.route(logits=torch.randn(64, 8, device="cuda"))
    bad = np.zeros((2, 8), dtype=np.int32)
    with pytest.raises(moe.MoeError):
        ranks.plan(bad)                                # this rank's counts no longer match its plan
