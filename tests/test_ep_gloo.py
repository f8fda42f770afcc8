"""Exchange tables of the expert-parallel form (moe_ep_exchange_plan, host code in libmoe.so),
run as gloo ranks on the CPU.

Every rank routes its own seeded tokens (the oracle's top-k selection stands in for the GPU's
router here), counts its pairs per expert, all-gathers the counts over gloo, and asks the
library for its tables. Checked: each rank's tables equal the expert-parallel oracle's
(oracle.ep_plan) bit for bit, and what a rank expects to receive from each other rank in each
round is exactly what that rank computed it would send (exchanged with a real all-to-all)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from dropless_moe_layer_b200 import moe


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_idx(rank, T, E, k, skew):
    rng = np.random.default_rng(1000 + rank)
    z = rng.standard_normal((T, E)) - skew * np.log1p(rng.permutation(E))[None, :]
    return oracle.select_topk(z.astype(np.float32), k)


def _rank_main(rank, world, port, cfg, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, E, k, C, skew = cfg
        idx = _rank_idx(rank, T, E, k, skew)
        mine = torch.from_numpy(np.bincount(idx.ravel(), minlength=E).astype(np.int32))
        gathered = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, mine)
        loads = torch.stack(gathered).numpy()
        shape = moe.make_shape(T, 64, E, k, 64, C)
        tab = moe.ep_exchange_plan(shape, world, rank, loads)
        # every rank runs the same number of rounds; exchange this round's send counts
        R = tab["R"]
        got_from = np.zeros((R, world), dtype=np.int32)
        for r in range(R):
            recv = torch.zeros(world, dtype=torch.int32)
            dist.all_to_all_single(recv, torch.from_numpy(tab["send_counts"][r].copy()))
            got_from[r] = recv.numpy()
        out[rank] = dict(tab=tab, got_from=got_from, loads=loads)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, cfg):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), cfg, out), nprocs=world,
                           start_method="spawn", join=True)
        return dict(out)


@pytest.mark.parametrize("world,cfg", [(2, (40, 8, 2, 7, 1.5)), (4, (33, 16, 4, 16, 1.0)),
                                       (2, (25, 4, 4, 1, 0.0))], ids=["2ranks", "4ranks", "2ranks-C1-k=E"])
def test_exchange_tables_match_oracle_over_gloo(world, cfg):
    T, E, k, C, skew = cfg
    res = _run(world, cfg)
    p = oracle.ep_plan([_rank_idx(s, T, E, k, skew) for s in range(world)], E, C, world)
    per = E // world
    for s in range(world):
        tab, got = res[s]["tab"], res[s]["got_from"]
        assert np.array_equal(res[s]["loads"], p["load"])
        assert tab["R"] == p["R"]
        assert np.array_equal(tab["base"], p["base"][s])
        assert np.array_equal(tab["send_counts"], p["send"][:, s, :])
        assert np.array_equal(tab["send_offsets"], p["send_off"][:, s, :])
        assert np.array_equal(tab["recv_counts"], p["send"][:, :, s])
        assert np.array_equal(tab["recv_offsets"], p["recv_off"][:, s, :])
        assert np.array_equal(tab["n_owned"], p["n"][:, s * per:(s + 1) * per])
        # what the other ranks said they send is what this rank computed it receives
        assert np.array_equal(got, tab["recv_counts"])


def test_exchange_plan_rejects_bad_arguments():
    lib = moe.load_library()
    shape = moe.make_shape(4, 64, 6, 2, 64, 3)
    P = __import__("ctypes").POINTER(moe.c_i32)
    R = moe.c_i32(-1)
    ok = np.array([[2, 2, 2, 1, 1, 0], [0, 0, 0, 0, 0, 8]], dtype=np.int32)
    call = lambda G, rank, loads: lib.moe_ep_exchange_plan(  # noqa: E731
        __import__("ctypes").byref(shape), G, rank, loads.ctypes.data_as(P), 0, __import__("ctypes").byref(R),
        None, None, None, None, None, None)
    assert call(2, 0, ok) == 0 and R.value == 3            # expert 5 holds 8 pairs: ceil(8 / 3)
    assert call(4, 0, ok) == -1                            # 6 experts do not split over 4 ranks
    assert call(2, 2, ok) == -1                            # rank out of range
    bad = ok.copy()
    bad[0, 0] = 3                                          # rank 0's counts no longer add up to T k
    assert call(2, 0, bad) == -1
    bad = ok.copy()
    bad[1, 0] = -1
    assert call(2, 0, bad) == -1


def test_ep_workspace_size_is_fixed_by_shape_and_ranks():
    lib = moe.load_library()
    s = moe.make_shape(256, 128, 8, 2, 256, 32)
    n2, n4 = lib.moe_ep_workspace_bytes(__import__("ctypes").byref(s), 2), lib.moe_ep_workspace_bytes(
        __import__("ctypes").byref(s), 4)
    assert 0 < n2 < n4                               # more ranks: more possible rounds to plan
    assert lib.moe_ep_workspace_bytes(__import__("ctypes").byref(s), 3) == 0     # 8 experts over 3 ranks
    assert lib.moe_ep_workspace_bytes(__import__("ctypes").byref(s), 0) == 0
