"""Host logic of the multi-GPU benchmark (replicas, no data-path collective), run as two
gloo ranks on the CPU: the job time is the max over ranks, the throughput counts every
rank's tokens, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
        job = bench.max_over_ranks(local_ms, dist, "cpu")
        out[rank] = (job, bench.job_throughput(4096, 20, world, job))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == pytest.approx(4096 * 2 * 20 / 0.015)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(100, 10, 1, 1000.0) == 1000.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    class A:
        steps, warmup, gpus = 1, 1, 2
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(A, bench.wl.BY_NAME["tiny-zipf1"])   # must return without work
    assert capsys.readouterr().out == ""
