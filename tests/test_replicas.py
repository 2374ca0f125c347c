"""The N-replica bookkeeping of bench.py on CPU: two gloo ranks meet at the
barrier, both take the slower rank's time, and the whole-job value counts
both ranks' steps; one rank exchanges nothing; the reference arm runs on
rank 0 only.  (The verify step does not shard: each GPU runs a replica.)"""
import datetime
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        reps = bench.Replicas(world, rank, torch.device("cpu"))
        reps.barrier()
        step_ms = reps.max_over_ranks(1.0 + rank)  # rank 1 is the slower replica
        reps.barrier()
        q.put((rank, step_ms, reps.job_value(step_ms)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert [r for r, _, _ in results] == [0, 1]
    for _, step_ms, value in results:
        assert step_ms == 2.0
        assert value == 2 * 1e3 / 2.0


def test_one_rank_exchanges_nothing():
    reps = bench.Replicas(1, 0, torch.device("cpu"))
    reps.barrier()
    assert reps.max_over_ranks(3.5) == 3.5
    assert reps.job_value(2.0) == 500.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        warmup, steps, gpus = 3, 1, 2

    bench.run_reference(Args, bench.CONFIGS["tiny"], 1)
    assert capsys.readouterr().out == ""
