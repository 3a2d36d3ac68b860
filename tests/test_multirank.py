"""The multi-rank path of the benchmark on CPU (gloo, world size 2): every rank serves its own
batch of the same shape (the path shards by sequences with no exchange), the step time is the
maximum over ranks, and the job throughput counts every rank's sequences."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = bench.rank_workload(rank)
        local_ms = 1.0 + rank * 0.5                     # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.job_throughput(wl.num_seqs, world, ms)
        out.put((rank, ms, value, wl.num_seqs, wl.seq_lens.copy(), bench.dist_env()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, n0, lens0, env0), (r1, ms1, v1, n1, lens1, env1) = res
    assert ms0 == ms1 == 1.5                                 # max over ranks
    assert v0 == v1 == pytest.approx(2 * 64 / 1.5e-3)        # every rank's sequences, slowest time
    assert n0 == n1 == 64 and lens0.shape == lens1.shape      # same shapes (weak scaling)
    assert not np.array_equal(lens0, lens1)                   # each rank its own batch
    assert env0 == (0, 0, 2) and env1 == (1, 1, 2)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_throughput(64, 1, 0.1) == pytest.approx(640000.0)
