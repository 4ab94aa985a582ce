"""The multi-GPU benchmark path, on CPU: two gloo ranks.

Decode shards by sequence with no collective in the data path; the only
cross-rank step is the timing aggregation (max of the timed milliseconds, sum of
the bytes and sequences processed).  These tests run it with world_size 2 on the
gloo backend and check the numbers each rank sees.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    bench.init_dist(world, "gloo")
    try:
        # rank r timed (10 + r) ms for its own batch of (100 + r) MB and 256 sequences
        ms, nbytes, seqs = bench.aggregate(10.0 + rank, (100 + rank) * 1e6, 256.0)
        bench.barrier()
        world_env, rank_env, local_env = bench.dist_env()
        # the bench line's figures: rank r ran 4 steps of (0.1 + 0.01 r) ms over its
        # own batch of (800 + r) MB and 256 sequences
        per_step, gbs, seqs_s = bench.job_throughput([0.1 + 0.01 * rank] * 4, (800 + rank) * 1e6, 256.0)
        q.put((rank, ms, nbytes, seqs, world_env, rank_env, local_env, per_step, gbs, seqs_s))
    finally:
        dist.destroy_process_group()


def test_aggregate_takes_max_time_and_total_work_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, nbytes, seqs, world_env, rank_env, local_env, per_step, gbs, seqs_s in results:
        assert ms == 11.0                     # the slower rank's time
        assert nbytes == 201e6                # both ranks' bytes
        assert seqs == 512.0
        assert (world_env, rank_env, local_env) == (2, rank, rank)
        # slowest rank: 0.11 ms per step; both ranks' 1601 MB per step over it
        assert per_step == pytest.approx(0.11)
        assert gbs == pytest.approx(1601e6 / 0.11e-3 / 1e9)
        assert seqs_s == pytest.approx(512 / 0.11e-3)


def test_single_process_aggregate_is_identity():
    import bench

    assert not dist.is_initialized()
    assert bench.aggregate(3.5, 7.0, 2.0) == (3.5, 7.0, 2.0)


def test_gpus_flag_launches_one_rank_per_gpu():
    import bench

    cmd = bench.rank_launch_command(["--gpus", "4", "--steps", "3"], 4, 29555)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29555" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"] and cmd[-5].endswith("bench.py")


def test_job_throughput_single_process():
    import bench

    per_step, gbs, seqs_s = bench.job_throughput([0.2, 0.2], 1e9, 100.0)
    assert per_step == pytest.approx(0.2)
    assert gbs == pytest.approx(1e9 / 0.2e-3 / 1e9)
    assert seqs_s == pytest.approx(100 / 0.2e-3)
