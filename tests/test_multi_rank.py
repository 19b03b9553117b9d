"""The N > 1 host logic of bench.py on CPU: two gloo ranks, replicas of the same
workload (no data-path collective), job time = max over ranks, job throughput =
all ranks' units / that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    assert bench.dist_env() == (rank, rank, world)
    bench.init_dist(world, "gloo")
    try:
        bench.barrier()
        # each rank "measured" a different time; the job time is the slowest rank's
        t = bench.max_over_ranks(10.0 + rank)
        thr = bench.job_throughput(4096 * 5, world, t / 1e3)
        out.put((rank, t, thr))
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_sum_the_work():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, thr in res:
        assert t == pytest.approx(11.0)                       # max over ranks, on every rank
        assert thr == pytest.approx(2 * 4096 * 5 / 0.011)     # weak scaling: both ranks' tokens


def test_single_process_needs_no_process_group():
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(100, 1, 2.0) == 50.0


def test_algorithmic_work_figures():
    import bench
    # model-shape prefill: 206.0 MB moved, 23.6 GFLOP of dense tensor-core work
    assert bench.prefill_bytes(4096, 1) == 206045184
    assert bench.prefill_tc_flops(4096) == 4096 * 32 * (6 * 128 * 128 + 10 * 64 * 128)
    # decode: two passes over a 64 KiB fp32 state per (sequence, head) plus the token
    assert bench.decode_bytes(256) == 256 * 32 * (2 * 128 * 128 * 4 + 4 * 128 * 2 + 128 * 4 + 4)
