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
    # model-shape prefill: 206.0 MB moved; 18.25 GFLOP of tensor-core work counted
    # triangle-aware (139,264 flops per token-head), 23.6 GFLOP as issued on dense tiles
    assert bench.prefill_bytes(4096, 1) == 206045184
    assert bench.prefill_tc_flops(4096) == 4096 * 32 * 139264
    assert bench.prefill_tc_flops_issued(4096) == 4096 * 32 * (6 * 128 * 128 + 10 * 64 * 128)
    # decode: two passes over a 64 KiB fp32 state per (sequence, head) plus the token
    assert bench.decode_bytes(256) == 256 * 32 * (2 * 128 * 128 * 4 + 4 * 128 * 2 + 128 * 4 + 4)


def test_traffic_figure_is_tied_to_the_kernel_sources(tmp_path, monkeypatch):
    import json
    import bench
    # the committed figure is reported only while the kernel sources hash the same
    j = json.load(open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")))
    expected = float(j["bytes_per_call"]) if j["source_sha256"] == bench.kernel_sources_sha256() else None
    assert bench.load_traffic() == expected
    assert bench.load_traffic(123.0) == 123.0  # an explicit figure wins
    # a figure captured from other sources reads null
    fake_root = tmp_path / "root"
    (fake_root / "profiles").mkdir(parents=True)
    (fake_root / "profiles" / "traffic.json").write_text(json.dumps({"source_sha256": "0" * 64, "bytes_per_call": 1.0}))
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    monkeypatch.setattr(bench, "kernel_sources_sha256", lambda: "f" * 64)
    assert bench.load_traffic() is None


def test_launch_count_follows_the_dispatch():
    import bench
    assert bench.kernels_per_call(256) == 1          # status word only: single-pass kernel
    assert bench.kernels_per_call(303_000_000) == 3  # two-pass scratch: plan, intra, recurrence


def test_mixer_decode_work_figure():
    import bench
    # state r+w, conv history r+w (3 tensors x 3 rows, bf16), q/k/v/gate/out bf16, log_alpha, beta, index
    per_seq_head = 2 * 128 * 128 * 4 + 2 * 9 * 128 * 2 + 5 * 128 * 2 + 128 * 4 + 4
    assert bench.mixer_decode_bytes(256) == 256 * 32 * per_seq_head + 256 * 4


def test_mixer_decode_tokens_work_figure():
    import bench
    assert bench.mixer_decode_tokens_bytes(256, 1) == bench.mixer_decode_bytes(256)
    per_token = 5 * 128 * 2 + 128 * 4 + 4
    assert bench.mixer_decode_tokens_bytes(256, 4) - bench.mixer_decode_tokens_bytes(256, 1) == 256 * 32 * 3 * per_token


def test_backward_work_figure():
    import bench
    # per token-head: q, k, v, d_out bf16 and log_alpha fp32 + beta read; dq, dk, dv,
    # d_log_alpha fp32 + d_beta written; per chain: initial state, d_final read, d_initial written
    per_tok = 4 * 128 * 2 + 128 * 4 + 4 + 4 * 128 * 4 + 4
    assert per_tok == 3592
    assert bench.backward_bytes(4096, 1) == 4096 * 32 * per_tok + 3 * 32 * 128 * 128 * 4
    assert bench.backward_bytes(0, 2) == 3 * 2 * 32 * 128 * 128 * 4


def test_reference_arm_line_on_the_host():
    """`bench.py --impl reference` times the fp64 oracle on the host (no GPU) and prints
    one line on the headline's metric, unit and config, with the sample it timed."""
    import json
    import subprocess
    import sys
    import bench
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=bench.ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == "tokens/s"
    assert j["higher_is_better"] is True and j["steps"] == 1 and j["n_gpus"] == 1
    assert j["config"] == bench.headline_config(1)
    assert j["value"] > 0 and j["cpu_baseline"]["value"] == j["value"]
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1 and j["cpu_baseline"]["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
