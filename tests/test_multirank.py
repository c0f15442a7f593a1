"""The multi-rank plumbing of bench.py, on CPU: two gloo ranks.

The decode path shards into independent (batch, kv-head) units, so several
GPUs run replicas with no collective on the data path; the only exchanges are
the barriers around the timed region and the max over ranks of the device
time, from which the whole-job rate is computed.  These run here on gloo.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = 10.0 + 5.0 * rank  # the ranks' device times differ
        slowest = bench.max_over_ranks(ms, world)
        results.put((rank, slowest, bench.whole_job_rate(world, 100, slowest)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(results.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1]
    for _, slowest, rate in got:
        assert slowest == 15.0
        # 2 ranks x 100 steps in the slowest rank's 15 ms
        assert rate == pytest.approx(2 * 100 / 0.015)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the CPU reference arm runs on rank 0; other ranks exit 0
    at once and print nothing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_launch_count_follows_the_step_path():
    """gpu_launches in the bench line counts the kernels of the path the step
    took: four on the separate path (one more scoring launch per further 64
    tables), three with the fused selection + attention kernel, one for the
    one-kernel step."""
    sys.path.insert(0, ROOT)
    import bench
    import soft_lsh_top_b200 as sk

    assert bench.kernels_per_step(sk.SOCKET_STEP_SEPARATE, 32) == 4
    assert bench.kernels_per_step(sk.SOCKET_STEP_SEPARATE, 64) == 4
    assert bench.kernels_per_step(sk.SOCKET_STEP_SEPARATE, 80) == 5
    assert bench.kernels_per_step(sk.SOCKET_STEP_SEPARATE, 128) == 5
    assert bench.kernels_per_step(sk.SOCKET_STEP_FUSED, 60) == 3
    assert bench.kernels_per_step(sk.SOCKET_STEP_ONE_KERNEL, 16) == 1


def test_step_kernel_times_are_named_by_path():
    """The bench names the intervals between a step's events after the kernels
    its path launched (the library records events 1..4 right after the last
    kernel when a path has fewer than four)."""
    sys.path.insert(0, ROOT)
    import bench
    import soft_lsh_top_b200 as sk

    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    stamps = [0.0, 1.0, 3.0, 6.0, 10.0]  # intervals 1, 2, 3, 4 ms
    evs = [[Ev(t) for t in stamps] for _ in range(3)]
    assert bench.step_kernel_times(evs, 3, sk.SOCKET_STEP_SEPARATE) == {
        "soft_tables": 1.0, "score": 2.0, "topk": 3.0, "attention": 4.0}
    assert bench.step_kernel_times(evs, 3, sk.SOCKET_STEP_FUSED) == {
        "soft_tables": 1.0, "score": 2.0, "select_attend": 3.0}
    assert bench.step_kernel_times(evs, 3, sk.SOCKET_STEP_ONE_KERNEL) == {"small_step": 1.0}
