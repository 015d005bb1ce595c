"""The N > 1 path of bench.py on CPU: two gloo ranks run as replicas and the
timing of the job is the max over ranks (no GPU needed)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (10 + r, 2 + 3r) ms: every rank must see (10 + world - 1, 2 + 3(world - 1))
        red = bench.max_over_ranks([10.0 + rank, 2.0 + 3 * rank], world, "cpu")
        out[rank] = red
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_gloo(world):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        assert out[r] == [10.0 + world - 1, 2.0 + 3 * (world - 1)]


def test_single_rank_and_job_throughput():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    # 50 MB per rank in 10 us on each of 4 ranks: 20 TB/s for the job
    assert bench.job_throughput(50e6, 0.01, 4) == pytest.approx(20000.0)
    assert bench.job_throughput(50e6, 0.01, 1) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        cpu_rows = 16
        warmup = 0
        steps = 1

    assert bench.run_reference(Args()) is None
