"""The N > 1 path of bench.py on CPU: two gloo ranks stand in for two GPUs.

Each rank times its own independent problem instance; the job's time is the slowest rank's
(an all-reduce MAX), and the throughput counts the units of all ranks (weak scaling).  The
reference arm runs on rank 0 only.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        units = 16384 * 16 * 3                               # T * B * steps on each rank
        out[rank] = (ms, bench.job_throughput(units, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_whole_job_throughput():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        ms, value = res[rank]
        assert ms == 15.0                                    # the slower rank's time, on every rank
        assert value == pytest.approx(16384 * 16 * 3 * 2 / 0.015)


def test_single_rank_is_local_time():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, None, None) == 12.5
    assert bench.job_throughput(1000, 1, 500.0) == pytest.approx(2000.0)


def _ref_worker(rank, world, port, out):
    import contextlib
    import io
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import pn_inputs as pi

        class Args:
            steps, warmup = 1, 0
        prob = pi.random_problem(3, pi.CELL_TANH_RNN, 4, 4, T=64, B=2)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.reference_arm(Args, prob, pi.MODE_QUASI, rank, world)
        out[rank] = buf.getvalue()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reference_arm_runs_on_rank0_only():
    import json
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_ref_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[1] == ""
    line = json.loads(res[0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
