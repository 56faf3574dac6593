"""The N > 1 path of bench.py on CPU: two gloo ranks run the same host-side
helpers the NCCL run uses (rank barrier, max over ranks, whole-job value),
and the reference arm does its work on rank 0 only."""

import io
import os
import socket
import sys
from contextlib import redirect_stdout
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, local = bench.dist_setup(world)
        # per-rank device times of 4 steps: rank 1 is the slower one
        step_ms = [10.0 + rank] * 4
        total = bench.rank_max(sum(step_ms), w, torch.device("cpu"))
        bench.rank_barrier(w, torch.device("cpu"))
        value = bench.whole_job_value(w, 4608, 4, total)
        q.put((r, w, local, total, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_time_and_count_every_rank():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0]
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [x[0] for x in res] == [0, 1] and all(x[1] == 2 for x in res)
    # both ranks see rank 1's 44 ms; the job moved 2 x 4608 tokens per step
    assert all(x[3] == 44.0 for x in res)
    assert all(x[4] == pytest.approx(2 * 4608 * 4 / 0.044) for x in res)


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.rank_max(3.5, 1, None) == 3.5
    bench.rank_barrier(1, None)
    assert bench.whole_job_value(1, 4608, 10, 5.0) == pytest.approx(4608 * 10 / 0.005)


def test_dist_setup_rejects_a_world_that_does_not_match_gpus(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.dist_setup(4)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from synth import WORKLOADS

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        gpus, steps, warmup = 2, 1, 3

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args, WORKLOADS["t2i_1024"])
    assert buf.getvalue() == ""
