"""Multi-rank logic of the benchmark on CPU (gloo, world size 2): timings are
reduced by max over ranks, the whole-job throughput counts every rank's
weights, and the CPU reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 is the slow one on the step time, rank 0 on the backward
        mx = bench.reduce_max([10.0 + 5.0 * rank, 3.0 - rank], "cpu", world)
        value = bench.step_throughput(1_000_000_000, world, mx[0] / 2)
        out.put((rank, mx, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_max_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, value in res:
        assert mx == [15.0, 3.0]          # both ranks see the max
        # 2 ranks x 1e9 weights in 7.5 ms per step
        assert value == pytest.approx(2e9 / 7.5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max([1.0, 2.0], "cpu", 1) == [1.0, 2.0]
    assert bench.step_throughput(6_979_321_856, 1, 18.78) == pytest.approx(371.64, rel=1e-3)


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "sample_rows_for_oracle", lambda *a: called.append(a))

    class A:
        steps, warmup, gpus, cpu_seconds = 2, 1, 2, 1.0
    assert bench.run_reference(A()) == 0
    assert not called  # no work on ranks other than 0
