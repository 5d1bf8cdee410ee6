"""The N > 1 path of bench.py on CPU: two ranks over gloo, launched the way
torchrun launches them (RANK / WORLD_SIZE / LOCAL_RANK / MASTER_* in the
environment).  The layer runs as independent replicas, so what the ranks share
is the timing protocol: barriers, the max-over-ranks step time, the job-wide
value, and rank 0 alone running the reference arm."""
import multiprocessing as mp
import os
import socket
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))


def _timing_worker(rank, world, port, out):
    _env(rank, world, port)
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks("gloo", torch.device("cpu"), timeout_s=60)
    # each rank reports its own step time; the job is timed by the slowest
    step_ms = 10.0 * (rank + 1) + 0.5
    r.barrier()
    slowest = r.max_over_ranks(step_ms)
    out.put((rank, r.world, slowest, bench.job_value(slowest, r.world)))
    r.close()


def _reference_worker(rank, world, port, out):
    _env(rank, world, port)
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse_args(["--impl", "reference", "--gpus", str(world), "--steps", "1",
                             "--warmup", "0", "--workload", "vs_n2k_h1_d64"])
    rc = bench.run_reference(args) if rank != 0 else 0  # rank 0's oracle run is not under test
    out.put((rank, rc))


def _run(target, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_two_ranks_time_the_job_by_the_slowest_rank():
    res = _run(_timing_worker)
    assert [r[0] for r in res] == [0, 1]
    for rank, world, slowest, value in res:
        assert world == 2
        assert slowest == pytest.approx(20.5)          # max over ranks, on every rank
        assert value == pytest.approx(20.5 / 2)        # two layers per 20.5 ms step


def test_reference_arm_runs_on_rank_zero_only():
    res = _run(_reference_worker)
    assert res == [(0, 0), (1, 0)]                    # rank 1 exits 0 without work


def test_single_process_needs_no_process_group():
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks("gloo", torch.device("cpu"))
    assert r.world == 1 and r.rank == 0 and r.dist is None
    assert r.max_over_ranks(3.25) == 3.25
    r.barrier()
    r.close()
