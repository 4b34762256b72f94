"""The replica plumbing bench.py uses for N > 1, run as 2 gloo ranks on the CPU: every
rank takes the same collective steps, the timing is the max over ranks, and the job
throughput counts every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from global_interleaved_layers_b200.replicas import Replicas
    r = Replicas(backend="gloo", timeout_s=30)
    try:
        r.barrier()
        seconds = 1.0 + rank  # rank 1 is the slow one
        slowest = r.max_over_ranks(seconds)
        value = r.aggregate_throughput(work_per_rank=6.0, seconds_per_rank=seconds)
        r.barrier()
        q.put((rank, r.world, slowest, value))
    finally:
        r.close()


def test_two_rank_replicas_max_and_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, w, slowest, value in got:
        assert w == 2
        assert slowest == pytest.approx(2.0)  # max over ranks, seen by every rank
        assert value == pytest.approx(2 * 6.0 / 2.0)


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    from global_interleaved_layers_b200.replicas import Replicas
    r = Replicas(backend="gloo")
    assert r.world == 1 and r.rank == 0
    r.barrier()
    assert r.max_over_ranks(3.5) == 3.5
    assert r.aggregate_throughput(10.0, 2.0) == pytest.approx(5.0)
