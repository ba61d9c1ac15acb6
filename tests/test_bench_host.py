"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks started the
way torchrun starts them (RANK / WORLD_SIZE / MASTER_* in the environment)
set up the process group, meet at the barrier, agree on the max of their
timings, and compute the weak-scaling value from it."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_init(backend="gloo")
    bench.barrier(w)
    t = bench.max_over_ranks(1.5 + rank, w)          # this rank's "seconds"
    v = bench.weak_value(100.0, w, t)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((r, w, local, t, v))


def test_two_gloo_ranks_agree_on_max_time_and_weak_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1]
    for r, w, local, t, v in got:
        assert w == world and local == r
        assert t == pytest.approx(2.5)                 # max over ranks, not the local value
        assert v == pytest.approx(world * 100.0 / 2.5)


def test_single_rank_needs_no_process_group(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_init(backend="gloo") == (1, 0, 0)
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.weak_value(10.0, 1, 2.0) == 5.0
