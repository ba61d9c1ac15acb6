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


RANK_SCRIPT = """
import os, sys
sys.path.insert(0, {root!r})
import bench
w, r, local = bench.dist_init(backend="gloo")
bench.check_world(int(sys.argv[1]), w)
t = bench.max_over_ranks(1.0 + r, w)
if r == 0:
    print("RESULT", w, t, bench.weak_value(10.0, w, t), flush=True)
bench.barrier(w)
import torch.distributed as dist
dist.destroy_process_group()
"""


def test_relaunch_command_starts_one_rank_per_gpu(tmp_path):
    """bench.py --gpus N started without a launcher re-executes itself through
    torch.distributed.run; the command it builds starts N ranks that find each
    other on 127.0.0.1 and agree on the slowest rank's time."""
    import subprocess
    import sys
    import bench
    root = os.path.dirname(os.path.abspath(bench.__file__))
    script = tmp_path / "ranks.py"
    script.write_text(RANK_SCRIPT.format(root=root))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    cmd = bench.relaunch_cmd(str(script), ["2"], 2, _free_port())
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=2" in cmd
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=180, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    line = [l for l in res.stdout.splitlines() if l.startswith("RESULT")][0].split()
    assert int(line[1]) == 2 and float(line[2]) == 2.0 and float(line[3]) == 10.0


def test_gpus_must_match_world_size():
    import bench
    bench.check_world(1, 1)
    with pytest.raises(SystemExit):
        bench.check_world(8, 1)
