"""The N > 1 launch path of bench.py on CPU: two gloo ranks.

The hot path has no data-path collective (every rank runs an independent
replica), so what N > 1 adds is host logic: the process-group set-up, the
barrier, the max-over-ranks time, and the reference arm's rule that only
rank 0 works.  These run here as two spawned processes on 127.0.0.1.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench

    r, local, w, pg = bench.dist_setup(world)
    assert (r, local, w) == (rank, rank, world)
    assert pg is not None
    bench.barrier(pg)
    # each rank reports its own time; every rank must see the largest
    t = bench.max_over_ranks(pg, 1.0 + 2.5 * rank)
    bench.barrier(pg)
    pg.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(t))


def test_two_gloo_ranks_agree_on_the_max_time(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [float((tmp_path / f"rank{r}.txt").read_text()) for r in range(world)]
    assert got == [3.5, 3.5]


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench

    rank, local, world, pg = bench.dist_setup(1)
    assert (rank, local, world, pg) == (0, 0, 1, None)
    assert bench.max_over_ranks(None, 7.25) == 7.25
    bench.barrier(None)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    # a non-zero rank returns before any work or output (the args are not even read)
    assert bench.bench_reference(None) is None
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("world", [2])
def test_ranks_fail_together_when_one_never_joins(world, tmp_path):
    """A rank that never joins ends the others' set-up with an error, not a hang."""
    port = _free_port()
    code = (
        "import os, sys, datetime, torch.distributed as dist\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "os.environ.update({'WORLD_SIZE': '2', 'RANK': '0', 'LOCAL_RANK': '0', "
        f"'MASTER_ADDR': '127.0.0.1', 'MASTER_PORT': '{port}'}})\n"
        "try:\n"
        "    dist.init_process_group('gloo', timeout=datetime.timedelta(seconds=3))\n"
        "    print('joined')\n"
        "except Exception as e:\n"
        "    print('error', type(e).__name__)\n"
    )
    import subprocess

    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert "error" in p.stdout and "joined" not in p.stdout
