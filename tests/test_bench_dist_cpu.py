"""bench.py's multi-rank set-up and teardown, on the CPU (gloo, 2 ranks).

bench.py runs every rank inside shard.ProcessGroup, which creates the
default process group on entry and destroys it exactly once on exit, so a
multi-GPU bench exits 0 on every rank after rank 0 prints its line.  The
test drives that context with the collectives bench.py takes (barriers,
max-over-ranks, the sharded gather) and checks a clean exit code on both
ranks, also when the body raises on one rank after the collectives.
"""
from __future__ import annotations

import ast
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import os, sys
sys.path.insert(0, {root!r})
import torch
from sparse_attention_indexer_ftk_b200 import shard
world, rank = int(os.environ["WORLD_SIZE"]), int(os.environ["RANK"])
raise_after = os.environ.get("RAISE_AFTER") == str(rank)
try:
    with shard.ProcessGroup(world, rank, "gloo", timeout_s=30) as pg:
        pg.barrier()
        m = shard.max_over_ranks(1.0 + rank)
        assert m == float(world), m
        T = 7
        lo, hi = shard.row_shard(T, world, rank)
        local = torch.arange(lo, hi, dtype=torch.int32).reshape(-1, 1).repeat(1, 3)
        got = shard.gather_rows(local, T)
        if rank == 0:
            assert torch.equal(got[:, 0], torch.arange(T, dtype=torch.int32)), got
        else:
            assert got is None
        pg.barrier()
        if raise_after:
            raise KeyError("planted")
    assert not torch.distributed.is_initialized()
except KeyError:
    assert not torch.distributed.is_initialized()  # destroyed on the way out
    sys.exit(3)
print("rank", rank, "clean")
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(world: int, extra_env: dict) -> list[subprocess.CompletedProcess]:
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, WORLD_SIZE=str(world), RANK=str(r), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), **extra_env)
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_SCRIPT.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    out = []
    for p in procs:
        so, se = p.communicate(timeout=120)
        out.append(subprocess.CompletedProcess(p.args, p.returncode, so, se))
    return out


def test_two_ranks_set_up_and_tear_down_cleanly():
    res = _run_ranks(2, {})
    for r, p in enumerate(res):
        assert p.returncode == 0, (r, p.stderr[-2000:])
        assert f"rank {r} clean" in p.stdout


def test_teardown_runs_once_when_a_rank_raises():
    res = _run_ranks(2, {"RAISE_AFTER": "1"})
    assert res[0].returncode == 0, res[0].stderr[-2000:]
    assert res[1].returncode == 3, res[1].stderr[-2000:]
    assert "Process group cannot be None" not in res[1].stderr


def test_bench_sets_up_and_tears_down_only_through_the_context():
    """bench.py creates and destroys the process group only through
    shard.ProcessGroup (one teardown per run)."""
    src = open(os.path.join(ROOT, "bench.py")).read()
    calls = [n.func.attr for n in ast.walk(ast.parse(src))
             if isinstance(n, ast.Call) and isinstance(n.func, ast.Attribute)]
    assert "destroy_process_group" not in calls
    assert "init_process_group" not in calls
    assert "ProcessGroup" in calls
