"""Row sharding across processes (world size 2, gloo on the CPU).

Each rank selects its block of rows with the oracle; the blocks gathered on
rank 0 equal the selection of all rows in one process, so the data path
needs no collective.  The measurement's max-over-ranks reduction is checked
with different per-rank values.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle as orc
from sparse_attention_indexer_ftk_b200 import shard
from sparse_attention_indexer_ftk_b200 import workloads as wl


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    return wl.small_case(seed=61, dtype="fp8", T=23, S=900, topk=40, windows="random")


def _rank_main(rank: int, world: int, port: int, out_path: str):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = _case()
        lo, hi = shard.row_shard(c.T, world, rank)
        rows = np.arange(lo, hi)
        idx, val, flags = orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk, rows=rows)
        got_idx = shard.gather_rows(torch.from_numpy(idx), c.T)
        got_val = shard.gather_rows(torch.from_numpy(val), c.T)
        mx = shard.max_over_ranks(10.0 + rank)
        if rank == 0:
            torch.save({"idx": got_idx, "val": got_val, "max": mx}, out_path)
        else:
            assert got_idx is None and got_val is None
            assert mx == 10.0 + world - 1
    finally:
        dist.destroy_process_group()


def test_row_shard_tiles_the_rows():
    for T in (0, 1, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            blocks = [shard.row_shard(T, world, r) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == T
            assert all(blocks[r][1] == blocks[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in blocks]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.row_shard(5, 2, 2)


def test_max_over_ranks_without_a_group():
    assert shard.max_over_ranks(3.5) == 3.5


def test_two_ranks_gather_equals_single_process(tmp_path):
    world = 2
    out = str(tmp_path / "rank0.pt")
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    res = torch.load(out)
    c = _case()
    idx, val, flags = orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk)
    assert np.array_equal(res["idx"].numpy(), idx)
    assert np.array_equal(res["val"].numpy(), val)
    assert res["max"] == 10.0 + world - 1
