"""Multi-GPU plumbing for ftk_select: one process per GPU, rows sharded.

Each query row's selection depends only on its own window, weights and
threshold (the threshold comes from a strided sample of the row's own window:
FlashTopK README, "Highlights", context-parallel compatible), so rows shard
across GPUs with no collective on the data path.  What needs the process
group is the measurement (the step time is the max over ranks) and, if a
caller wants every row's result on one rank, a gather after the fact.
"""
from __future__ import annotations

import datetime

import torch
import torch.distributed as dist


class ProcessGroup:
    """One process per GPU: the default process group for `world` ranks,
    set up on entry and destroyed exactly once on exit (also when the body
    raises).  With world == 1 nothing is set up.  backend "nccl" makes
    cuda:local_rank current first; "gloo" runs on the CPU.  The timeout is
    short so that ranks waiting for a rank that died end with an error."""

    def __init__(self, world: int, local_rank: int = 0, backend: str = "nccl", timeout_s: float = 120.0):
        self.world, self.local, self.backend, self.timeout_s = world, local_rank, backend, timeout_s
        self.active = False

    def __enter__(self) -> "ProcessGroup":
        if self.world > 1:
            kw = {}
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=self.timeout_s), **kw)
            self.active = True
        return self

    def barrier(self) -> None:
        if self.active:
            dist.barrier()

    def __exit__(self, *exc) -> bool:
        if self.active and dist.is_initialized():
            dist.destroy_process_group()
        self.active = False
        return False


def row_shard(T: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous block [lo, hi) of the T query rows owned by `rank`; the
    blocks of ranks 0 .. world-1 tile [0, T) in order, sizes differing by at
    most one row."""
    if world < 1 or not 0 <= rank < world or T < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, T >= 0")
    base, extra = divmod(T, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(x: float, device: torch.device | str = "cpu") -> float:
    """The maximum of x over all ranks of the default process group (x
    itself without one).  device: where the reduction tensor lives (a CUDA
    device for NCCL, the CPU for gloo)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_rows(local: torch.Tensor, T: int, device: torch.device | str = "cpu") -> torch.Tensor | None:
    """Every rank passes its row block (as row_shard assigns it) of a
    [rows, ...] result; rank 0 receives the [T, ...] concatenation, the
    other ranks None.  Blocks are padded to the largest block for the
    collective and trimmed after."""
    world, rank = dist.get_world_size(), dist.get_rank()
    n_max = row_shard(T, world, 0)[1]  # rank 0 holds the largest block
    pad = torch.zeros((n_max,) + tuple(local.shape[1:]), dtype=local.dtype, device=device)
    pad[: local.shape[0]] = local.to(device)
    parts = [torch.empty_like(pad) for _ in range(world)] if rank == 0 else None
    dist.gather(pad, parts, dst=0)
    if rank != 0:
        return None
    out = []
    for r in range(world):
        lo, hi = row_shard(T, world, r)
        out.append(parts[r][: hi - lo])
    return torch.cat(out, dim=0)
