"""Host-side logic that needs no GPU: the bench's reading of the committed
ncu summary, and the seeded workload generators."""
from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_attention_indexer_ftk_b200 import workloads as wl  # noqa: E402


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    good = tmp_path / "ok.md"
    good.write_text(f"traffic_bytes_per_launch: 1234\nkernel_source_hash: {bench.scan_kernel_hash()}\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(good))
    assert bench.profiled_traffic() == 1234.0
    stale = tmp_path / "stale.md"
    stale.write_text("traffic_bytes_per_launch: 1234\nkernel_source_hash: 000000000000\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(stale))
    assert bench.profiled_traffic() is None  # counters of another kernel source are not reported
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "missing.md"))
    assert bench.profiled_traffic() is None


def test_generators_are_seeded_and_shaped():
    a = wl.small_case(seed=3, dtype="fp8", T=9, S=500, topk=16, windows="random")
    b = wl.small_case(seed=3, dtype="fp8", T=9, S=500, topk=16, windows="random")
    assert torch.equal(a.q.view(torch.uint8), b.q.view(torch.uint8))
    assert torch.equal(a.ks, b.ks) and torch.equal(a.ke, b.ke)
    assert a.q.shape == (9, 32, 128) and a.kv.shape == (500, 128) and a.weights.shape == (9, 32)
    assert bool(torch.all((a.ks >= 0) & (a.ks <= a.ke) & (a.ke <= 500)))


def test_block_structured_keys():
    c = wl.block_structured(seed=5, dtype="bf16", T=4, S=1000, topk=8)
    base = wl.small_case(seed=5, dtype="bf16", T=4, S=1000, topk=8, windows="causal")
    blk = torch.arange(1000) // 128
    hot = blk % 8 == 0
    assert torch.equal(c.kv_scales[hot], base.kv_scales[hot])
    assert torch.allclose(c.kv_scales[~hot], base.kv_scales[~hot] * 2.0 ** -7)
    assert bool(torch.all(c.weights[:, 1:8] >= 0)) and bool(torch.all(c.weights[:, ::8] <= 0))
