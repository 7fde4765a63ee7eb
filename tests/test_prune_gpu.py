"""Score-bound key pruning (FlashTopK README, "Highlights": adaptive key
pruning decides per call whether to skip keys by a score bound).

* ftk_block_bound (the bound the pruning uses) against the oracle's fp64
  box bound, with +inf for blocks that must never be skipped;
* pruning never changes a result: with pruning auto, forced on and off,
  ftk_select gives the same bits, and they match the oracle;
* the per-call decision: it prunes block-structured keys (most blocks far
  below the threshold) and declines on N(0,1) keys, where the bound is loose.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from sparse_attention_indexer_ftk_b200 import ftk
from sparse_attention_indexer_ftk_b200 import workloads as wl
from tests.parity import to_np
from tests.test_select_gpu import check_case, run_select

pytestmark = pytest.mark.gpu

STATUS_NAN, STATUS_BAD_SCALE = 0x2, 0x8


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_block_bound_matches_oracle(dtype):
    c = wl.small_case(seed=51, dtype=dtype, T=37, S=1000, topk=8, windows="causal")
    g = c.to("cuda")
    ub = to_np(ftk.block_bound(g.q, g.kv, g.weights, g.kv_scales)).astype(np.float64)
    oub, scale = orc.block_bound(c.q, c.kv, c.kv_scales, c.weights, block=128)
    assert ub.shape == oub.shape == (37, 8)
    err = np.abs(ub - oub) / scale
    assert err.max() <= 1e-5, err.max()


def test_block_bound_unskippable_blocks_are_inf():
    c = wl.small_case(seed=52, dtype="fp8", T=16, S=640, topk=8, windows="causal")
    kv, sc = c.kv.clone(), c.kv_scales.clone()
    kv.view(torch.uint8)[130, 5] = 0x7F   # NaN key in block 1
    sc[300] = 0.0                         # sigma <= 0 in block 2
    sc[520] = float("inf")                # sigma not finite in block 4
    g = wl.SelectInputs(c.name, c.q, kv, sc, c.weights, c.ks, c.ke, c.topk).to("cuda")
    ub = to_np(ftk.block_bound(g.q, g.kv, g.weights, g.kv_scales))
    assert np.all(np.isposinf(ub[:, [1, 2, 4]]))
    assert np.all(np.isfinite(ub[:, [0, 3]]))


def _same(a, b):
    return np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.int32), b[1].view(np.int32))


@pytest.mark.parametrize("dtype,T,S,topk", [("fp8", 150, 9000, 128), ("bf16", 133, 5000, 64)])
def test_pruning_fires_on_block_structured_keys(dtype, T, S, topk):
    c = wl.block_structured(seed=53, dtype=dtype, T=T, S=S, topk=topk)
    idx, val, info, worst, overlaps = check_case(c)
    assert info["prune_enabled"] == 1, info
    assert info["blocks_pruned"] >= info["blocks_total"] // 2, info
    g = c.to("cuda")
    off = run_select(g, {"prune": -1})
    on = run_select(g, {"prune": 1})
    assert off[2]["prune_enabled"] == 0 and off[2]["blocks_pruned"] == 0
    assert on[2]["blocks_pruned"] == info["blocks_pruned"]
    assert _same((idx, val), off) and _same((idx, val), on)


def _expected_blocks_total(c, rt):
    ks, ke = to_np(c.ks).astype(np.int64), to_np(c.ke).astype(np.int64)
    total = 0
    for t0 in range(0, c.T, rt):
        rows = [t for t in range(t0, min(t0 + rt, c.T)) if 0 <= ks[t] < ke[t] <= c.S]
        if rows:
            lo = min(ks[t] for t in rows) // 128 * 128
            hi = max(ke[t] for t in rows)
            total += (hi - lo + 127) // 128
    return total


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_pruning_declines_on_normal_keys(dtype):
    c = wl.small_case(seed=54, dtype=dtype, T=140, S=6000, topk=100, windows="causal")
    idx, val, info, worst, overlaps = check_case(c)
    assert info["prune_enabled"] == 0 and info["blocks_pruned"] == 0, info
    assert info["blocks_total"] == _expected_blocks_total(c, 16 if dtype == "fp8" else 8)
    g = c.to("cuda")
    on = run_select(g, {"prune": 1})
    assert on[2]["prune_enabled"] == 1
    assert _same((idx, val), on)


def test_pruning_keeps_nan_and_bad_scale_visible():
    c = wl.block_structured(seed=55, dtype="fp8", T=33, S=4000, topk=64)
    kv, sc = c.kv.clone(), c.kv_scales.clone()
    kv.view(torch.uint8)[128 * 3 + 7, 11] = 0x7F   # NaN in a cold block
    sc[128 * 5 + 2] = 0.0                          # sigma 0 in another cold block
    g = wl.SelectInputs(c.name, c.q, kv, sc, c.weights, c.ks, c.ke, c.topk).to("cuda")
    for prune in (0, 1, -1):  # auto, always, off
        _, _, info = run_select(g, {"prune": prune})
        assert info["status"] & STATUS_NAN and info["status"] & STATUS_BAD_SCALE, (prune, info)
