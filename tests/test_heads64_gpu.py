"""Indexers of 64 heads (FlashTopK README, "Roadmap": other head counts such
as 64): ftk_select and ftk_score_dense with q [T, 64, 128], weights [T, 64]
against the oracle (which takes the head count from q's shape), with the
same bar as the 32-head cases: fused scores within 1e-4 * E, the selection
bit-exact against the oracle's selection of the GPU's own dumped scores,
index sets equal to the fp64 oracle's up to swaps inside the tie band."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from sparse_attention_indexer_ftk_b200 import ftk
from sparse_attention_indexer_ftk_b200 import workloads as wl
from tests.parity import to_np
from tests.test_select_gpu import check_case, gpu_inputs, run_select

pytestmark = pytest.mark.gpu

CASES = [
    dict(seed=31, dtype="fp8", T=37, S=3000, topk=64, windows="causal"),
    dict(seed=32, dtype="bf16", T=21, S=1500, topk=100, windows="random"),
    dict(seed=33, dtype="fp8", T=16, S=777, topk=300, windows="short"),
    dict(seed=34, dtype="fp8", T=41, S=2600, topk=128, windows="empty_mix"),
    dict(seed=35, dtype="bf16", T=24, S=2100, topk=200, windows="packed"),
    dict(seed=36, dtype="fp8", T=5, S=60000, topk=2048, windows="causal"),  # few rows, long windows
    dict(seed=38, dtype="fp8", T=9, S=5000, topk=16, windows="causal", kv_levels=4),
]


@pytest.mark.parametrize("spec", CASES, ids=[f"{s['dtype']}-{s['windows']}-{s['seed']}" for s in CASES])
def test_small_cases_64_heads(spec):
    c = wl.small_case(heads=64, **spec)
    assert c.q.shape[1] == 64 and c.weights.shape[1] == 64
    _, _, info, worst, overlaps = check_case(c)
    assert worst < 1e-4


@pytest.mark.parametrize("config", [dict(dense_rows=-1, capacity=64), dict(dense_rows=-1, oversample=0.05),
                                    dict(dense_rows=-1, recovery_rows=8, capacity=64), dict(dense_rows=-1, prune=1)])
def test_config_does_not_change_the_result_64_heads(config):
    c = wl.small_case(seed=37, dtype="fp8", T=29, S=9000, topk=64, windows="random", heads=64)
    g = gpu_inputs(c)
    ref_idx, ref_val, _ = run_select(g)
    idx, val, info = run_select(g, config)
    assert np.array_equal(ref_idx, idx)
    assert np.array_equal(ref_val.view(np.uint32), val.view(np.uint32))
    if "capacity" in config:
        assert info["rows_overflow"] > 0
    if "oversample" in config:
        assert info["rows_underflow"] > 0
    check_case(c, config=config)


def test_64_head_score_is_the_sum_of_its_halves():
    """Scoring q [T, 64, 128] equals, within the rounding of two float32
    sums, scoring its two 32-head halves and adding (each half its own
    32-head call)."""
    c = wl.small_case(seed=39, dtype="bf16", T=12, S=700, topk=32, windows="causal", heads=64)
    g = gpu_inputs(c)
    full = to_np(ftk.score_dense(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales))
    halves = [to_np(ftk.score_dense(g.q[:, h:h + 32].contiguous(), g.kv, g.weights[:, h:h + 32].contiguous(),
                                    g.ks, g.ke, g.kv_scales)) for h in (0, 32)]
    _, E = orc.index_scores(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke)
    for t in range(c.T):
        L = int(c.ke[t] - c.ks[t])
        d = np.abs(full[t, :L].astype(np.float64) - (halves[0][t, :L].astype(np.float64) +
                                                      halves[1][t, :L].astype(np.float64)))
        assert np.all(d <= 1e-5 * E[t, :L]), t


def test_selector_64_heads_and_determinism():
    c = wl.small_case(seed=40, dtype="fp8", T=48, S=20000, topk=512, windows="causal", heads=64)
    g = gpu_inputs(c)
    sel = ftk.Selector(topk=512, dtype=torch.float8_e4m3fn, heads=64).plan(64, 20000)
    a = to_np(sel.run(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales))
    b = to_np(sel.run(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales))
    assert np.array_equal(a, b) and sel.last_info["status"] == 0
    ref, _, _ = run_select(g)
    assert np.array_equal(a, ref)
    with pytest.raises(ftk.FtkError):  # a 32-head Selector refuses 64-head inputs
        ftk.Selector(topk=512).plan(64, 20000).run(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales)


def test_full_size_64_heads():
    """fp8_prefill_64h (4096 queries x 128K FP8 keys, 64 heads, topk 2048):
    every row against the invariants, 64 seeded rows bit-exact against the
    oracle's selection of the GPU's dumped scores, 8 of them against the
    fp64 oracle."""
    c = wl.get("fp8_prefill_64h")
    rows = wl.sample_rows(c.T, 64, seed=2)
    fp64_rows = rows[:: len(rows) // 8][:8] + [rows[-1]]
    _, _, info, worst, overlaps = check_case(c, rows=rows, fp64_rows=fp64_rows)
    assert worst < 1e-4 and min(overlaps) >= 0.99


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_block_bound_64_heads_matches_oracle(dtype):
    """The 64-head score bound (both halves of every row) against the
    oracle's fp64 box bound over all 64 heads."""
    c = wl.small_case(seed=41, dtype=dtype, T=21, S=1000, topk=8, windows="causal", heads=64)
    g = c.to("cuda")
    ub = to_np(ftk.block_bound(g.q, g.kv, g.weights, g.kv_scales)).astype(np.float64)
    oub, scale = orc.block_bound(c.q, c.kv, c.kv_scales, c.weights, block=128)
    assert ub.shape == oub.shape == (21, 8)
    assert (np.abs(ub - oub) / scale).max() <= 1e-5


@pytest.mark.parametrize("dtype,T,S,topk", [("fp8", 150, 9000, 128), ("bf16", 133, 5000, 64)])
def test_pruning_64_heads_fires_and_changes_nothing(dtype, T, S, topk):
    c = wl.block_structured(seed=42, dtype=dtype, T=T, S=S, topk=topk, heads=64)
    idx, val, info, worst, overlaps = check_case(c)
    assert info["prune_enabled"] == 1, info
    assert info["blocks_pruned"] >= info["blocks_total"] // 2, info
    g = c.to("cuda")
    off = run_select(g, {"prune": -1})
    on = run_select(g, {"prune": 1})
    assert off[2]["prune_enabled"] == 0 and on[2]["blocks_pruned"] == info["blocks_pruned"]
    for r in (off, on):
        assert np.array_equal(idx, r[0]) and np.array_equal(val.view(np.int32), r[1].view(np.int32))
