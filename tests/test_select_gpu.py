"""ftk_select / ftk_score_dense against the oracle.

For every case:
* the fused scores (ftk_score_dense, the same kernel and bits ftk_select
  uses) are within 1e-4 * E of the oracle's fp64 scores;
* ftk_select equals, bit for bit, the oracle's exact selection of the GPU's
  own dumped scores (index set and values);
* ftk_select's sets equal the fp64 oracle's up to swaps inside the tie band,
  and every row satisfies the invariants.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from sparse_attention_indexer_ftk_b200 import ftk
from sparse_attention_indexer_ftk_b200 import workloads as wl
from tests.parity import (check_against_fp64, check_exact_vs_dump, check_row_invariants,
                          check_scores_close, to_np)

pytestmark = pytest.mark.gpu


def gpu_inputs(c: wl.SelectInputs):
    return c.to("cuda")


def run_select(g: wl.SelectInputs, config=None):
    ws = torch.empty(ftk.select_workspace_size(g.T, g.S, g.topk, config, g.q.shape[1]), dtype=torch.uint8,
                     device="cuda")
    idx, val = ftk.select(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales, g.topk,
                          return_scores=True, workspace=ws, config=config)
    info = ftk.read_info(ws)
    return to_np(idx), to_np(val), info


def check_case(c: wl.SelectInputs, rows=None, fp64_rows=None, config=None, expect_status=0):
    g = gpu_inputs(c)
    idx, val, info = run_select(g, config)
    assert info["status"] == expect_status, info
    T = c.T
    ks, ke = to_np(c.ks).astype(np.int64), to_np(c.ke).astype(np.int64)
    rows = list(range(T)) if rows is None else rows
    fp64_rows = rows if fp64_rows is None else fp64_rows
    # invariants on every row
    for t in range(T):
        if 0 <= ks[t] <= ke[t] <= c.S:
            check_row_invariants(idx[t], int(ks[t]), int(ke[t]), c.topk)
        else:
            assert np.all(idx[t] == -1)
    # bit-exact against the oracle's selection of the GPU's own scores
    dump = ftk.score_dense(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales,
                           rows=torch.tensor(rows, dtype=torch.int32))
    dump = to_np(dump)
    oidx, oval, nflag = orc.select_f32_rows(dump, c.ks, c.ke, c.S, c.topk, row_ids=rows)
    for r, t in enumerate(rows):
        check_exact_vs_dump(idx[t], val[t], oidx[r], oval[r], c.topk)
    # fp64 oracle: scores within tolerance, sets up to band swaps
    I64, E = orc.index_scores(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, rows=fp64_rows)
    worst = 0.0
    overlaps = []
    row_pos = {t: r for r, t in enumerate(rows)}
    for r, t in enumerate(fp64_rows):
        L = int(ke[t] - ks[t])
        if L <= 0:
            continue
        worst = max(worst, check_scores_close(dump[row_pos[t], :L], I64[r, :L], E[r, :L], f"row {t}"))
        overlaps.append(check_against_fp64(idx[t], val[t], I64[r, :L], E[r, :L], int(ks[t]), c.topk))
    return idx, val, info, worst, overlaps


SMALL = [
    dict(seed=1, dtype="fp8", T=37, S=3000, topk=64, windows="causal"),
    dict(seed=2, dtype="bf16", T=20, S=1500, topk=100, windows="random"),
    dict(seed=3, dtype="fp8", T=16, S=777, topk=300, windows="short"),
    dict(seed=4, dtype="fp8", T=41, S=2600, topk=128, windows="empty_mix"),
    dict(seed=5, dtype="bf16", T=24, S=2100, topk=200, windows="packed"),
    dict(seed=6, dtype="fp8", T=9, S=5000, topk=16, windows="causal", kv_levels=4),
    dict(seed=7, dtype="fp8", T=8, S=40000, topk=2048, windows="causal"),
    dict(seed=8, dtype="bf16", T=3, S=129, topk=1, windows="causal", scales=False),
    dict(seed=9, dtype="fp8", T=12, S=20000, topk=4096, windows="random"),
    # decode-shaped: a few query rows over long windows (split into many
    # sample and scan work items, candidates merged across items)
    dict(seed=11, dtype="fp8", T=3, S=100000, topk=2048, windows="causal"),
    dict(seed=12, dtype="bf16", T=5, S=40000, topk=512, windows="random"),
    # edge sizes: one query, one key; topk above every window; one query over a long window
    dict(seed=21, dtype="fp8", T=1, S=1, topk=1, windows="causal"),
    dict(seed=22, dtype="bf16", T=2, S=300, topk=4096, windows="random"),
    dict(seed=23, dtype="fp8", T=1, S=70000, topk=4096, windows="causal"),
]


@pytest.mark.parametrize("spec", SMALL, ids=[f"{s['dtype']}-{s['windows']}-{s['seed']}" for s in SMALL])
def test_small_cases(spec):
    c = wl.small_case(**spec)
    check_case(c)


def test_bf16_small_workload_all_rows():
    c = wl.bf16_small()
    _, _, info, worst, overlaps = check_case(c)
    assert worst < 1e-4
    assert min(overlaps) >= 0.99


def test_bf16_ties_workload():
    """The tie workload straddles: on some rows the k-th score is shared by
    more window keys than there are slots left for it (oracle, fp64), and
    the GPU takes the smallest key indices of that group (FlashTopK README,
    "Highlights": ties keep the smallest key indices)."""
    c = wl.bf16_ties()
    idx, val, _, _, _ = check_case(c)
    I64, _ = orc.index_scores(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke)
    g = gpu_inputs(c)
    dump = to_np(ftk.score_dense(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales))
    straddles = 0
    for t in range(c.T):
        ks, ke = int(c.ks[t]), int(c.ke[t])
        L = ke - ks
        n = min(L, c.topk)
        if n == 0:
            continue
        # oracle: the group of the k-th score against its selected share
        order = sorted(range(L), key=lambda j: (-I64[t, j], j))
        kth = I64[t, order[n - 1]]
        group = [j for j in range(L) if I64[t, j] == kth]
        taken = [j for j in order[:n] if I64[t, j] == kth]
        assert taken == group[:len(taken)]
        if len(group) > len(taken):
            straddles += 1
        # GPU: the selected members of its k-th score's group are the
        # smallest indices of that group (scores as the GPU computed them)
        sel = idx[t, :n].astype(np.int64) - ks
        gv = dump[t, :L]
        gk = gv[sel].min()
        ggroup = np.flatnonzero(gv == gk)
        gsel = np.sort(sel[gv[sel] == gk])
        assert np.array_equal(gsel, ggroup[:gsel.size]), f"row {t}"
        if len(group) > len(taken):
            assert ggroup.size > gsel.size, f"row {t}: the GPU sees no straddling group"
    assert straddles >= 1


def test_all_equal_workload_closed_form():
    c = wl.bf16_all_equal()
    idx, _, _, _, _ = check_case(c)
    for t in range(c.T):
        ks = int(c.ks[t])
        assert idx[t].tolist() == list(range(ks, ks + c.topk))


@pytest.mark.parametrize("config", [
    dict(dense_rows=-1),               # the sampled-threshold path (29 rows would go dense)
    dict(dense_rows=-1, capacity=64),  # every long row overflows -> dense recovery
    dict(dense_rows=-1, oversample=0.05),  # thresholds too high -> underflow -> recovery
    dict(dense_rows=-1, sample_keys=64),   # coarse samples
    dict(dense_rows=-1, recovery_rows=8, capacity=64),  # many recovery passes
    dict(dense_rows=-1, prune=-1),
    dict(dense_rows=-1, prune=1),
])
def test_config_does_not_change_the_result(config):
    """The reference run takes the default (dense) path for these 29 rows;
    every config forces the sampled-threshold path: identical bits."""
    c = wl.small_case(seed=11, dtype="fp8", T=29, S=9000, topk=64, windows="random")
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


@pytest.mark.parametrize("dtype,T,S,topk", [("fp8", 64, 40000, 512), ("bf16", 100, 20000, 256),
                                           ("fp8", 7, 60000, 2048)])
def test_dense_path_matches_threshold_path(dtype, T, S, topk):
    """Calls of few query rows score every key and select with the row
    top-k (three launches); forcing the sampled-threshold path gives the
    same bits, and both match the oracle."""
    c = wl.small_case(seed=T + S, dtype=dtype, T=T, S=S, topk=topk, windows="causal")
    g = gpu_inputs(c)
    d_idx, d_val, d_info = run_select(g)
    t_idx, t_val, t_info = run_select(g, dict(dense_rows=-1))
    assert d_info["kernel_launches"] == 3 and t_info["kernel_launches"] > 3
    assert np.array_equal(d_idx, t_idx)
    assert np.array_equal(d_val.view(np.uint32), t_val.view(np.uint32))
    lens = (c.ke - c.ks).numpy().astype(np.int64)
    assert d_info["candidates_total"] == int(lens.sum()) and d_info["candidates_max"] == int(lens.max())
    check_case(c)


def test_programmatic_launch_off_gives_the_same_bits(tmp_path):
    """Launching without programmatic dependent launch (FTK_NO_PDL=1, read
    once per process, so in a child process) gives the same bits as the
    default launches, on the sampled-threshold path (11 launches)."""
    import os
    import subprocess
    import sys
    spec = dict(seed=41, dtype="fp8", T=200, S=20000, topk=256, windows="causal")
    g = gpu_inputs(wl.small_case(**spec))
    idx, val, _ = run_select(g)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys, numpy as np\n"
        f"sys.path.insert(0, {root!r})\n"
        "from sparse_attention_indexer_ftk_b200 import ftk, workloads as wl\n"
        f"c = wl.small_case(**{spec!r}).to('cuda')\n"
        "i, v = ftk.select(c.q, c.kv, c.weights, c.ks, c.ke, c.kv_scales, c.topk, return_scores=True)\n"
        f"np.save({str(tmp_path / 'i.npy')!r}, i.cpu().numpy())\n"
        f"np.save({str(tmp_path / 'v.npy')!r}, v.cpu().numpy())\n")
    subprocess.run([sys.executable, "-c", code], env=dict(os.environ, FTK_NO_PDL="1"), check=True, timeout=900)
    assert np.array_equal(np.load(tmp_path / "i.npy"), idx)
    assert np.array_equal(np.load(tmp_path / "v.npy").view(np.uint32), val.view(np.uint32))


def test_determinism():
    c = wl.small_case(seed=12, dtype="fp8", T=64, S=30000, topk=512, windows="causal")
    g = gpu_inputs(c)
    a = run_select(g)
    b = run_select(g)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))


def test_bad_windows_flagged_and_padded():
    c = wl.small_case(seed=13, dtype="bf16", T=10, S=500, topk=20, windows="causal")
    c.ks[3] = 7
    c.ke[3] = 5     # ks > ke
    c.ke[4] = 501   # beyond S
    c.ks[5] = -1
    g = gpu_inputs(c)
    idx, val, info = run_select(g)
    assert info["status"] & ftk.STATUS_BAD_WINDOW
    for t in (3, 4, 5):
        assert np.all(idx[t] == -1) and np.all(np.isneginf(val[t]))
    oidx, _, flags = orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk)
    for t in (0, 1, 2, 6, 7, 8, 9):
        n = int(np.sum(oidx[t] >= 0))
        assert n == int(np.sum(idx[t] >= 0))


def test_nan_weight_is_flagged():
    c = wl.small_case(seed=14, dtype="fp8", T=8, S=3000, topk=32, windows="causal")
    c.weights[2, 5] = float("nan")
    g = gpu_inputs(c)
    _, _, info = run_select(g)
    assert info["status"] & ftk.STATUS_NAN


def test_windows_from_cu_seqlens():
    cq = torch.tensor([0, 5, 5, 12, 20], dtype=torch.int32)
    ck = torch.tensor([0, 100, 103, 110, 115], dtype=torch.int32)
    ks, ke = ftk.windows_from_cu_seqlens(cq.cuda(), ck.cuda())
    want_ks, want_ke = wl.packed_causal_windows([5, 0, 7, 8], [100, 3, 7, 5])
    assert torch.equal(ks.cpu(), want_ks)
    # sequence 3 has fewer keys than queries: early queries get empty windows
    want_ke = torch.maximum(want_ke, want_ks)
    assert torch.equal(ke.cpu(), want_ke)


def test_selector_and_last_info():
    c = wl.small_case(seed=15, dtype="fp8", T=16, S=4000, topk=64, windows="causal")
    g = gpu_inputs(c)
    sel = ftk.Selector(topk=64, dtype=torch.float8_e4m3fn).plan(32, 8000)
    idx = sel.run(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales)
    info = sel.last_info
    assert info["rows"] == 16 and info["status"] == 0
    assert info["candidates_total"] >= 16 * 64
    ref, _, _ = run_select(g)
    assert np.array_equal(to_np(idx), ref)


@pytest.mark.parametrize("name", ["fp8_prefill", "fp8_packed", "fp8_large"])
def test_full_size_workloads(name):
    """Full-size FP8 workloads: every row checked against the invariants,
    64 seeded rows (first and last included) bit-exact against the oracle's
    selection of the GPU's own scores and against the fp64 oracle (scores
    within 1e-4 * E, sets up to tie-band swaps)."""
    c = wl.get(name)
    rows = wl.sample_rows(c.T, 64, seed=1)
    _, _, info, worst, overlaps = check_case(c, rows=rows, fp64_rows=rows)
    assert worst < 1e-4
    assert min(overlaps) >= 0.99
    print(f"{name}: worst |dI|/E {worst:.2e}, info {info}")


def test_nan_key_is_flagged():
    """A NaN in kv makes the dot products NaN; ReLU propagates it and the
    status reports it (the row's result is unspecified, nothing traps)."""
    c = wl.small_case(seed=16, dtype="fp8", T=8, S=3000, topk=32, windows="causal")
    c.kv.view(torch.uint8)[1234, 7] = 0x7F  # e4m3fn NaN
    g = gpu_inputs(c)
    _, _, info = run_select(g)
    assert info["status"] & ftk.STATUS_NAN
