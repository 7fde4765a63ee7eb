"""Pins of the CPU oracle against things other than itself.

Each ``check_*`` function raises AssertionError on a mismatch; the ``test_*``
wrappers run them, and tests/test_oracle_mutations.py runs them against
deliberately broken copies of the oracle to show that each planted mistake
fails at least one pin.

What pins what:
* dtype decoding: torch's own float8_e4m3fn / bfloat16 -> float32 conversion
  tables (library routines) over every code;
* the score: numpy matmul in special cases where the score reduces to a
  plain matrix product (equal heads with uniform weights on non-negative
  data; one-hot weights), linearity in the weights, exact homogeneity, a
  hand-worked example (tests/golden/hand_score.json);
* the selection: brute-force enumeration of all subsets on tiny windows,
  the all-equal row, windows shorter than topk, torch.topk on tie-free rows,
  signed zeros;
* fused select: the all-equal workload's closed form and window locality;
* the block score bound: it dominates every score of its block (checked
  against the score oracle, which the pins above tie down), it equals the
  score for one-key blocks (closed form), and a hand-worked case.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(1234 + seed)


# ---------------------------------------------------------------------------
# dtype decoding
# ---------------------------------------------------------------------------

def check_e4m3_table():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).double().numpy()
    got = orc.decode(codes.view(torch.float8_e4m3fn))
    assert np.array_equal(np.isnan(ref), np.isnan(got)), "NaN codes differ"
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok]), "e4m3 values differ"
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(got[ok])), "signed zero differs"


def check_bf16_table():
    codes = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    x = codes.view(torch.bfloat16)
    ref = x.to(torch.float32).double().numpy()
    got = orc.decode(x)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_e4m3_table():
    check_e4m3_table()


def test_bf16_table():
    check_bf16_table()


# ---------------------------------------------------------------------------
# score
# ---------------------------------------------------------------------------

def _decoded(t):
    return t.to(torch.float32).double().numpy()


def _case(seed, dtype, T, S, nonneg=False, heads=32):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((T, heads, 128), generator=g)
    kv = torch.randn((S, 128), generator=g)
    if nonneg:
        q, kv = q.abs(), kv.abs()
    cast = (lambda x: x.to(torch.float8_e4m3fn)) if dtype == "fp8" else (lambda x: x.to(torch.bfloat16))
    sc = (1.0 - 0.5 * torch.rand(S, generator=g)).float()
    return cast(q), cast(kv), sc


def _full_windows(T, S):
    return torch.zeros(T, dtype=torch.int32), torch.full((T,), S, dtype=torch.int32)


def check_score_equal_heads_matmul(dtype):
    """Equal heads, w = 1/32, non-negative data: I = sigma * (q . k)."""
    T, S = 5, 40
    q, kv, sc = _case(11, dtype, T, S, nonneg=True)
    q = q[:, :1, :].expand(T, 32, 128).contiguous()
    w = torch.full((T, 32), 1.0 / 32)
    ks, ke = _full_windows(T, S)
    I, E = orc.index_scores(q, kv, sc, w, ks, ke)
    ref = (_decoded(q[:, 0, :]) @ _decoded(kv).T) * sc.double().numpy()[None, :]
    np.testing.assert_allclose(I, ref, rtol=1e-12, atol=0)
    np.testing.assert_allclose(E, ref, rtol=1e-12, atol=0)


def check_score_one_hot_heads(dtype):
    """w = c * e_h: I = c * sigma * ReLU(q_h . k) for every head h."""
    T, S = 32, 50
    q, kv, sc = _case(12, dtype, T, S)
    heads = [(7 * t + 3) % 32 for t in range(T)]
    coef = [(-1.0) ** t * (0.75 if t % 3 else 1.25) for t in range(T)]
    w = torch.zeros((T, 32))
    for t in range(T):
        w[t, heads[t]] = coef[t]
    ks, ke = _full_windows(T, S)
    I, _ = orc.index_scores(q, kv, sc, w, ks, ke)
    qd, kd, s = _decoded(q), _decoded(kv), sc.double().numpy()
    for t in range(T):
        dots = qd[t, heads[t], :] @ kd.T
        ref = coef[t] * s * np.maximum(dots, 0.0)
        np.testing.assert_allclose(I[t], ref, rtol=1e-12, atol=1e-300)


def check_score_linear_in_weights(dtype):
    """I(w) = sum_h w_h * I(e_h) (the score is linear in the weights)."""
    T, S = 3, 30
    q, kv, sc = _case(13, dtype, T, S)
    g = torch.Generator().manual_seed(5)
    w = torch.randn((T, 32), generator=g)
    ks, ke = _full_windows(T, S)
    I, _ = orc.index_scores(q, kv, sc, w, ks, ke)
    acc = np.zeros_like(I)
    for h in range(32):
        eh = torch.zeros((T, 32))
        eh[:, h] = 1.0
        Ih, _ = orc.index_scores(q, kv, sc, eh, ks, ke)
        acc += w[:, h].double().numpy()[:, None] * Ih
    np.testing.assert_allclose(I, acc, rtol=1e-12, atol=1e-12)


def check_score_single_head(dtype):
    """H = 1 (FlashTopK README, "Roadmap": other head counts): the score is
    the closed form w * sigma * ReLU(q . k) and E = |w| * sigma * (|q| . |k|),
    one numpy matmul each; weights of both signs (one row per call)."""
    S = 60
    q, kv, sc = _case(15, dtype, 1, S, heads=1)
    ks, ke = _full_windows(1, S)
    qd, kd, s = _decoded(q)[:, 0, :], _decoded(kv), sc.double().numpy()
    for c in (0.625, -1.375):
        w = torch.full((1, 1), c)
        I, E = orc.index_scores(q, kv, sc, w, ks, ke)
        np.testing.assert_allclose(I[0], c * s * np.maximum(qd @ kd.T, 0.0)[0], rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(E[0], abs(c) * s * (np.abs(qd) @ np.abs(kd).T)[0], rtol=1e-12, atol=0)


def check_score_heads_split(dtype):
    """A 64-head score is the sum of the scores of its two 32-head halves
    (and so is E): the head sum covers every head of q[t], with the row
    stride of H heads."""
    T, S = 4, 45
    q, kv, sc = _case(16, dtype, T, S, heads=64)
    w = torch.randn((T, 64), generator=torch.Generator().manual_seed(8)) / 8
    ks, ke = _full_windows(T, S)
    I, E = orc.index_scores(q, kv, sc, w, ks, ke)
    Ia, Ea = orc.index_scores(q[:, :32].contiguous(), kv, sc, w[:, :32].contiguous(), ks, ke)
    Ib, Eb = orc.index_scores(q[:, 32:].contiguous(), kv, sc, w[:, 32:].contiguous(), ks, ke)
    np.testing.assert_allclose(I, Ia + Ib, rtol=0, atol=1e-12 * E.max())
    np.testing.assert_allclose(E, Ea + Eb, rtol=1e-12, atol=0)
    assert np.abs(Ib).max() > 0 and np.abs(Ia).max() > 0


def check_score_head_permutation():
    """Permuting the heads of q and w together leaves the score unchanged
    (H = 48, not a power of two)."""
    T, S = 3, 37
    q, kv, sc = _case(17, "bf16", T, S, heads=48)
    w = torch.randn((T, 48), generator=torch.Generator().manual_seed(9))
    perm = torch.randperm(48, generator=torch.Generator().manual_seed(10))
    ks, ke = _full_windows(T, S)
    I, E = orc.index_scores(q, kv, sc, w, ks, ke)
    Ip, Ep = orc.index_scores(q[:, perm].contiguous(), kv, sc, w[:, perm].contiguous(), ks, ke)
    np.testing.assert_allclose(Ip, I, rtol=0, atol=1e-12 * E.max())
    np.testing.assert_allclose(Ep, E, rtol=1e-12, atol=0)


def check_score_homogeneity():
    """I(2q) = 2 I(q), I(2 sigma) = 2 I(sigma) exactly (BF16, power-of-two)."""
    T, S = 4, 33
    q, kv, sc = _case(14, "bf16", T, S)
    w = torch.randn((T, 32), generator=torch.Generator().manual_seed(6))
    ks, ke = _full_windows(T, S)
    I, _ = orc.index_scores(q, kv, sc, w, ks, ke)
    I2, _ = orc.index_scores((q.float() * 2).to(torch.bfloat16), kv, sc, w, ks, ke)
    I3, _ = orc.index_scores(q, kv, sc * 2, w, ks, ke)
    assert np.array_equal(I2, 2 * I) and np.array_equal(I3, 2 * I)
    In, _ = orc.index_scores(q, kv, None, w, ks, ke)
    I1, _ = orc.index_scores(q, kv, torch.ones(S), w, ks, ke)
    assert np.array_equal(In, I1), "NULL kv_scales must mean all ones"


def _hand():
    with open(os.path.join(GOLDEN, "hand_score.json")) as f:
        d = json.load(f)
    q = torch.zeros((1, 32, 128))
    for t, h, dd, v in d["q_entries"]:
        q[t, h, dd] = v
    w = torch.zeros((1, 32))
    for t, h, v in d["w_entries"]:
        w[t, h] = v
    kv = torch.zeros((5, 128))
    for s, dd, v in d["k_entries"]:
        kv[s, dd] = v
    return d, q.to(torch.bfloat16), kv.to(torch.bfloat16), torch.tensor(d["kv_scales"]), w


def check_hand_example():
    d, q, kv, sc, w = _hand()
    ks = torch.tensor([0], dtype=torch.int32)
    ke = torch.tensor([5], dtype=torch.int32)
    I, E = orc.index_scores(q, kv, sc, w, ks, ke)
    assert I[0].tolist() == d["I"], (I, d["I"])
    assert E[0].tolist() == d["E"], (E, d["E"])
    for sel in d["selections"]:
        ks = torch.tensor([sel["ks"]], dtype=torch.int32)
        ke = torch.tensor([sel["ke"]], dtype=torch.int32)
        idx, val, flags = orc.fused_select(q, kv, sc, w, ks, ke, sel["topk"])
        assert idx[0].tolist() == sel["idx"], (idx, sel)
        want = [float(v) for v in sel["val"]]
        assert val[0].tolist() == want, (val, sel)
        assert flags[0] == 0


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_score_equal_heads_matmul(dtype):
    check_score_equal_heads_matmul(dtype)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_score_one_hot_heads(dtype):
    check_score_one_hot_heads(dtype)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_score_linear_in_weights(dtype):
    check_score_linear_in_weights(dtype)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_score_single_head(dtype):
    check_score_single_head(dtype)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_score_heads_split(dtype):
    check_score_heads_split(dtype)


def test_score_head_permutation():
    check_score_head_permutation()


def test_heads_shape_checked():
    q, kv, sc = _case(18, "bf16", 2, 10, heads=64)
    ks, ke = _full_windows(2, 10)
    with pytest.raises(ValueError):
        orc.index_scores(q, kv, sc, torch.ones((2, 32)), ks, ke)


def test_score_homogeneity():
    check_score_homogeneity()


def test_hand_example():
    check_hand_example()


def test_score_windows_relative_and_error_bound():
    """Window entries are relative to ks; |I| <= E everywhere."""
    T, S = 6, 70
    q, kv, sc = _case(15, "fp8", T, S)
    w = torch.randn((T, 32), generator=torch.Generator().manual_seed(7))
    ks = torch.tensor([0, 5, 10, 33, 69, 70], dtype=torch.int32)
    ke = torch.tensor([70, 60, 11, 69, 70, 70], dtype=torch.int32)
    I, E = orc.index_scores(q, kv, sc, w, ks, ke)
    Ifull, _ = orc.index_scores(q, kv, sc, w, torch.zeros(T, dtype=torch.int32),
                                torch.full((T,), S, dtype=torch.int32))
    for t in range(T):
        L = int(ke[t] - ks[t])
        assert np.array_equal(I[t, :L], Ifull[t, int(ks[t]):int(ke[t])])
        assert np.all(np.isnan(I[t, L:]))
        assert np.all(np.abs(I[t, :L]) <= E[t, :L])


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------

def brute_force_topk(vals, first, k):
    """The unique subset X (|X| = min(k, L)) such that every key in X beats
    every key outside it: larger score, or equal score and smaller index.
    Found by trying every subset."""
    L = len(vals)
    n = min(k, L)
    keys = list(range(L))
    found = []
    for X in itertools.combinations(keys, n):
        inside = set(X)
        ok = all((vals[a] > vals[b]) or (vals[a] == vals[b] and a < b)
                 for a in inside for b in keys if b not in inside)
        if ok:
            found.append(X)
    assert len(found) == 1, found
    return sorted(first + j for j in found[0])


def check_select_brute_force():
    r = _rng(0)
    for trial in range(150):
        L = int(r.integers(0, 9))
        vals = r.integers(-3, 4, size=L).astype(np.float64) * 0.5
        first = int(r.integers(0, 1000))
        for k in range(1, L + 3):
            idx, val, nan = orc.select_f64(vals, first, k)
            want = brute_force_topk(vals.tolist(), first, k)
            n = min(k, L)
            assert sorted(idx[:n].tolist()) == want, (vals, k, idx)
            assert np.all(idx[n:] == -1) and np.all(np.isneginf(val[n:]))
            assert [vals[i - first] for i in idx[:n]] == val[:n].tolist()
            assert not nan


def check_select_all_equal():
    vals = np.full(300, 2.5)
    for first, k in [(0, 1), (17, 64), (5, 300), (9, 400)]:
        idx, _, _ = orc.select_f64(vals, first, k)
        n = min(k, 300)
        assert idx[:n].tolist() == list(range(first, first + n))


def check_select_torch_topk_tie_free():
    r = _rng(1)
    for L, k in [(1000, 37), (4096, 512), (50, 50), (20, 1)]:
        vals = r.permutation(L).astype(np.float64) + r.random(L) * 0.5  # distinct
        idx, val, _ = orc.select_f64(vals, 100, k)
        tv, ti = torch.topk(torch.from_numpy(vals), k)
        assert sorted(idx.tolist()) == sorted((ti + 100).tolist())
        assert np.array_equal(val, tv.numpy())


def check_select_signed_zero():
    vals = np.array([0.0, -0.0, 0.0, -0.0, 1.0, -1.0])
    idx, val, _ = orc.select_f64(vals, 0, 3)
    assert sorted(idx.tolist()) == [0, 1, 4]
    idx, val, _ = orc.select_f64(vals, 0, 5)
    assert sorted(idx.tolist()) == [0, 1, 2, 3, 4]


def test_select_brute_force():
    check_select_brute_force()


def test_select_all_equal():
    check_select_all_equal()


def test_select_torch_topk_tie_free():
    check_select_torch_topk_tie_free()


def test_select_signed_zero():
    check_select_signed_zero()


def test_select_nan_flag():
    _, _, nan = orc.select_f64(np.array([1.0, np.nan, 2.0]), 0, 2)
    assert nan
    _, _, nan = orc.select_f64(np.array([1.0, 3.0, 2.0]), 0, 2)
    assert not nan


def test_select_f32_rows_matches_f64():
    r = _rng(2)
    sc = r.standard_normal((4, 300)).astype(np.float32)
    sc[2, :] = np.round(sc[2, :])            # many ties
    ks = np.array([0, 10, 0, 5], dtype=np.int32)
    ke = np.array([300, 250, 300, 5], dtype=np.int32)
    idx, val, nflag = orc.select_f32_rows(sc, ks, ke, 400, 40)
    assert nflag == 0
    for rr in range(4):
        L = ke[rr] - ks[rr]
        i2, v2, _ = orc.select_f64(sc[rr, :L].astype(np.float64), int(ks[rr]), 40)
        assert np.array_equal(idx[rr], i2) and np.array_equal(val[rr], v2)


# ---------------------------------------------------------------------------
# row top-k
# ---------------------------------------------------------------------------

def check_topk_rows_brute_force():
    r = _rng(3)
    for dt in (torch.bfloat16, torch.float32):
        for trial in range(40):
            cols = int(r.integers(1, 9))
            x = torch.from_numpy(r.integers(-2, 3, size=(2, cols)).astype(np.float32) * 0.25).to(dt)
            for k in range(1, cols + 2):
                idx, val, flags = orc.topk_rows(x, k)
                for row in range(2):
                    vals = x[row].float().tolist()
                    want = brute_force_topk(vals, 0, k)
                    n = min(k, cols)
                    assert sorted(idx[row, :n].tolist()) == want
                    assert np.all(idx[row, n:] == -1)
                    assert flags[row] == 0


def check_topk_rows_torch_tie_free():
    r = _rng(4)
    x = torch.from_numpy(np.stack([r.permutation(5000) for _ in range(3)]).astype(np.float32) * 0.001)
    idx, val, _ = orc.topk_rows(x, 300)
    tv, ti = torch.topk(x, 300, dim=1)
    for row in range(3):
        assert sorted(idx[row].tolist()) == sorted(ti[row].tolist())
        assert np.array_equal(val[row], tv[row].double().numpy())


def test_topk_rows_brute_force():
    check_topk_rows_brute_force()


def test_topk_rows_torch_tie_free():
    check_topk_rows_torch_tie_free()


def test_topk_rows_heavy_ties_and_nan():
    x = torch.tensor([[1.0, 3.0, 3.0, 2.0, 3.0, 3.0], [1.0, float("nan"), 0.0, 0.0, 0.0, 0.0]])
    idx, val, flags = orc.topk_rows(x, 3)
    assert idx[0].tolist() == [1, 2, 4] and flags[0] == 0
    assert flags[1] == 1


# ---------------------------------------------------------------------------
# fused select
# ---------------------------------------------------------------------------

def check_fused_all_equal():
    """Constant keys: every score of the row is equal, so the result is
    ks .. ks+k-1 (the tie rule) -- the bf16_all_equal workload."""
    from sparse_attention_indexer_ftk_b200 import workloads as wl
    c = wl.bf16_all_equal()
    idx, val, flags = orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk)
    for t in range(c.T):
        ks = int(c.ks[t])
        assert idx[t].tolist() == list(range(ks, ks + c.topk))
        assert np.all(val[t] == val[t][0])
        assert flags[t] == 0


def test_fused_all_equal():
    check_fused_all_equal()


def test_fused_matches_scores_then_select():
    T, S = 9, 120
    q, kv, sc = _case(16, "fp8", T, S)
    w = torch.randn((T, 32), generator=torch.Generator().manual_seed(8))
    ks = torch.tensor([0, 0, 3, 50, 100, 119, 120, 7, 0], dtype=torch.int32)
    ke = torch.tensor([120, 1, 90, 60, 120, 120, 120, 7, 64], dtype=torch.int32)
    k = 16
    idx, val, flags = orc.fused_select(q, kv, sc, w, ks, ke, k)
    I, _ = orc.index_scores(q, kv, sc, w, ks, ke)
    for t in range(T):
        L = int(ke[t] - ks[t])
        i2, v2, _ = orc.select_f64(I[t, :L], int(ks[t]), k)
        assert np.array_equal(idx[t], i2) and np.array_equal(val[t], v2)
        assert flags[t] == 0


def test_fused_invalid_window_flag():
    T, S = 3, 20
    q, kv, sc = _case(17, "bf16", T, S)
    w = torch.ones((T, 32))
    ks = torch.tensor([5, -1, 0], dtype=torch.int32)
    ke = torch.tensor([4, 3, 21], dtype=torch.int32)
    idx, val, flags = orc.fused_select(q, kv, sc, w, ks, ke, 4)
    assert flags.tolist() == [2, 2, 2]
    assert np.all(idx == -1) and np.all(np.isneginf(val))


def test_fused_window_locality():
    """Changing keys outside a row's window does not change its result."""
    T, S = 4, 90
    q, kv, sc = _case(18, "fp8", T, S)
    w = torch.randn((T, 32), generator=torch.Generator().manual_seed(9))
    ks = torch.tensor([10, 20, 0, 40], dtype=torch.int32)
    ke = torch.tensor([50, 60, 30, 90], dtype=torch.int32)
    a = orc.fused_select(q, kv, sc, w, ks, ke, 8)
    kv2 = kv.clone()
    kv2.view(torch.uint8)[:10] = 0x38  # 1.0 in e4m3, outside every window but row 2's
    b = orc.fused_select(q, kv2, sc, w, ks, ke, 8)
    for t in (0, 1, 3):
        assert np.array_equal(a[0][t], b[0][t])


# ---------------------------------------------------------------------------
# block score bound
# ---------------------------------------------------------------------------

def _bound_case(dtype, seed=21, T=3, S=300, heads=32):
    q, kv, sc = _case(seed, dtype, T, S, heads=heads)
    w = torch.randn((T, heads), generator=torch.Generator().manual_seed(seed + 1)) / math.sqrt(heads)
    return q, kv, sc, w


def check_bound_dominates_scores(dtype, heads=32):
    """UB(t, b) >= I(t, s) for every key s of block b (blocks of 128 and a
    ragged last block of 44 keys), with weights of both signs."""
    q, kv, sc, w = _bound_case(dtype, heads=heads)
    T, S = q.shape[0], kv.shape[0]
    ks, ke = _full_windows(T, S)
    I, _ = orc.index_scores(q, kv, sc, w, ks, ke)
    ub, scale = orc.block_bound(q, kv, sc, w, block=128)
    assert ub.shape == (T, 3)
    for b in range(3):
        blk = I[:, b * 128:min(S, (b + 1) * 128)]
        assert np.all(ub[:, b] >= blk.max(axis=1) - 1e-12 * scale[:, b]), (b, ub[:, b], blk.max(axis=1))
    # the bound is not vacuous: it stays within the size of its own terms
    assert np.all(np.abs(ub) <= scale * (1 + 1e-12))


def check_bound_one_key_blocks(dtype):
    """A block of one key is a point box: UB(t, s) = I(t, s)."""
    q, kv, sc, w = _bound_case(dtype, seed=22, T=2, S=40)
    ks, ke = _full_windows(2, 40)
    I, E = orc.index_scores(q, kv, sc, w, ks, ke)
    ub, scale = orc.block_bound(q, kv, sc, w, block=1)
    np.testing.assert_allclose(ub, I, rtol=0, atol=1e-12 * E.max())
    np.testing.assert_allclose(scale, E, rtol=1e-12, atol=0)


def check_bound_hand_example():
    """Worked by hand from the definition.  Row 0: q[0,0,0] = 2,
    q[0,1,0] = -1, q[0,2,1] = 1; w = (0.5, -2, -1, 0, ...); two keys with
    k0 = (-1, 2, 0...), k1 = (3, 5, 0...), sigma = 1.  Box: hi = (3, 5),
    lo = (-1, 2).  Head 0: U = max(6, -2) = 6.  Head 1: U = max(-3, 1) = 1,
    L = -3.  Head 2: U = 5, L = 2.  UB = 0.5*6 + (-2)*ReLU(-3) + (-1)*ReLU(2)
    = 1.  Term sizes: 0.5*2*3 + 2*1*3 + 1*1*5 = 14.  The scores are
    I(k0) = 0 - 2 - 2 = -4 and I(k1) = 3 + 0 - 5 = -2."""
    q = torch.zeros((1, 32, 128))
    q[0, 0, 0], q[0, 1, 0], q[0, 2, 1] = 2.0, -1.0, 1.0
    w = torch.zeros((1, 32))
    w[0, 0], w[0, 1], w[0, 2] = 0.5, -2.0, -1.0
    kv = torch.zeros((2, 128))
    kv[0, 0], kv[0, 1], kv[1, 0], kv[1, 1] = -1.0, 2.0, 3.0, 5.0
    qb, kb = q.to(torch.bfloat16), kv.to(torch.bfloat16)
    ub, scale = orc.block_bound(qb, kb, None, w, block=128)
    assert ub.tolist() == [[1.0]] and scale.tolist() == [[14.0]], (ub, scale)
    ks, ke = _full_windows(1, 2)
    I, _ = orc.index_scores(qb, kb, None, w, ks, ke)
    assert I[0].tolist() == [-4.0, -2.0]


def test_bound_rows_outside_the_batch_are_nan():
    q, kv, sc, w = _bound_case("bf16", T=2, S=200)
    ub, scale = orc.block_bound(q, kv, sc, w, rows=[1, 2, -1])
    assert np.all(np.isfinite(ub[0])) and np.all(np.isnan(ub[1:])) and np.all(np.isnan(scale[1:]))


def test_bound_dominates_scores_64_heads():
    check_bound_dominates_scores("fp8", heads=64)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_bound_dominates_scores(dtype):
    check_bound_dominates_scores(dtype)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_bound_one_key_blocks(dtype):
    check_bound_one_key_blocks(dtype)


def test_bound_hand_example():
    check_bound_hand_example()
