"""ftk_select_noalloc: fused score + top-k for callers that cannot allocate
device memory (its scratch is a fixed array inside libftk).

Called through the C ABI; each call must give exactly what ftk_select gives
with a caller-owned workspace, also on the second of two calls in a row
(the fixed array keeps the previous call's contents).  This file is named to
be collected last.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from sparse_attention_indexer_ftk_b200 import ftk
from sparse_attention_indexer_ftk_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def call_noalloc(g, topk, config=None):
    T, S = g.q.shape[0], g.kv.shape[0]
    idx = torch.full((T, topk), 7, dtype=torch.int32, device="cuda")
    val = torch.full((T, topk), 7.0, dtype=torch.float32, device="cuda")
    st = ftk.lib().ftk_select_noalloc(
        ftk._dtype_code(g.q), _p(g.q), _p(g.kv), _p(g.kv_scales), _p(g.weights), _p(g.ks), _p(g.ke),
        T, S, topk, _p(idx), _p(val), None, _stream())
    return st, idx, val


def noalloc_info():
    info = ftk.FtkInfo()
    st = ftk.lib().ftk_noalloc_read_info(ctypes.byref(info), _stream())
    assert st == 0, ftk.lib().ftk_status_string(st)
    return info.as_dict()


def reference(g, topk):
    ws = torch.empty(ftk.select_workspace_size(g.T, g.S, topk), dtype=torch.uint8, device="cuda")
    idx, val = ftk.select(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales, topk, return_scores=True,
                          workspace=ws)
    return idx, val, ftk.read_info(ws)


def same(a, b):
    ia, va = a
    ib, vb = b
    return torch.equal(ia, ib) and torch.equal(va.view(torch.int32), vb.view(torch.int32))


def test_noalloc_matches_select_on_two_calls_in_a_row():
    first = wl.small_case(seed=31, dtype="fp8", T=40, S=20000, topk=512, windows="causal").to("cuda")
    second = wl.small_case(seed=32, dtype="bf16", T=24, S=6000, topk=128, windows="random").to("cuda")
    for g, k in ((first, 512), (second, 128)):
        st, idx, val = call_noalloc(g, k)
        assert st == 0, ftk.lib().ftk_status_string(st)
        info = noalloc_info()
        ridx, rval, rinfo = reference(g, k)
        assert same((idx, val), (ridx, rval))
        assert info["status"] == rinfo["status"] == 0
        assert info["rows"] == g.T


def test_noalloc_status_bits_are_readable():
    """A row whose window is invalid (ks > ke) is written as (-1, -inf) and
    raises FTK_STATUS_BAD_WINDOW in the info the caller reads back."""
    c = wl.small_case(seed=34, dtype="bf16", T=10, S=500, topk=20, windows="causal")
    c.ks[3] = 7
    c.ke[3] = 5
    g = c.to("cuda")
    st, idx, val = call_noalloc(g, 20)
    assert st == 0
    info = noalloc_info()
    assert info["status"] & ftk.STATUS_BAD_WINDOW
    assert torch.all(idx[3] == -1) and torch.all(torch.isneginf(val[3]))
    ridx, rval, _ = reference(g, 20)
    assert same((idx, val), (ridx, rval))


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Valid arguments whose scratch would exceed the fixed array: rejected
    with FTK_ERR_WORKSPACE before anything is launched; argument errors are
    still reported first."""
    c = wl.small_case(seed=33, dtype="fp8", T=16, S=3000, topk=64, windows="causal").to("cuda")
    big_T, big_S = 1 << 20, 1 << 22  # needs far more than FTK_NOALLOC_SCRATCH_BYTES
    out = torch.empty(16, dtype=torch.int32, device="cuda")
    L = ftk.lib()
    st = L.ftk_select_noalloc(1, _p(c.q), _p(c.kv), None, _p(c.weights), _p(c.ks), _p(c.ke),
                              big_T, big_S, 4096, _p(out), None, None, None)
    assert st == -5  # FTK_ERR_WORKSPACE
    st = L.ftk_select_noalloc(1, None, _p(c.kv), None, _p(c.weights), _p(c.ks), _p(c.ke),
                              big_T, big_S, 4096, _p(out), None, None, None)
    assert st == -1  # FTK_ERR_INVALID_ARG (NULL q) comes before the size check
