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


def call_noalloc(g, topk, config=None):
    T, S = g.q.shape[0], g.kv.shape[0]
    idx = torch.full((T, topk), 7, dtype=torch.int32, device="cuda")
    val = torch.full((T, topk), 7.0, dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = ftk.lib().ftk_select_noalloc(
        ftk._dtype_code(g.q), p(g.q), p(g.kv), p(g.kv_scales), p(g.weights), p(g.ks), p(g.ke),
        T, S, topk, p(idx), p(val), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, idx, val


def reference(g, topk):
    return ftk.select(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales, topk, return_scores=True)


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
        torch.cuda.synchronize()
        assert same((idx, val), reference(g, k))


def test_noalloc_rejects_problems_beyond_its_scratch():
    c = wl.small_case(seed=33, dtype="fp8", T=16, S=3000, topk=64, windows="causal").to("cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    big_T, big_S = 1 << 20, 1 << 22  # needs far more than FTK_NOALLOC_SCRATCH_BYTES
    st = ftk.lib().ftk_select_noalloc(1, p(c.q), p(c.kv), None, p(c.weights), p(c.ks), p(c.ke),
                                      big_T, big_S, 4096, p(c.ks), None, None, None)
    assert st == -5  # FTK_ERR_WORKSPACE, nothing launched
