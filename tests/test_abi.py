"""The C-ABI library loads, exports every symbol include/ftk.h declares, and
rejects bad arguments on the host before touching a GPU."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

from sparse_attention_indexer_ftk_b200 import build as ftk_build
from sparse_attention_indexer_ftk_b200 import ftk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ftk.h")


@pytest.fixture(scope="module")
def lib():
    ftk_build.build()
    return ftk.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ftk_[a-z0-9_]+)\s*\(", text)))


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C11 program includes include/ftk.h, links libftk.so and calls the
    host-side entry points (no GPU): the boundary needs no C++ or torch."""
    exe = tmp_path / "c_abi_check"
    libdir = os.path.dirname(ftk.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe), "-L", libdir, "-lftk",
                           "-Wl,-rpath," + libdir, "-lm"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "OK", out.stdout + out.stderr


def test_header_matches_binding_list():
    assert declared_functions() == sorted(ftk.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", ftk.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (ftk_[a-z0-9_]+)$", out, flags=re.M))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(lib, f)


def test_version_and_strings(lib):
    assert lib.ftk_version() == 100
    assert lib.ftk_status_string(0) == b"ok"
    assert b"topk" in lib.ftk_status_string(-3)
    assert lib.ftk_status_string(12345) == b"unknown status"


def test_structs_match_header_sizes():
    assert ctypes.sizeof(ftk.FtkConfig) == 32
    assert ctypes.sizeof(ftk.FtkInfo) == 8 + 8 * 8


def test_workspace_size(lib):
    n1 = lib.ftk_select_workspace_size(4096, 131072, 2048, None)
    n2 = lib.ftk_select_workspace_size(128, 2048, 256, None)
    assert n1 > n2 > 0
    assert lib.ftk_select_workspace_size(0, 10, 5, None) == 0
    assert lib.ftk_select_workspace_size(10, 10, 5000, None) == 0
    cfg = ftk.FtkConfig(capacity=4096 * 2)
    assert lib.ftk_select_workspace_size(4096, 131072, 2048, ctypes.byref(cfg)) >= n1


def test_workspace_planned_for_larger_sizes_serves_smaller_calls(lib):
    """The size is non-decreasing in T and S (the header's promise behind
    Selector.plan(max_rows, max_kv)): a workspace planned for (T, S) is
    large enough for every call with smaller T and S.  The recovery scratch
    once broke this: rows x row length rounded to multiples of 16 rows
    grew for some smaller S."""
    cfgs = [None, ftk.FtkConfig(recovery_rows=8), ftk.FtkConfig(recovery_rows=100, capacity=64),
            ftk.FtkConfig(prune=-1), ftk.FtkConfig(sample_keys=64)]
    for cfg in cfgs:
        ref = None if cfg is None else ctypes.byref(cfg)
        for T, S in [(17, 129), (4096, 1000000), (8192, 262144), (64, 3000000)]:
            big = lib.ftk_select_workspace_size(T, S, 2048, ref)
            for S2 in sorted({1, S // 2 + 1} | set(range(S // 2 + 1, S + 1, max(1, S // 61)))):
                for T2 in (1, T // 2 + 1, T):
                    assert lib.ftk_select_workspace_size(T2, S2, 2048, ref) <= big, (cfg, T, S, T2, S2)


A = 0x10000  # a 16-byte aligned stand-in pointer (never dereferenced on the host)


def test_topk_rows_end_host_validation(lib):
    P = ctypes.c_void_p
    assert lib.ftk_topk_rows_end(2, P(A), 4, 100, 104, None, 8, P(A), None, None, None) == -1
    assert lib.ftk_topk_rows_end(2, P(A), 4, 100, 104, P(A), 0, P(A), None, None, None) == -3
    assert lib.ftk_topk_rows_end(1, P(A), 4, 100, 104, P(A), 8, P(A), None, None, None) == -2
    assert lib.ftk_topk_rows_end(2, P(A + 2), 4, 100, 104, P(A), 8, P(A), None, None, None) == -4


def test_topk_rows_sorted_host_validation(lib):
    P = ctypes.c_void_p
    # out_val is required: the sort needs the values
    assert lib.ftk_topk_rows_sorted(2, P(A), 4, 100, 104, None, 8, P(A), None, None, None) == -1
    assert lib.ftk_topk_rows_sorted(2, P(A), 4, 100, 104, None, 0, P(A), P(A), None, None) == -3


def test_rows_options_init_defaults(lib):
    o = ftk.FtkRowsOptions(sorted=5, index_bits=7, out_stride=9, idx_fill=11, val_fill=13.0)
    lib.ftk_rows_options_init(ctypes.byref(o))
    assert (o.sorted, o.index_bits, o.out_stride, o.idx_fill) == (0, 32, 0, -1)
    assert o.val_fill == float("-inf")
    lib.ftk_rows_options_init(None)  # no-op
    assert ctypes.sizeof(ftk.FtkRowsOptions) == 32  # int32, int32, int64, int64, float + padding


def test_topk_rows_ex_host_validation(lib):
    P = ctypes.c_void_p

    def call(idx=A, val=None, topk=8, **opt):
        o = ftk.FtkRowsOptions()
        lib.ftk_rows_options_init(ctypes.byref(o))
        for k, v in opt.items():
            setattr(o, k, v)
        return lib.ftk_topk_rows_ex(2, P(A), 4, 100, 104, None, topk, ctypes.byref(o), P(idx),
                                    None if val is None else P(val), None, None)
    assert call(sorted=2) == -1
    assert call(index_bits=16) == -1 and call(index_bits=0) == -1
    assert call(out_stride=7) == -1 and call(out_stride=-8) == -1 and call(out_stride=1 << 31) == -1
    assert call(idx_fill=1 << 31) == -1 and call(idx_fill=-(1 << 31) - 1) == -1
    assert call(topk=0) == -3 and call(topk=4097) == -3
    assert call(idx=0) == -1
    assert call(idx=A + 4, index_bits=64) == -4   # int64 output on a 4-byte boundary
    assert call(idx=A + 2) == -4                   # int32 output on a 2-byte boundary
    assert call(val=A + 1) == -4                   # bf16 values on an odd address
    # options=NULL means the defaults; the bad x pointer is still caught first
    assert lib.ftk_topk_rows_ex(2, None, 4, 100, 104, None, 8, None, P(A), None, None, None) == -1


def test_block_bound_host_validation(lib):
    P = ctypes.c_void_p
    need = lib.ftk_block_bound_workspace_size(1000)
    assert need >= 8 * 257 * 4 and lib.ftk_block_bound_workspace_size(0) == 0

    def call(dtype=1, q=A, kv=A, w=A, T=4, S=1000, out=A, ld=8, ws=A, wsz=None):
        return lib.ftk_block_bound(dtype, P(q), P(kv), None, P(w), T, S, P(out), ld, P(ws),
                                   need if wsz is None else wsz, None)
    assert call(dtype=3) == -2
    assert call(q=0) == -1 and call(out=0) == -1
    assert call(T=0) == -1 and call(S=0) == -1
    assert call(ld=7) == -1                  # ld < ceil(S / 128)
    assert call(kv=A + 8) == -4
    assert call(ws=0) == -5 and call(ws=A + 16) == -5 and call(wsz=need - 1) == -5


def test_topk_rows_host_validation(lib):
    P = ctypes.c_void_p
    assert lib.ftk_topk_rows(2, P(A), 4, 100, 104, 0, P(A), None, None, None) == -3
    assert lib.ftk_topk_rows(2, P(A), 4, 100, 104, 4097, P(A), None, None, None) == -3
    assert lib.ftk_topk_rows(2, None, 4, 100, 104, 8, P(A), None, None, None) == -1
    assert lib.ftk_topk_rows(1, P(A), 4, 100, 104, 8, P(A), None, None, None) == -2
    assert lib.ftk_topk_rows(2, P(A + 2), 4, 100, 104, 8, P(A), None, None, None) == -4
    assert lib.ftk_topk_rows(2, P(A), 4, 100, 101, 8, P(A), None, None, None) == -4
    assert lib.ftk_topk_rows(3, P(A), 4, 100, 99, 8, P(A), None, None, None) == -1
    assert lib.ftk_topk_rows(3, P(A), 4, 1 << 31, 1 << 31, 8, P(A), None, None, None) == -2


def test_select_host_validation(lib):
    P = ctypes.c_void_p
    args = lambda **kw: dict(dict(dtype=1, q=P(A), kv=P(A), sc=None, w=P(A), ks=P(A), ke=P(A), T=16,
                                  S=1000, k=8, oi=P(A), ov=None, ws=P(A), wsb=1 << 30, cfg=None,
                                  st=None), **kw)

    def call(**kw):
        a = args(**kw)
        return lib.ftk_select(a["dtype"], a["q"], a["kv"], a["sc"], a["w"], a["ks"], a["ke"], a["T"],
                              a["S"], a["k"], a["oi"], a["ov"], a["ws"], a["wsb"], a["cfg"], a["st"])

    assert call(k=0) == -3
    assert call(k=4097) == -3
    assert call(dtype=3) == -2
    assert call(q=None) == -1
    assert call(T=0) == -1
    assert call(q=P(A + 8)) == -4
    assert call(ws=None) == -5
    assert call(ws=P(A + 16)) == -5
    assert call(wsb=1000) == -5
    bad = ftk.FtkConfig()
    bad.reserved = 1
    assert call(cfg=ctypes.byref(bad)) == -1


def test_score_dense_host_validation(lib):
    P = ctypes.c_void_p
    r = lib.ftk_score_dense(1, P(A), P(A), None, P(A), P(A), P(A), 16, 1000, None, 16, P(A), 1002,
                            P(A), 256, None)
    assert r == -1  # ld not a multiple of 4
    r = lib.ftk_score_dense(1, P(A), P(A), None, P(A), P(A), P(A), 16, 1000, None, 17, P(A), 1000,
                            P(A), 256, None)
    assert r == -1  # more rows than T without a row list
    r = lib.ftk_score_dense(1, P(A), P(A), None, P(A), P(A), P(A), 16, 1000, None, 16, P(A), 996,
                            P(A), 256, None)
    assert r == -1  # ld < S: a window could run past its row


def test_head_count_validation(lib):
    """ftk_config.heads: 0 or 32 (default) or 64; anything else is refused
    by ftk_select, by the workspace query (0) and by ftk_score_dense_heads."""
    P = ctypes.c_void_p
    for h in (0, 32, 64):
        assert lib.ftk_select_workspace_size(100, 1000, 16, ctypes.byref(ftk.FtkConfig(heads=h))) > 0
    for h in (-1, 1, 16, 48, 128):
        cfg = ftk.FtkConfig(heads=h)
        assert lib.ftk_select_workspace_size(100, 1000, 16, ctypes.byref(cfg)) == 0
        assert lib.ftk_select(1, P(A), P(A), None, P(A), P(A), P(A), 100, 1000, 16, P(A), None, P(A),
                              1 << 30, ctypes.byref(cfg), None) == -1
        assert lib.ftk_score_dense_heads(1, h, P(A), P(A), None, P(A), P(A), P(A), 16, 1000, None, 16,
                                         P(A), 1000, P(A), 256, None) == -1
        assert lib.ftk_block_bound_heads(1, h, P(A), P(A), None, P(A), 4, 1000, P(A), 8, P(A), 1 << 20,
                                         None) == -1
    # 64 heads: twice the row tiles (4 or 8 queries per tile instead of 8 or 16)
    n32 = lib.ftk_select_workspace_size(4096, 131072, 2048, None)
    n64 = lib.ftk_select_workspace_size(4096, 131072, 2048, ctypes.byref(ftk.FtkConfig(heads=64)))
    assert n64 > 0 and n32 > 0


def test_stage_events_host_validation(lib):
    """The hook takes 7 or 8 non-NULL handles (copied), and n = 0 or NULL
    switches it off; nothing is recorded until an ftk_select call."""
    P = ctypes.c_void_p
    fake = (P * 8)(*[P(A + 64 * i) for i in range(8)])  # never recorded: no select runs here
    try:
        assert lib.ftk_set_stage_events(fake, 6) == -1
        holes = (P * 8)(*[P(A + 64 * i) for i in range(8)])
        holes[3] = None
        assert lib.ftk_set_stage_events(holes, 8) == -1
        assert lib.ftk_set_stage_events(fake, 7) == 0
        assert lib.ftk_set_stage_events(fake, 12) == 0
    finally:
        assert lib.ftk_set_stage_events(None, 0) == 0
    assert lib.ftk_set_stage_events(fake, 0) == 0


def test_windows_host_validation(lib):
    P = ctypes.c_void_p
    assert lib.ftk_windows_from_cu_seqlens(None, P(A), 2, 10, P(A), P(A), None) == -1
    assert lib.ftk_windows_from_cu_seqlens(P(A), P(A), 0, 10, P(A), P(A), None) == -1
    assert lib.ftk_windows_from_cu_seqlens(P(A), P(A), 2, 0, P(A), P(A), None) == 0


def test_product_has_no_cpu_fallback(tmp_path, monkeypatch):
    """Without libftk.so the binding raises instead of computing on the CPU."""
    monkeypatch.setattr(ftk, "_lib", None)
    monkeypatch.setattr(ftk, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ftk.FtkError):
        ftk.load_library(str(tmp_path / "missing.so"))


def test_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "sparse_attention_indexer_ftk_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"(from|import)\s+oracle|liboracle|orc_", text), f
