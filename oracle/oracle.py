"""ctypes front end of the CPU oracle (``oracle/oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``.  The product package never
imports this module and shares no code with it.

The oracle computes, in IEEE double, the plain definitions from the pages:

* FlashTopK README, "Quick start": I[t,s] = sigma_s * sum_h w[t,h] *
  ReLU(q[t,h] . k[s]) over the window [ks[t], ke[t]); the head count H is
  q.shape[1] (32 on the pages; "Roadmap": other head counts, such as 64);
* FlashTopK README, "Highlights": the exact top-k, ties at the k-th score
  to the smallest key indices;
* DeepSelect README, "Usage": the row top-k of a bf16 / fp32 matrix.

Parity: pinned by tests/test_oracle.py (dtype tables against torch, score
special cases against numpy matmul, brute-force subset enumeration, closed
forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

E4M3, BF16, F32 = 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
             "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def load(path: str):
    """Open an oracle shared library and declare its functions."""
    L = ctypes.CDLL(path)
    P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
    L.orc_e4m3_value.restype = D
    L.orc_e4m3_value.argtypes = [ctypes.c_uint]
    L.orc_bf16_value.restype = D
    L.orc_bf16_value.argtypes = [ctypes.c_uint]
    L.orc_decode.restype = None
    L.orc_decode.argtypes = [I32, P, I64, P]
    L.orc_index_scores.restype = I64
    L.orc_index_scores.argtypes = [I32, I32, P, P, P, P, I64, I64, P, P, P, I64, I64, P, P]
    L.orc_select_f64.restype = I32
    L.orc_select_f64.argtypes = [P, I64, I64, I32, P, P]
    L.orc_select_f32_rows.restype = I64
    L.orc_select_f32_rows.argtypes = [P, I64, I64, P, P, I64, P, I32, P, P]
    L.orc_fused_select.restype = I64
    L.orc_fused_select.argtypes = [I32, I32, P, P, P, P, I64, I64, P, P, P, I64, I32, P, P, P]
    L.orc_topk_rows.restype = I64
    L.orc_topk_rows.argtypes = [I32, P, I64, I64, I64, I32, P, P, P]
    L.orc_num_threads.restype = I32
    L.orc_block_bound.argtypes = [I32, I32, P, P, P, P, I64, I64, I64, P, I64, P, P]
    L.orc_block_bound.restype = None
    L.orc_num_threads.argtypes = []
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(LIB)
    return _lib


class use_library:
    """Context manager: route this module's calls to another oracle build
    (the mutation tests load deliberately broken copies this way)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _raw(a) -> np.ndarray:
    """numpy view of the raw bytes/bits of an input (torch tensors accepted)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            t = a.detach().cpu().contiguous()
            if t.dtype == torch.float8_e4m3fn:
                return t.view(torch.uint8).numpy()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            return t.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(a)


def dtype_code(a) -> int:
    import torch
    if isinstance(a, torch.Tensor):
        return {torch.float8_e4m3fn: E4M3, torch.bfloat16: BF16, torch.float32: F32}[a.dtype]
    raise TypeError("pass torch tensors (dtype decides the decoding)")


def num_threads() -> int:
    return int(lib().orc_num_threads())


def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(code))


def bf16_value(bits: int) -> float:
    return float(lib().orc_bf16_value(bits))


def decode(x) -> np.ndarray:
    """All elements of a fp8/bf16/fp32 torch tensor, decoded to float64."""
    code = dtype_code(x)
    raw = np.ascontiguousarray(_raw(x)).reshape(-1)
    out = np.empty(raw.size, dtype=np.float64)
    lib().orc_decode(code, _ptr(raw), raw.size, _ptr(out))
    return out.reshape(tuple(x.shape))


def _heads(q, weights) -> int:
    """H of a [T, H, 128] q, checked against the [T, H] weights."""
    if q.dim() != 3 or q.shape[2] != 128 or q.shape[1] < 1:
        raise ValueError("q must be [T, H, 128]")
    if tuple(weights.shape) != (q.shape[0], q.shape[1]):
        raise ValueError("weights must be [T, H] for q of shape [T, H, 128]")
    return int(q.shape[1])


def _rows_arg(rows, T):
    if rows is None:
        rows = np.arange(T, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def index_scores(q, kv, kv_scales, weights, ks, ke, rows=None, ld=None):
    """fp64 scores I and error scales E of the listed rows' windows.

    Returns (I, E), each [len(rows), ld] float64, entry (r, s - ks[t]);
    entries past a row's window are NaN.
    """
    T, S = q.shape[0], kv.shape[0]
    qr, kr = _raw(q), _raw(kv)
    sc = None if kv_scales is None else np.ascontiguousarray(_raw(kv_scales), dtype=np.float32)
    w = np.ascontiguousarray(_raw(weights), dtype=np.float32)
    ks_, ke_ = (np.ascontiguousarray(_raw(a), dtype=np.int32) for a in (ks, ke))
    rows = _rows_arg(rows, T)
    if ld is None:
        ld = int(max(1, max((int(ke_[t]) - int(ks_[t]) for t in rows), default=1)))
    I = np.full((rows.size, ld), np.nan)
    E = np.full((rows.size, ld), np.nan)
    lib().orc_index_scores(dtype_code(q), _heads(q, weights), _ptr(qr), _ptr(kr), _ptr(sc), _ptr(w), T, S,
                           _ptr(ks_), _ptr(ke_), _ptr(rows), rows.size, ld, _ptr(I), _ptr(E))
    return I, E


def block_bound(q, kv, kv_scales, weights, block: int = 128, rows=None):
    """Score upper bound of every listed row over every key block of `block`
    keys (the box bound of orc_block_bound).

    Returns (UB, scale), each [len(rows), ceil(S / block)] float64.
    """
    T, S = q.shape[0], kv.shape[0]
    qr, kr = _raw(q), _raw(kv)
    sc = None if kv_scales is None else np.ascontiguousarray(_raw(kv_scales), dtype=np.float32)
    w = np.ascontiguousarray(_raw(weights), dtype=np.float32)
    rows = _rows_arg(rows, T)
    nb = (S + block - 1) // block
    ub = np.empty((rows.size, nb))
    scale = np.empty((rows.size, nb))
    lib().orc_block_bound(dtype_code(q), _heads(q, weights), _ptr(qr), _ptr(kr), _ptr(sc), _ptr(w), T, S, block,
                          _ptr(rows), rows.size, _ptr(ub), _ptr(scale))
    return ub, scale


def select_f64(vals: np.ndarray, first_index: int, k: int):
    """Exact top-k of one window of float64 values: (idx int64[k], val f64[k], nan)."""
    v = np.ascontiguousarray(vals, dtype=np.float64)
    idx = np.empty(k, dtype=np.int64)
    val = np.empty(k, dtype=np.float64)
    nan = lib().orc_select_f64(_ptr(v), v.size, first_index, k, _ptr(idx), _ptr(val))
    return idx, val, bool(nan)


def select_f32_rows(scores: np.ndarray, ks, ke, S: int, k: int, row_ids=None):
    """Exact top-k of float32 score rows (row r = window of query row_ids[r])."""
    sc = np.ascontiguousarray(scores, dtype=np.float32)
    rows, ld = sc.shape
    ks_, ke_ = (np.ascontiguousarray(_raw(a), dtype=np.int32) for a in (ks, ke))
    rid = None if row_ids is None else np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    idx = np.empty((rows, k), dtype=np.int64)
    val = np.empty((rows, k), dtype=np.float64)
    nflag = lib().orc_select_f32_rows(_ptr(sc), rows, ld, _ptr(ks_), _ptr(ke_), S, _ptr(rid), k,
                                      _ptr(idx), _ptr(val))
    return idx, val, int(nflag)


def fused_select(q, kv, kv_scales, weights, ks, ke, k: int, rows=None):
    """Definition-level fused score + top-k of the listed rows.

    Returns (idx int64[n,k], val f64[n,k], flags int32[n]) with rows in
    (score desc, index asc) order and (-1, -inf) padding.
    """
    T, S = q.shape[0], kv.shape[0]
    qr, kr = _raw(q), _raw(kv)
    sc = None if kv_scales is None else np.ascontiguousarray(_raw(kv_scales), dtype=np.float32)
    w = np.ascontiguousarray(_raw(weights), dtype=np.float32)
    ks_, ke_ = (np.ascontiguousarray(_raw(a), dtype=np.int32) for a in (ks, ke))
    rows = _rows_arg(rows, T)
    idx = np.empty((rows.size, k), dtype=np.int64)
    val = np.empty((rows.size, k), dtype=np.float64)
    flags = np.zeros(rows.size, dtype=np.int32)
    lib().orc_fused_select(dtype_code(q), _heads(q, weights), _ptr(qr), _ptr(kr), _ptr(sc), _ptr(w), T, S,
                           _ptr(ks_), _ptr(ke_), _ptr(rows), rows.size, k,
                           _ptr(idx), _ptr(val), _ptr(flags))
    return idx, val, flags


def topk_rows(x, k: int):
    """Row top-k of a [rows, cols] bf16/fp32 torch tensor.

    Returns (idx int64[rows,k], val f64[rows,k], flags int32[rows]).
    """
    code = dtype_code(x)
    raw = np.ascontiguousarray(_raw(x))
    rows, cols = raw.shape
    idx = np.empty((rows, k), dtype=np.int64)
    val = np.empty((rows, k), dtype=np.float64)
    flags = np.zeros(rows, dtype=np.int32)
    lib().orc_topk_rows(code, _ptr(raw), rows, cols, cols, k, _ptr(idx), _ptr(val), _ptr(flags))
    return idx, val, flags
