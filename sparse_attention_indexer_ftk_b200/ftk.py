"""Python binding of libftk (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this
module checks shapes and dtypes, allocates outputs with torch, and passes
raw device pointers plus the current CUDA stream through the C ABI declared
in include/ftk.h.  If libftk.so is missing the calls raise: there is no CPU
fallback.

API (names after the pages' own):
  select(q, kv, weights, ks, ke, kv_scales=None, topk=2048, return_scores=False)
      FlashTopK README, "Usage": flashtopk.select
  Selector(topk, dtype).plan(max_rows, max_kv).run(...)
      FlashTopK README, "Usage": Selector (owns the workspace)
  windows_from_cu_seqlens(cu_seqlens_q, cu_seqlens_k)
      FlashTopK README, "Usage"
  topk_rows(x, topk, return_value=True, end=None, sorted=False,
            indices_type=torch.int32, idx_fill=-1, val_fill=-inf)
      DeepSelect README, "Usage" and "Variable-length rows":
      deep_select.topk (unsorted output in ascending index order)
  score_dense(q, kv, weights, ks, ke, kv_scales=None, rows=None)
      the fused scores themselves, for checking
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libftk.so")

F8E4M3, BF16, F32 = 1, 2, 3
STATUS_BAD_WINDOW, STATUS_NAN, STATUS_TIMEOUT, STATUS_BAD_SCALE, STATUS_INTERNAL = 1, 2, 4, 8, 16
HEADS, DIM, MAX_TOPK = 32, 128, 4096
HEAD_COUNTS = (32, 64)  # indexer head counts the kernels take

# Every symbol include/ftk.h declares.
EXPORTS = (
    "ftk_select", "ftk_select_workspace_size", "ftk_read_info", "ftk_topk_rows",
    "ftk_score_dense", "ftk_score_dense_workspace_size", "ftk_windows_from_cu_seqlens",
    "ftk_set_stage_events", "ftk_status_string", "ftk_version", "ftk_select_noalloc",
    "ftk_block_bound", "ftk_block_bound_workspace_size", "ftk_topk_rows_end", "ftk_topk_rows_sorted",
    "ftk_rows_options_init", "ftk_topk_rows_ex", "ftk_score_dense_heads", "ftk_block_bound_heads",
    "ftk_noalloc_read_info",
)


class FtkError(RuntimeError):
    pass


class FtkConfig(ctypes.Structure):
    _fields_ = [("sample_keys", ctypes.c_int32), ("oversample", ctypes.c_float),
                ("capacity", ctypes.c_int32), ("prune", ctypes.c_int32),
                ("recovery_rows", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("dense_rows", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class FtkRowsOptions(ctypes.Structure):
    """ftk_rows_options (DeepSelect README, "Usage": sorted, indices_type,
    the out-of-bound fill values; out_stride: the output buffers' row
    stride)."""
    _fields_ = [("sorted", ctypes.c_int32), ("index_bits", ctypes.c_int32),
                ("out_stride", ctypes.c_int64), ("idx_fill", ctypes.c_int64),
                ("val_fill", ctypes.c_float)]


class FtkInfo(ctypes.Structure):
    _fields_ = [("status", ctypes.c_uint32), ("prune_enabled", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("rows_underflow", ctypes.c_int64),
                ("rows_overflow", ctypes.c_int64), ("blocks_total", ctypes.c_int64),
                ("blocks_pruned", ctypes.c_int64), ("candidates_total", ctypes.c_int64),
                ("candidates_max", ctypes.c_int64), ("kernel_launches", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_lib = None


def load_library(path: str = LIB_PATH):
    """Opens libftk.so and declares the C signatures."""
    if not os.path.exists(path):
        raise FtkError(f"{path} is not built: run `python -m sparse_attention_indexer_ftk_b200.build`")
    L = ctypes.CDLL(path)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.ftk_select.restype = I32
    L.ftk_select.argtypes = [I32, P, P, P, P, P, P, I64, I64, I32, P, P, P, SZ, P, P]
    L.ftk_select_workspace_size.restype = SZ
    L.ftk_select_workspace_size.argtypes = [I64, I64, I32, P]
    L.ftk_read_info.restype = I32
    L.ftk_read_info.argtypes = [P, P, P]
    L.ftk_topk_rows.restype = I32
    L.ftk_topk_rows.argtypes = [I32, P, I64, I64, I64, I32, P, P, P, P]
    L.ftk_score_dense.restype = I32
    L.ftk_score_dense.argtypes = [I32, P, P, P, P, P, P, I64, I64, P, I64, P, I64, P, SZ, P]
    L.ftk_score_dense_heads.restype = I32
    L.ftk_score_dense_heads.argtypes = [I32, I32, P, P, P, P, P, P, I64, I64, P, I64, P, I64, P, SZ, P]
    L.ftk_score_dense_workspace_size.restype = SZ
    L.ftk_score_dense_workspace_size.argtypes = [I64]
    L.ftk_windows_from_cu_seqlens.restype = I32
    L.ftk_windows_from_cu_seqlens.argtypes = [P, P, I64, I64, P, P, P]
    L.ftk_select_noalloc.restype = I32
    L.ftk_select_noalloc.argtypes = [I32, P, P, P, P, P, P, I64, I64, I32, P, P, P, P]
    L.ftk_noalloc_read_info.restype = I32
    L.ftk_noalloc_read_info.argtypes = [P, P]
    L.ftk_set_stage_events.restype = I32
    L.ftk_set_stage_events.argtypes = [P, I32]
    L.ftk_topk_rows_sorted.restype = I32
    L.ftk_topk_rows_sorted.argtypes = [I32, P, I64, I64, I64, P, I32, P, P, P, P]
    L.ftk_topk_rows_end.restype = I32
    L.ftk_topk_rows_end.argtypes = [I32, P, I64, I64, I64, P, I32, P, P, P, P]
    L.ftk_rows_options_init.restype = None
    L.ftk_rows_options_init.argtypes = [P]
    L.ftk_topk_rows_ex.restype = I32
    L.ftk_topk_rows_ex.argtypes = [I32, P, I64, I64, I64, P, I32, P, P, P, P, P]
    L.ftk_block_bound.restype = I32
    L.ftk_block_bound.argtypes = [I32, P, P, P, P, I64, I64, P, I64, P, SZ, P]
    L.ftk_block_bound_heads.restype = I32
    L.ftk_block_bound_heads.argtypes = [I32, I32, P, P, P, P, I64, I64, P, I64, P, SZ, P]
    L.ftk_block_bound_workspace_size.restype = SZ
    L.ftk_block_bound_workspace_size.argtypes = [I64]
    L.ftk_status_string.restype = ctypes.c_char_p
    L.ftk_status_string.argtypes = [I32]
    L.ftk_version.restype = I32
    L.ftk_version.argtypes = []
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _check(status: int, what: str):
    if status != 0:
        msg = lib().ftk_status_string(status).decode()
        raise FtkError(f"{what} failed: {msg} ({status})")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    codes = {torch.float8_e4m3fn: F8E4M3, torch.bfloat16: BF16, torch.float32: F32}
    if t.dtype not in codes:
        raise FtkError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise FtkError("inputs must be CUDA tensors")


def _config(cfg: dict | None, heads: int = HEADS):
    """ftk_config from a dict of knobs plus the indexer's head count (None:
    the library defaults)."""
    if not cfg and heads == HEADS:
        return None
    c = FtkConfig()
    for k, v in (cfg or {}).items():
        setattr(c, k, v)
    if cfg and cfg.get("heads", heads) != heads:
        raise FtkError(f"config heads={cfg['heads']} but q has {heads} heads")
    c.heads = heads
    return c


def _check_select_inputs(q, kv, weights, ks, ke, kv_scales):
    _need_cuda(q, kv, weights, ks, ke, kv_scales)
    if q.dim() != 3 or q.shape[1] not in HEAD_COUNTS or q.shape[2] != DIM or not q.is_contiguous():
        raise FtkError("q must be a contiguous [T, H, 128] tensor, H = 32 or 64")
    if kv.dim() != 2 or kv.shape[1] != DIM or not kv.is_contiguous() or kv.dtype != q.dtype:
        raise FtkError("kv must be a contiguous [S, 128] tensor of q's dtype")
    T = q.shape[0]
    if weights.shape != (T, q.shape[1]) or weights.dtype != torch.float32 or not weights.is_contiguous():
        raise FtkError("weights must be a contiguous float32 [T, H] tensor (H: q's heads)")
    for name, w in (("ks", ks), ("ke", ke)):
        if w.shape != (T,) or w.dtype != torch.int32 or not w.is_contiguous():
            raise FtkError(f"{name} must be a contiguous int32 [T] tensor")
    for t in (kv, weights, ks, ke, kv_scales):
        if t is not None and t.device != q.device:
            raise FtkError("all inputs must be on q's device")
    if kv_scales is not None and (kv_scales.shape != (kv.shape[0],) or kv_scales.dtype != torch.float32
                                  or not kv_scales.is_contiguous()):
        raise FtkError("kv_scales must be a contiguous float32 [S] tensor")


def _check_buffer(t: torch.Tensor | None, shape: tuple, dtype: torch.dtype, device: torch.device, what: str):
    """A caller-provided buffer the kernels write: exactly `shape`, `dtype`,
    contiguous and on the inputs' device (None passes)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous() or t.device != device:
        raise FtkError(f"{what} must be a contiguous {dtype} tensor of shape {list(shape)} on {device}")


def _check_workspace(ws: torch.Tensor | None, device: torch.device):
    if ws is not None and (ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous()
                           or ws.device != device):
        raise FtkError(f"workspace must be a contiguous 1-D uint8 tensor on {device}")


def _check_status(status: torch.Tensor | None, device: torch.device):
    """The status word the kernels OR bits into: a 32-bit integer tensor of
    at least one element on the inputs' device (None passes)."""
    if status is not None and (status.dtype not in (torch.int32, torch.uint32) or status.numel() < 1
                               or not status.is_contiguous() or status.device != device):
        raise FtkError(f"status must be a contiguous int32 tensor of at least one element on {device}")


def select_workspace_size(T: int, S: int, topk: int, config: dict | None = None, heads: int = HEADS) -> int:
    c = _config(config, heads)
    return int(lib().ftk_select_workspace_size(T, S, topk, ctypes.byref(c) if c else None))


def select(q, kv, weights, ks, ke, kv_scales=None, topk: int = 2048, return_scores: bool = False,
           workspace: torch.Tensor | None = None, config: dict | None = None,
           out_idx: torch.Tensor | None = None, out_val: torch.Tensor | None = None):
    """Exact top-k keys per query of I[t,s] = sigma_s sum_h w[t,h] ReLU(q[t,h].k[s]).

    Returns int32 indices [T, topk] in ascending key order (padding -1), and
    with return_scores=True also their float32 scores (padding -inf).
    """
    _check_select_inputs(q, kv, weights, ks, ke, kv_scales)
    T, S = q.shape[0], kv.shape[0]
    dev = q.device
    _check_workspace(workspace, dev)
    _check_buffer(out_idx, (T, topk), torch.int32, dev, "out_idx")
    if return_scores:
        _check_buffer(out_val, (T, topk), torch.float32, dev, "out_val")
    if workspace is None:
        workspace = torch.empty(select_workspace_size(T, S, topk, config, q.shape[1]), dtype=torch.uint8,
                                device=dev)
    if out_idx is None:
        out_idx = torch.empty((T, topk), dtype=torch.int32, device=dev)
    if return_scores and out_val is None:
        out_val = torch.empty((T, topk), dtype=torch.float32, device=dev)
    c = _config(config, q.shape[1])
    st = lib().ftk_select(_dtype_code(q), _ptr(q), _ptr(kv), _ptr(kv_scales), _ptr(weights), _ptr(ks),
                          _ptr(ke), T, S, topk, _ptr(out_idx), _ptr(out_val) if return_scores else None,
                          _ptr(workspace), workspace.numel(), ctypes.byref(c) if c else None,
                          _stream(dev))
    _check(st, "ftk_select")
    return (out_idx, out_val) if return_scores else out_idx


# Stage name -> (start event, end event), in the numbering of
# ftk_set_stage_events (event 7 marks the end of the pruning kernels).
STAGES = {"plan": (0, 1), "sample": (1, 2), "threshold": (2, 3), "prune": (3, 7), "scan": (7, 4),
          "refine": (4, 5), "recovery": (5, 6)}


class stage_events:
    """Context manager: records CUDA events at ftk_select's stage boundaries
    (diagnostic; see ftk_set_stage_events).  After synchronising, .times_ms()
    gives the duration of each stage of the last recorded call."""

    def __init__(self):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
        for e in self.events:  # torch creates the CUDA event on first record
            e.record()
        self._arr = (ctypes.c_void_p * len(self.events))(*[ctypes.c_void_p(e.cuda_event) for e in self.events])

    def __enter__(self):
        _check(lib().ftk_set_stage_events(self._arr, len(self.events)), "ftk_set_stage_events")
        return self

    def __exit__(self, *exc):
        lib().ftk_set_stage_events(None, 0)
        return False

    def times_ms(self) -> dict:
        return {name: self.events[a].elapsed_time(self.events[b]) for name, (a, b) in STAGES.items()}


def read_info(workspace: torch.Tensor) -> dict:
    """The last_info of the last select() that used this workspace (syncs)."""
    info = FtkInfo()
    _check(lib().ftk_read_info(_ptr(workspace), ctypes.byref(info), _stream(workspace.device)),
           "ftk_read_info")
    return info.as_dict()


@dataclass
class Selector:
    """Owns a workspace sized by plan(max_rows, max_kv) (FlashTopK README, "Usage")."""
    topk: int = 2048
    dtype: torch.dtype = torch.float8_e4m3fn
    config: dict | None = None
    heads: int = HEADS
    workspace: torch.Tensor | None = None
    max_rows: int = 0
    max_kv: int = 0

    def plan(self, max_rows: int, max_kv: int, device="cuda") -> "Selector":
        self.max_rows, self.max_kv = max_rows, max_kv
        nbytes = select_workspace_size(max_rows, max_kv, self.topk, self.config, self.heads)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        return self

    def run(self, q, kv, weights, ks, ke, kv_scales=None, return_scores=False, out_idx=None, out_val=None):
        if self.workspace is None:
            self.plan(q.shape[0], kv.shape[0], q.device)
        if q.shape[0] > self.max_rows or kv.shape[0] > self.max_kv:
            raise FtkError("inputs exceed the planned sizes")
        if q.dtype != self.dtype or q.shape[1] != self.heads:
            raise FtkError(f"this Selector was made for {self.dtype} inputs of {self.heads} heads, "
                           f"not {q.dtype} of {q.shape[1]}")
        return select(q, kv, weights, ks, ke, kv_scales, self.topk, return_scores,
                      workspace=self.workspace, config=self.config, out_idx=out_idx, out_val=out_val)

    @property
    def last_info(self) -> dict:
        return read_info(self.workspace)


def windows_from_cu_seqlens(cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor):
    """Causal (ks, ke) of packed sequences whose queries are their last tokens."""
    _need_cuda(cu_seqlens_q, cu_seqlens_k)
    cq = cu_seqlens_q.to(torch.int32).contiguous()
    ck = cu_seqlens_k.to(torch.int32).contiguous()
    nseq = cq.numel() - 1
    T = int(cq[-1].item())
    ks = torch.empty(T, dtype=torch.int32, device=cq.device)
    ke = torch.empty(T, dtype=torch.int32, device=cq.device)
    _check(lib().ftk_windows_from_cu_seqlens(_ptr(cq), _ptr(ck), nseq, T, _ptr(ks), _ptr(ke),
                                             _stream(cq.device)), "ftk_windows_from_cu_seqlens")
    return ks, ke


def _rows_out(given, rows: int, topk: int, dtype, device, stride: int | None, what: str):
    """A [rows, >= topk] output with a contiguous last dimension (the given
    one, checked) and its row stride; new ones get `stride` (or topk)."""
    if given is None:
        width = stride or topk
        full = torch.empty((rows, width), dtype=dtype, device=device)
        return full[:, :topk], width
    if (given.dim() != 2 or given.shape[0] != rows or given.shape[1] < topk or given.dtype != dtype
            or (given.stride(1) != 1 and given.shape[1] > 1) or given.device != device):
        raise FtkError(f"{what} must be a [{rows}, >= {topk}] {dtype} tensor on {device} with a contiguous "
                       "last dimension")
    return given, given.stride(0)


def topk_rows(x: torch.Tensor, topk: int, return_value: bool = True, status: torch.Tensor | None = None,
              out_idx: torch.Tensor | None = None, out_val: torch.Tensor | None = None,
              end: torch.Tensor | None = None, sorted: bool = False,
              indices_type: torch.dtype = torch.int32, idx_fill: int = -1, val_fill: float = float("-inf")):
    """Row top-k of a [rows, cols] bf16/fp32 CUDA tensor (ties to smaller columns).

    Returns (values, indices) like deep_select.topk, or indices alone when
    return_value=False.  Indices (int32 or int64: indices_type) come in
    ascending column order, or, with sorted=True, by value descending (ties
    by column ascending).  end: optional int32 [rows] per-row exclusive end.
    Rows shorter than topk are padded with idx_fill / val_fill (val_fill is
    stored in x's dtype).  out_idx / out_val: caller-owned outputs, [rows,
    >= topk] with a contiguous last dimension and one common row stride;
    only their first topk columns are written.  Calls ftk_topk_rows_ex.
    """
    _need_cuda(x, status, end)
    if x.dim() != 2 or x.stride(1) != 1:
        raise FtkError("x must be 2-D with a contiguous last dimension")
    if indices_type not in (torch.int32, torch.int64):
        raise FtkError("indices_type must be torch.int32 or torch.int64")
    rows, cols = x.shape
    out_idx, stride = _rows_out(out_idx, rows, topk, indices_type, x.device, None, "out_idx")
    if return_value or out_val is not None:
        out_val, vstride = _rows_out(out_val, rows, topk, x.dtype, x.device, stride, "out_val")
        if vstride != stride:
            raise FtkError("out_idx and out_val must have the same row stride")
    if end is not None and (end.shape != (rows,) or end.dtype != torch.int32 or not end.is_contiguous()
                            or end.device != x.device):
        raise FtkError("end must be a contiguous int32 [rows] tensor on x's device")
    _check_status(status, x.device)
    opt = FtkRowsOptions()
    lib().ftk_rows_options_init(ctypes.byref(opt))
    opt.sorted = 1 if sorted else 0
    opt.index_bits = 64 if indices_type == torch.int64 else 32
    opt.out_stride = stride
    opt.idx_fill = int(idx_fill)
    opt.val_fill = float(val_fill)
    st = lib().ftk_topk_rows_ex(_dtype_code(x), _ptr(x), rows, cols, x.stride(0), _ptr(end), topk,
                                ctypes.byref(opt), _ptr(out_idx), _ptr(out_val), _ptr(status),
                                _stream(x.device))
    _check(st, "ftk_topk_rows_ex")
    return (out_val, out_idx) if return_value else out_idx


def score_dense(q, kv, weights, ks, ke, kv_scales=None, rows: torch.Tensor | None = None,
                ld: int | None = None) -> torch.Tensor:
    """Fused scores of the listed rows: out[r, s - ks[t]] = I[t, s] (float32).

    Entries past a row's window are NaN.  Same kernel and bits as select().
    """
    _check_select_inputs(q, kv, weights, ks, ke, kv_scales)
    T, S = q.shape[0], kv.shape[0]
    dev = q.device
    if rows is not None:
        rows = rows.to(device=dev, dtype=torch.int32).contiguous()
    nrows = T if rows is None else rows.numel()
    if ld is None:
        ld = (S + 3) // 4 * 4
    out = torch.full((nrows, ld), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(int(lib().ftk_score_dense_workspace_size(nrows)), dtype=torch.uint8, device=dev)
    st = lib().ftk_score_dense_heads(_dtype_code(q), q.shape[1], _ptr(q), _ptr(kv), _ptr(kv_scales),
                                     _ptr(weights), _ptr(ks), _ptr(ke), T, S, _ptr(rows), nrows, _ptr(out), ld,
                                     _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ftk_score_dense_heads")
    return out


def block_bound(q, kv, weights, kv_scales=None) -> torch.Tensor:
    """Score upper bound of every row over every 128-key block:
    out[t, b] >= I[t, s] for all keys s of block b (float32, +inf for
    blocks that can never be skipped).  The bound select() prunes with."""
    _need_cuda(q, kv, weights, kv_scales)
    T, S = q.shape[0], kv.shape[0]
    dev = q.device
    nb = (S + 127) // 128
    out = torch.empty((T, nb), dtype=torch.float32, device=dev)
    ws = torch.empty(int(lib().ftk_block_bound_workspace_size(S)), dtype=torch.uint8, device=dev)
    st = lib().ftk_block_bound_heads(_dtype_code(q), q.shape[1], _ptr(q), _ptr(kv), _ptr(kv_scales),
                                     _ptr(weights), T, S, _ptr(out), nb, _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ftk_block_bound_heads")
    return out
