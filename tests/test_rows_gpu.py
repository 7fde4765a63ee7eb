"""ftk_topk_rows against the oracle: bit-exact index sets and values."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from sparse_attention_indexer_ftk_b200 import ftk
from sparse_attention_indexer_ftk_b200 import workloads as wl
from tests.parity import check_row_invariants, to_np

pytestmark = pytest.mark.gpu


def aligned_rows(x_cpu: torch.Tensor) -> torch.Tensor:
    """x on the GPU with its row stride padded to a 16-byte multiple (the
    row-alignment requirement; DeepSelect README, "Usage")."""
    rows, cols = x_cpu.shape
    per = 16 // x_cpu.element_size()
    ld = (cols + per - 1) // per * per
    buf = torch.zeros((rows, ld), dtype=x_cpu.dtype, device="cuda")
    buf[:, :cols] = x_cpu.cuda()
    return buf[:, :cols]


def run_and_compare(x_cpu: torch.Tensor, k: int, return_value=True, rows_subset=None):
    x = aligned_rows(x_cpu)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = ftk.topk_rows(x, k, return_value=return_value, status=status)
    torch.cuda.synchronize()
    if return_value:
        val, idx = res
    else:
        val, idx = None, res
    idx = to_np(idx)
    rows = range(x_cpu.shape[0]) if rows_subset is None else rows_subset
    xs = x_cpu[list(rows)]
    oidx, oval, flags = orc.topk_rows(xs, k)
    for r_out, r in enumerate(rows):
        check_row_invariants(idx[r], 0, x_cpu.shape[1], k)
        n = min(k, x_cpu.shape[1])
        want = np.sort(oidx[r_out, :n])
        assert np.array_equal(idx[r, :n], want), f"row {r}: index set differs"
        if val is not None:
            got = val[r, :n].float().cpu().numpy().astype(np.float64)
            # values in column order = x at those columns (bit-exact)
            ref = x_cpu[r, idx[r, :n]]
            assert torch.equal(val[r, :n].cpu().view(torch.int16 if x.dtype == torch.bfloat16 else torch.int32),
                               ref.view(torch.int16 if x.dtype == torch.bfloat16 else torch.int32))
            assert np.array_equal(np.sort(got), np.sort(oval[r_out, :n]))
    return int(status.item())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols,k", [(1, 1, 1), (3, 7, 5), (5, 100, 100), (4, 1000, 37),
                                         (2, 5000, 4096), (9, 33333, 512), (300, 2048, 64),
                                         (1, 393216, 4096), (2, 131072, 1),
                                         (1000, 3000, 64)])  # more rows than resident clusters
def test_random_rows(dtype, rows, cols, k):
    g = torch.Generator().manual_seed(rows * 1000 + cols + k)
    x = torch.randn((rows, cols), generator=g).to(dtype)
    assert run_and_compare(x, k) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols,k", [(3, 131072, 512), (4, 40000, 2048), (600, 5000, 100)])
def test_structured_rows(dtype, rows, cols, k):
    """Rows whose largest values crowd one part of the row (sorted
    descending, sorted ascending, one hot block): the sampled threshold
    misses the k-th value or a candidate list overflows, and the exact
    fallback gives the oracle's result.  With 600 rows (one CTA per row,
    the next row's stages already in flight) the fallback first drains
    them."""
    g = torch.Generator().manual_seed(rows + cols + k)
    x = torch.randn((rows, cols), generator=g)
    for r in range(0, rows, 3):
        x[r] = torch.sort(x[r], descending=True).values
    for r in range(1, rows, 3):
        x[r] = torch.sort(x[r]).values
    for r in range(2, rows, 3):
        x[r, (r * 97) % (cols // 2): (r * 97) % (cols // 2) + cols // 8] += 6.0
    assert run_and_compare(x.to(dtype), k) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantized_rows(dtype):
    """Values on a grid of quarters (hundreds of equal values around the
    k-th): some candidate lists overflow with values above the sample
    threshold, and those rows take the exact fallback, whose passes skip
    every key below the threshold once the row has topk keys at or above
    it."""
    g = torch.Generator().manual_seed(3)
    x = (torch.randn((256, 131072), generator=g) * 4).round() / 4
    assert run_and_compare(x.to(dtype), 512) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_heavy_ties_and_signed_zero(dtype):
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-2, 3, (8, 20000), generator=g).float() * 0.5
    x[1] = 0.0
    x[2, ::2] = -0.0
    x[3] = 1.0
    x[4, :] = torch.tensor(float("-inf"))
    x[4, 100:110] = 3.0
    x = x.to(dtype)
    for k in (1, 7, 511, 512, 4096):
        assert run_and_compare(x, k) == 0


def test_return_value_false_and_determinism():
    x = torch.randn((16, 50000), generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    run_and_compare(x, 512, return_value=False)
    xg = aligned_rows(x)
    a = ftk.topk_rows(xg, 512)
    b = ftk.topk_rows(xg, 512)
    assert torch.equal(a[1], b[1]) and torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))


def test_row_stride_padding():
    base = torch.randn((6, 1032), generator=torch.Generator().manual_seed(7))
    x = base[:, :1000]  # row stride 1032 floats (16-byte multiple), last dim contiguous
    val, idx = ftk.topk_rows(x.cuda(), 50)
    oidx, _, _ = orc.topk_rows(x.contiguous(), 50)
    for r in range(6):
        assert np.array_equal(to_np(idx[r]), np.sort(oidx[r]))


def test_nan_is_flagged_not_trapped():
    x = torch.randn((4, 3000), generator=torch.Generator().manual_seed(8))
    x[2, 17] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ftk.topk_rows(aligned_rows(x), 16, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & ftk.STATUS_NAN


@pytest.mark.parametrize("name", ["rows_bf16", "rows_f32"])
def test_full_size_workload(name):
    """The row top-k workload at full size (64 rows), every row bit-exact."""
    c = wl.get(name)
    assert run_and_compare(c.x, c.topk) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_variable_length_rows_end(dtype):
    """ftk_topk_rows_end: row r is x[r, :end[r]] (end clamped to [0, cols]),
    short rows padded with (-1, -inf) (DeepSelect README, "Variable-length
    rows"); compared row by row with the oracle on the truncated rows."""
    rows, cols, k = 40, 20000, 300
    g = torch.Generator().manual_seed(77)
    x_cpu = torch.randn((rows, cols), generator=g).to(dtype)
    ends = torch.randint(0, cols + 1, (rows,), generator=g).to(torch.int32)
    ends[:6] = torch.tensor([0, 1, k - 1, k, k + 1, cols], dtype=torch.int32)
    ends[6] = cols + 500   # beyond the row: clamped to cols
    ends[7] = -3           # negative: an empty row
    x = aligned_rows(x_cpu)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    val, idx = ftk.topk_rows(x, k, status=status, end=ends.cuda())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx, val = to_np(idx), val.cpu()
    for r in range(rows):
        e = max(0, min(int(ends[r]), cols))
        check_row_invariants(idx[r], 0, e, k)
        n = min(k, e)
        if n:
            oidx, _, _ = orc.topk_rows(x_cpu[r:r + 1, :e].contiguous(), k)
            assert np.array_equal(idx[r, :n], np.sort(oidx[0, :n])), f"row {r}"
            ref = x_cpu[r, idx[r, :n]]
            bits = torch.int16 if dtype == torch.bfloat16 else torch.int32
            assert torch.equal(val[r, :n].view(bits), ref.view(bits))
        assert np.all(idx[r, n:] == -1)
        assert torch.all(torch.isneginf(val[r, n:].float()))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sorted_output(dtype):
    """sorted=True (DeepSelect README, "Usage"): each row's topk by value
    descending, ties by column ascending, padding last -- element by element
    the oracle's order, values bit-exact (signed zeros kept)."""
    rows, cols, k = 24, 9000, 700
    g = torch.Generator().manual_seed(91)
    x_cpu = torch.randn((rows, cols), generator=g).to(dtype)
    x_cpu[3] = torch.randint(0, 4, (cols,), generator=g).to(dtype) - 1.5  # 4 values: heavy ties
    x_cpu[4] = 0.0
    x_cpu[4, ::3] = -0.0                                                 # signed zeros only
    ends = torch.full((rows,), cols, dtype=torch.int32)
    ends[5], ends[6] = 100, 0                                            # short and empty rows
    x = aligned_rows(x_cpu)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    val, idx = ftk.topk_rows(x, k, status=status, end=ends.cuda(), sorted=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx, val = to_np(idx), val.cpu()
    bits = torch.int16 if dtype == torch.bfloat16 else torch.int32
    for r in range(rows):
        e = int(ends[r])
        n = min(k, e)
        if n:
            oidx, _, _ = orc.topk_rows(x_cpu[r:r + 1, :e].contiguous(), k)
            assert np.array_equal(idx[r, :n], oidx[0, :n]), f"row {r}: order differs"
            ref = x_cpu[r, idx[r, :n]]
            assert torch.equal(val[r, :n].view(bits), ref.view(bits)), f"row {r}: value bits"
        assert np.all(idx[r, n:] == -1)
        assert torch.all(torch.isneginf(val[r, n:].float()))


def _options_case(dtype, seed):
    """Rows with short, empty and full lengths, heavy ties and signed zeros."""
    rows, cols, k = 20, 7000, 500
    g = torch.Generator().manual_seed(seed)
    x_cpu = torch.randn((rows, cols), generator=g).to(dtype)
    x_cpu[2] = torch.randint(0, 4, (cols,), generator=g).to(dtype) - 1.5
    x_cpu[3] = 0.0
    x_cpu[3, ::5] = -0.0
    ends = torch.full((rows,), cols, dtype=torch.int32)
    ends[4], ends[5], ends[6], ends[7] = 0, 1, k - 1, 37
    return x_cpu, ends, k


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("sorted_", [False, True])
def test_int64_indices_fill_values_and_output_stride(dtype, sorted_):
    """indices_type=int64, idx_oob_fill_value / value_oob_fill_value and a
    caller-owned output with a row stride (DeepSelect README, "Usage" and
    "Variable-length rows").  The fill value 0.5 lies inside the rows'
    values, so a sort that let padding move would misplace it.  Each row
    equals the oracle (order included when sorted); padding holds the fills;
    columns past topk keep their contents."""
    x_cpu, ends, k = _options_case(dtype, 123)
    rows, cols = x_cpu.shape
    x = aligned_rows(x_cpu)
    width = k + 13
    idx_buf = torch.full((rows, width), 4242, dtype=torch.int64, device="cuda")
    val_buf = torch.full((rows, width), 7.0, dtype=dtype, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    val, idx = ftk.topk_rows(x, k, status=status, end=ends.cuda(), sorted=sorted_, indices_type=torch.int64,
                             idx_fill=-(1 << 40), val_fill=0.5, out_idx=idx_buf, out_val=val_buf)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert idx.dtype == torch.int64 and idx.data_ptr() == idx_buf.data_ptr()
    bits = torch.int16 if dtype == torch.bfloat16 else torch.int32
    idx_all, val_all = idx_buf.cpu(), val_buf.cpu()
    assert torch.all(idx_all[:, k:] == 4242) and torch.all(val_all[:, k:] == 7.0)
    for r in range(rows):
        e = int(ends[r])
        n = min(k, e)
        got = idx_all[r, :k].numpy()
        if n:
            oidx, _, _ = orc.topk_rows(x_cpu[r:r + 1, :e].contiguous(), k)
            want = oidx[0, :n] if sorted_ else np.sort(oidx[0, :n])
            assert np.array_equal(got[:n], want.astype(np.int64)), f"row {r}"
            ref = x_cpu[r, torch.from_numpy(got[:n])]
            assert torch.equal(val_all[r, :n].view(bits), ref.view(bits)), f"row {r}: value bits"
        assert np.all(got[n:] == -(1 << 40))
        assert torch.all(val_all[r, n:k] == 0.5)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sorted_without_values_reads_x(dtype):
    """sorted=True with return_value=False: the sort takes each selected
    value from x; the order equals the sorted call with values."""
    x_cpu, ends, k = _options_case(dtype, 321)
    x = aligned_rows(x_cpu)
    _, want = ftk.topk_rows(x, k, end=ends.cuda(), sorted=True)
    got = ftk.topk_rows(x, k, end=ends.cuda(), sorted=True, return_value=False)
    assert torch.equal(got, want)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fixed_entry_points_equal_the_options_call(dtype):
    """ftk_topk_rows, ftk_topk_rows_end and ftk_topk_rows_sorted give the
    same bits as ftk_topk_rows_ex with the matching options."""
    import ctypes
    x_cpu, ends, k = _options_case(dtype, 555)
    rows, cols = x_cpu.shape
    x = aligned_rows(x_cpu)
    end_d = ends.cuda()
    L = ftk.lib()
    code = ftk.BF16 if dtype == torch.bfloat16 else ftk.F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731

    def fresh():
        return (torch.full((rows, k), 99, dtype=torch.int32, device="cuda"),
                torch.full((rows, k), 3.0, dtype=dtype, device="cuda"))

    i0, v0 = fresh()
    assert L.ftk_topk_rows(code, P(x), rows, cols, x.stride(0), k, P(i0), P(v0), None, stream) == 0
    v, i = ftk.topk_rows(x, k)
    assert torch.equal(i0, i) and torch.equal(v0.view(torch.uint8), v.contiguous().view(torch.uint8))
    i1, v1 = fresh()
    assert L.ftk_topk_rows_end(code, P(x), rows, cols, x.stride(0), P(end_d), k, P(i1), P(v1), None,
                               stream) == 0
    v, i = ftk.topk_rows(x, k, end=end_d)
    assert torch.equal(i1, i) and torch.equal(v1.view(torch.uint8), v.contiguous().view(torch.uint8))
    i2, v2 = fresh()
    assert L.ftk_topk_rows_sorted(code, P(x), rows, cols, x.stride(0), P(end_d), k, P(i2), P(v2), None,
                                  stream) == 0
    v, i = ftk.topk_rows(x, k, end=end_d, sorted=True)
    assert torch.equal(i2, i) and torch.equal(v2.view(torch.uint8), v.contiguous().view(torch.uint8))
