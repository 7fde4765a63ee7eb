"""Host-side logic that needs no GPU: the bench's reading of the committed
ncu summary, and the seeded workload generators."""
from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_attention_indexer_ftk_b200 import workloads as wl  # noqa: E402


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    good = tmp_path / "ok.md"
    good.write_text(f"traffic_bytes_per_launch: 1234\nkernel_source_hash: {bench.scan_kernel_hash()}\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(good))
    assert bench.profiled_traffic() == 1234.0
    stale = tmp_path / "stale.md"
    stale.write_text("traffic_bytes_per_launch: 1234\nkernel_source_hash: 000000000000\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(stale))
    assert bench.profiled_traffic() is None  # counters of another kernel source are not reported
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "missing.md"))
    assert bench.profiled_traffic() is None


def test_generators_are_seeded_and_shaped():
    a = wl.small_case(seed=3, dtype="fp8", T=9, S=500, topk=16, windows="random")
    b = wl.small_case(seed=3, dtype="fp8", T=9, S=500, topk=16, windows="random")
    assert torch.equal(a.q.view(torch.uint8), b.q.view(torch.uint8))
    assert torch.equal(a.ks, b.ks) and torch.equal(a.ke, b.ke)
    assert a.q.shape == (9, 32, 128) and a.kv.shape == (500, 128) and a.weights.shape == (9, 32)
    assert bool(torch.all((a.ks >= 0) & (a.ks <= a.ke) & (a.ke <= 500)))


def test_block_structured_keys():
    c = wl.block_structured(seed=5, dtype="bf16", T=4, S=1000, topk=8)
    base = wl.small_case(seed=5, dtype="bf16", T=4, S=1000, topk=8, windows="causal")
    blk = torch.arange(1000) // 128
    hot = blk % 8 == 0
    assert torch.equal(c.kv_scales[hot], base.kv_scales[hot])
    assert torch.allclose(c.kv_scales[~hot], base.kv_scales[~hot] * 2.0 ** -7)
    assert bool(torch.all(c.weights[:, 1:8] >= 0)) and bool(torch.all(c.weights[:, ::8] <= 0))


def test_binding_rejects_buffers_the_kernels_would_overrun():
    """Caller-provided outputs, workspaces and status words are checked in
    the binding before any pointer reaches the library (CPU tensors stand in
    for device ones: the checks compare shapes, dtypes, layout, devices)."""
    import pytest
    from sparse_attention_indexer_ftk_b200 import ftk
    cpu = torch.device("cpu")
    ok = torch.empty((5, 7), dtype=torch.int32)
    ftk._check_buffer(ok, (5, 7), torch.int32, cpu, "out_idx")
    ftk._check_buffer(None, (5, 7), torch.int32, cpu, "out_idx")
    for bad in (torch.empty((5, 6), dtype=torch.int32), torch.empty((4, 7), dtype=torch.int32),
                torch.empty((5, 7), dtype=torch.int64), torch.empty((7, 5), dtype=torch.int32).t(),
                torch.empty(35, dtype=torch.int32)):
        with pytest.raises(ftk.FtkError):
            ftk._check_buffer(bad, (5, 7), torch.int32, cpu, "out_idx")
    ftk._check_workspace(torch.empty(100, dtype=torch.uint8), cpu)
    for bad in (torch.empty(100, dtype=torch.float32), torch.empty((10, 10), dtype=torch.uint8),
                torch.empty(200, dtype=torch.uint8)[::2]):
        with pytest.raises(ftk.FtkError):
            ftk._check_workspace(bad, cpu)
    ftk._check_status(torch.zeros(1, dtype=torch.int32), cpu)
    ftk._check_status(None, cpu)
    for bad in (torch.zeros(0, dtype=torch.int32), torch.zeros(1, dtype=torch.int16),
                torch.zeros(1, dtype=torch.float32)):
        with pytest.raises(ftk.FtkError):
            ftk._check_status(bad, cpu)
    with pytest.raises(ftk.FtkError):
        ftk._check_status(torch.zeros(1, dtype=torch.int32), torch.device("cuda", 0))


class _FakeLib:
    """Stands in for libftk: records calls, returns FTK_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 1024 if name.endswith("workspace_size") else 0
        return fn


def test_binding_accepts_the_calls_bench_and_tests_make(monkeypatch):
    """select(), Selector.run() and topk_rows() with conforming buffers (the
    patterns bench.py and the GPU tests use) pass the binding's checks and
    reach the library; CPU tensors and a fake library stand in for the GPU."""
    import pytest
    from sparse_attention_indexer_ftk_b200 import ftk
    fake = _FakeLib()
    monkeypatch.setattr(ftk, "lib", lambda: fake)
    monkeypatch.setattr(ftk, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(ftk, "_stream", lambda dev: None)
    c = wl.small_case(seed=3, dtype="fp8", T=9, S=300, topk=16, windows="causal")
    T, k = c.T, c.topk
    ws = torch.empty(ftk.select_workspace_size(T, c.S, k), dtype=torch.uint8)
    oi = torch.empty((T, k), dtype=torch.int32)
    ov = torch.empty((T, k), dtype=torch.float32)
    ftk.select(c.q, c.kv, c.weights, c.ks, c.ke, c.kv_scales, k, return_scores=True, workspace=ws,
               out_idx=oi, out_val=ov)
    ftk.select(c.q, c.kv, c.weights, c.ks, c.ke, c.kv_scales, k, return_scores=True, workspace=ws,
               config={"prune": 1})
    ftk.select(c.q, c.kv, c.weights, c.ks, c.ke, None, k)
    sel = ftk.Selector(topk=k, dtype=torch.float8_e4m3fn).plan(32, 8000, device="cpu")
    sel.run(c.q, c.kv, c.weights, c.ks, c.ke, c.kv_scales)
    assert fake.calls.count("ftk_select") == 4
    with pytest.raises(ftk.FtkError):
        ftk.select(c.q, c.kv, c.weights, c.ks, c.ke, c.kv_scales, k, out_idx=oi[:, :-1])
    with pytest.raises(ftk.FtkError):
        ftk.Selector(topk=k, dtype=torch.bfloat16).plan(32, 8000, device="cpu").run(
            c.q, c.kv, c.weights, c.ks, c.ke, c.kv_scales)
    x = torch.randn(6, 1000).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32)
    end = torch.full((6,), 500, dtype=torch.int32)
    xi = torch.empty((6, 64), dtype=torch.int32)
    xv = torch.empty((6, 64), dtype=torch.bfloat16)
    ftk.topk_rows(x, 64, out_idx=xi, out_val=xv)
    ftk.topk_rows(x, 64, status=st, end=end, sorted=True)
    ftk.topk_rows(x, 64, return_value=False)
    val, idx = ftk.topk_rows(x, 64, end=end, indices_type=torch.int64, idx_fill=-5, val_fill=0.0,
                             out_idx=torch.empty((6, 70), dtype=torch.int64))
    assert val.shape == (6, 64) and val.stride(0) == 70 and idx.dtype == torch.int64
    assert fake.calls.count("ftk_topk_rows_ex") == 4


def test_clock_summary(tmp_path):
    """The clock record beside every bench number: median SM clock under
    load, the max clock, and the throttle reasons seen in any sample."""
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("0, 1965, 1965, 800.5, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("0, 1800, 1965, 1001.2, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("garbage line\n")
        f.write("0, 1900, 1965, [N/A], 0x0, Not Active, Not Active, Not Active, Not Active\n")
    out = s.summary()
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 1001.2
    assert not os.path.exists(s.path)
    s.path = str(tmp_path / "none.csv")
    with open(s.path, "w") as f:
        f.write("0, 1965, 1965, [N/A], 0x0, Not Active, Active, Not Active, Not Active\n")
    out = s.summary()
    assert out["power_w_max"] is None and out["reasons"] == ["hw_thermal_slowdown"]
    s.path = str(tmp_path / "missing.csv")
    assert s.summary()["reasons"] == ["unsampled"]
