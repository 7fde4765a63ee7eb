"""The oracle under AddressSanitizer and UndefinedBehaviorSanitizer: a
sanitized build of oracle/oracle.c runs every pin of tests/test_oracle.py
plus edge sizes (one key, 64 heads, topk above the window, bound rows
outside the batch) in a child process; any out-of-bounds access or
undefined behaviour fails the test."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RUNNER = r'''
import inspect, sys
sys.path.insert(0, ROOT)
import torch
from oracle import oracle as orc
from sparse_attention_indexer_ftk_b200 import workloads as wl
from tests import test_oracle as pins
with orc.use_library(LIB):
    n = 0
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("check_"):
            continue
        params = inspect.signature(fn).parameters
        if "dtype" in params:
            for dt in ("fp8", "bf16"):
                fn(dt)
                n += 1
        elif not params:
            fn()
            n += 1
    for spec in [dict(seed=1, dtype="fp8", T=3, S=1, topk=5, windows="causal"),
                 dict(seed=2, dtype="bf16", T=4, S=300, topk=4096, windows="random", heads=64),
                 dict(seed=3, dtype="fp8", T=6, S=500, topk=16, windows="empty_mix")]:
        c = wl.small_case(**spec)
        orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk)
        orc.index_scores(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke)
        orc.block_bound(c.q, c.kv, c.kv_scales, c.weights, rows=[0, c.T - 1, c.T, -1])
    x = torch.randn(3, 777)
    orc.topk_rows(x, 1000)
    orc.topk_rows(x.to(torch.bfloat16), 5)
    print("clean", n)
'''


def _runtime(name: str) -> str | None:
    p = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


def test_oracle_is_clean_under_asan_and_ubsan(tmp_path):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not (asan and ubsan):
        pytest.skip("gcc sanitizer runtimes not available")
    lib = tmp_path / "liboracle_sanitized.so"
    subprocess.check_call(["gcc", "-O1", "-g", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fsanitize=address,undefined", "-fno-omit-frame-pointer",
                           "-o", str(lib), os.path.join(ROOT, "oracle", "oracle.c"), "-lm"])
    env = dict(os.environ, LD_PRELOAD=f"{asan}:{ubsan}", ASAN_OPTIONS="detect_leaks=0:halt_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1", OMP_NUM_THREADS="4")
    code = f"ROOT = {ROOT!r}\nLIB = {str(lib)!r}\n" + RUNNER
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and "clean" in out.stdout, (out.stdout[-2000:], out.stderr[-4000:])
