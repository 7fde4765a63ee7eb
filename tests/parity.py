"""Comparison rules between the CUDA path and the CPU oracle.

* Row top-k and selection on the GPU's own dumped scores: bit-exact (index
  set and value bits).
* Fused scores: |I_gpu - I_oracle| <= 1e-4 * E with
  E = sigma_s * sum_h |w[t,h]| * sum_d |q[t,h,d] k[s,d]| (the tolerance the
  accuracy target states).
* Index sets against the fp64 oracle: equal except for swaps among keys
  whose exact score lies within the band 1e-4 * (E_s + E_k) of the oracle's
  k-th score.
"""
from __future__ import annotations

import numpy as np
import torch

SCORE_RTOL = 1e-4


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def check_row_invariants(idx: np.ndarray, ks: int, ke: int, k: int):
    """Distinct, ascending, inside [ks, ke), min(k, L) real entries then -1."""
    L = max(0, ke - ks)
    n = min(k, L)
    real = idx[:n]
    assert np.all(idx[n:] == -1), "padding must be -1"
    assert np.all(real >= ks) and np.all(real < ke), "index outside the window"
    assert np.all(np.diff(real) > 0), "indices must be distinct and ascending"


def check_scores_close(gpu: np.ndarray, I64: np.ndarray, E: np.ndarray, what: str = ""):
    err = np.abs(gpu.astype(np.float64) - I64)
    bound = SCORE_RTOL * E
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {bad.sum()} scores outside 1e-4*E; worst |dI|/E = "
        f"{np.max(err / np.maximum(E, 1e-300)):.3e}")
    return float(np.max(err / np.maximum(E, 1e-300))) if err.size else 0.0


def check_against_fp64(gpu_idx: np.ndarray, gpu_val: np.ndarray | None, I64: np.ndarray,
                       E: np.ndarray, ks: int, k: int):
    """One row: the GPU set against the exact fp64 top-k, up to band swaps.

    I64 / E are the row's window (length L).  Returns the overlap p
    (|GPU set & exact set| / n).
    """
    L = I64.shape[0]
    n = min(k, L)
    got = gpu_idx[:n].astype(np.int64) - ks
    order = np.lexsort((np.arange(L), -I64))
    exact = order[:n]
    if n == 0:
        return 1.0
    vk = I64[exact[-1]]
    ek = E[exact[-1]]
    gs, es = set(got.tolist()), set(exact.tolist())
    for s in gs ^ es:
        assert abs(I64[s] - vk) <= SCORE_RTOL * (E[s] + ek), (
            f"key {s + ks} differs from the exact top-k outside the tie band: "
            f"I={I64[s]!r}, k-th={vk!r}")
    if gpu_val is not None:
        check_scores_close(gpu_val[:n], I64[got], E[got], "selected scores")
        assert np.all(np.isneginf(gpu_val[n:]))
    return len(gs & es) / n


def check_exact_vs_dump(gpu_idx: np.ndarray, gpu_val: np.ndarray | None, oidx: np.ndarray,
                        oval: np.ndarray, k: int):
    """One row: GPU selection equals the oracle's selection of the GPU's own
    dumped fp32 scores, bit for bit (oracle rows come in score order)."""
    n = int(np.sum(oidx >= 0))
    order = np.argsort(oidx[:n], kind="stable")
    want_idx = oidx[:n][order]
    assert np.array_equal(gpu_idx[:n].astype(np.int64), want_idx), "index sets differ"
    assert np.all(gpu_idx[n:] == -1)
    if gpu_val is not None:
        want_val = oval[:n][order].astype(np.float32)
        assert np.array_equal(gpu_val[:n].view(np.uint32), want_val.view(np.uint32)), "values differ"
