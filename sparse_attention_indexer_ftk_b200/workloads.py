"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and lays out windows: it holds none of
the method's arithmetic (no scoring, no selection).  Both the CPU oracle's
tests and the CUDA path are fed from here, so the two always see the same
bytes.  Every generator runs on the CPU with a ``torch.Generator`` seeded
with ``SEED_BASE + workload number``; draws happen in a fixed order
(q, kv, kv_scales, weights, then extras).

Workloads (sizes as in the FlashTopK README "Quick start" example and the
DeepSelect README "Supported Cases" / "Performance"):

1. ``bf16_small``     BF16 indexer, q [128,32,128], kv [2048,128] ~ N(0,1),
                      weights N(0,1)/sqrt(32), no kv_scales, causal windows
                      ke[t] = 1920 + t + 1, topk 256; plus ``bf16_ties``
                      (8 rows, keys copied from 16 prototypes with entries in
                      {-1.5,-0.5,0.5,1.5}, so tie groups straddle the k-th
                      score) and ``bf16_all_equal`` (constant keys).
2. ``rows_bf16``      row top-k, BF16 [64,131072] ~ N(0,1), topk 512;
   ``rows_f32``       FP32 [64,129280] = N(0, variance 2) + Gumbel noise,
                      rows 48..63 drawn from 8 distinct values, topk 512.
3. ``fp8_prefill``    FP8-e4m3 q [4096,32,128], kv [131072,128] ~ N(0,1),
                      kv_scales in (0.5,1], weights N(0,1)/sqrt(32), causal
                      ke[t] = 126976 + t + 1, topk 2048.
4. ``fp8_packed``     4 packed sequences x 32768 keys, the last 1024 tokens
                      of each sequence are queries (causal windows), keys and
                      queries carry a rank-8 component on 64 sink tokens and
                      the 1024-token local band, topk 2048.
5. ``fp8_large``      FP8 q [8192,32,128], kv [262144,128], causal
                      ke[t] = 253952 + t + 1, topk 4096.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SEED_BASE = 20261202

WORKLOADS = ("bf16_small", "rows_bf16", "fp8_prefill", "fp8_packed", "fp8_large")


@dataclass
class SelectInputs:
    """Inputs of one fused score + top-k call (CPU tensors)."""
    name: str
    q: torch.Tensor            # [T, 32, 128] float8_e4m3fn or bfloat16
    kv: torch.Tensor           # [S, 128] same dtype as q
    kv_scales: torch.Tensor | None  # [S] float32 or None (all ones)
    weights: torch.Tensor      # [T, 32] float32
    ks: torch.Tensor           # [T] int32
    ke: torch.Tensor           # [T] int32
    topk: int
    extra: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    @property
    def S(self) -> int:
        return int(self.kv.shape[0])

    def pairs(self) -> int:
        """Number of (query, key) pairs inside the windows."""
        return int((self.ke.to(torch.int64) - self.ks.to(torch.int64)).clamp(min=0).sum())

    def to(self, device) -> "SelectInputs":
        mv = lambda t: None if t is None else t.to(device)
        return SelectInputs(self.name, mv(self.q), mv(self.kv), mv(self.kv_scales),
                            mv(self.weights), mv(self.ks), mv(self.ke), self.topk,
                            dict(self.extra))


@dataclass
class RowsInputs:
    """Inputs of one row top-k call (CPU tensors)."""
    name: str
    x: torch.Tensor            # [rows, cols] bfloat16 or float32
    topk: int


def _gen(n: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(SEED_BASE + n)
    return g


def _normal(g, shape, std=1.0):
    return torch.randn(shape, generator=g, dtype=torch.float32) * std


def _scales(g, S):
    # 1 - U[0,1) lies in (0.5, 1] after halving the draw.
    return 1.0 - 0.5 * torch.rand(S, generator=g, dtype=torch.float32)


def _weights(g, T, H=32):
    return _normal(g, (T, H)) / math.sqrt(H)


def causal_windows(T: int, S: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Queries are the last T tokens: query i sees keys [0, S - T + i + 1)."""
    ke = torch.arange(S - T + 1, S + 1, dtype=torch.int32)
    return torch.zeros_like(ke), ke


def packed_causal_windows(q_lens, k_lens) -> tuple[torch.Tensor, torch.Tensor]:
    """Causal windows of packed sequences whose queries are the last tokens."""
    ks, ke = [], []
    k0 = 0
    for nq, nk in zip(q_lens, k_lens):
        for i in range(nq):
            ks.append(k0)
            ke.append(k0 + nk - nq + i + 1)
        k0 += nk
    return torch.tensor(ks, dtype=torch.int32), torch.tensor(ke, dtype=torch.int32)


# ---------------------------------------------------------------------------
# Workload 1: BF16 small
# ---------------------------------------------------------------------------

def bf16_small() -> SelectInputs:
    g = _gen(1)
    T, S = 128, 2048
    q = _normal(g, (T, 32, 128)).to(torch.bfloat16)
    kv = _normal(g, (S, 128)).to(torch.bfloat16)
    w = _weights(g, T)
    ks = torch.zeros(T, dtype=torch.int32)
    ke = torch.arange(1920 + 1, 1920 + T + 1, dtype=torch.int32)
    return SelectInputs("bf16_small", q, kv, None, w, ks, ke, 256)


def bf16_ties() -> SelectInputs:
    """8 rows whose keys repeat 16 prototypes with entries from 4 levels.

    Identical keys give identical scores, so the 256th score lies inside a
    group of equal scores and the tie rule decides the result.
    """
    g = _gen(1)
    torch.randn((1,), generator=g)  # keep this stream distinct from bf16_small's
    T, S, P = 8, 2048, 16
    levels = torch.tensor([-1.5, -0.5, 0.5, 1.5])
    qi = torch.randint(0, 4, (T, 32, 128), generator=g)
    pi = torch.randint(0, 4, (P, 128), generator=g)
    q = levels[qi].to(torch.bfloat16)
    proto = levels[pi]
    kv = proto[torch.arange(S) % P].to(torch.bfloat16)
    w = _weights(g, T)
    ks = torch.zeros(T, dtype=torch.int32)
    ke = torch.arange(S - T + 1, S + 1, dtype=torch.int32)
    return SelectInputs("bf16_ties", q, kv, None, w, ks, ke, 256)


def bf16_all_equal() -> SelectInputs:
    """Constant keys: every score of a row is equal."""
    g = _gen(1)
    T, S = 2, 512
    q = _normal(g, (T, 32, 128)).to(torch.bfloat16)
    kv = torch.full((S, 128), 0.5).to(torch.bfloat16)
    w = _weights(g, T)
    ks = torch.tensor([3, 0], dtype=torch.int32)
    ke = torch.tensor([400, 512], dtype=torch.int32)
    return SelectInputs("bf16_all_equal", q, kv, None, w, ks, ke, 64)


# ---------------------------------------------------------------------------
# Workload 2: row top-k
# ---------------------------------------------------------------------------

def rows_bf16() -> RowsInputs:
    g = _gen(2)
    x = _normal(g, (64, 131072)).to(torch.bfloat16)
    return RowsInputs("rows_bf16", x, 512)


def rows_bf16_1024() -> RowsInputs:
    """A scaled-up copy of rows_bf16 (1024 rows, 268 MB): not one of the
    pages' configurations; it shows the row kernel where HBM bandwidth, not
    launch and phase latency, decides."""
    g = _gen(12)
    x = _normal(g, (1024, 131072)).to(torch.bfloat16)
    return RowsInputs("rows_bf16_1024", x, 512)


def rows_f32() -> RowsInputs:
    g = _gen(2)
    torch.randn((1,), generator=g)
    rows, cols = 64, 129280
    x = _normal(g, (rows, cols), std=math.sqrt(2.0))
    u = torch.rand((rows, cols), generator=g, dtype=torch.float64)
    u = u.clamp(min=1e-300, max=1.0 - 1e-16)
    gumbel = (-torch.log(-torch.log(u))).to(torch.float32)
    x = x + gumbel
    distinct = _normal(g, (8,)) * 3.0
    pick = torch.randint(0, 8, (16, cols), generator=g)
    x[48:64] = distinct[pick]
    return RowsInputs("rows_f32", x.contiguous(), 512)


# ---------------------------------------------------------------------------
# Workloads 3-5: FP8 prefill
# ---------------------------------------------------------------------------

def _fp8(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float8_e4m3fn)


def fp8_causal(n: int, name: str, T: int, S: int, topk: int, heads: int = 32) -> SelectInputs:
    g = _gen(n)
    q = _fp8(_normal(g, (T, heads, 128)))
    kv = _fp8(_normal(g, (S, 128)))
    sc = _scales(g, S)
    w = _weights(g, T, heads)
    ks, ke = causal_windows(T, S)
    return SelectInputs(name, q, kv, sc, w, ks, ke, topk)


def fp8_prefill() -> SelectInputs:
    return fp8_causal(3, "fp8_prefill", 4096, 131072, 2048)


def fp8_large() -> SelectInputs:
    return fp8_causal(5, "fp8_large", 8192, 262144, 4096)


def fp8_prefill_64h() -> SelectInputs:
    """The fp8_prefill shape for a 64-head indexer (FlashTopK README,
    "Roadmap": other head counts such as 64): q [4096, 64, 128], weights
    N(0,1)/sqrt(64)."""
    return fp8_causal(6, "fp8_prefill_64h", 4096, 131072, 2048, heads=64)


def fp8_packed(gamma: float = 6.0) -> SelectInputs:
    """Packed sequences with a concentrated (trained-indexer-like) top-k.

    Each sequence j has a unit direction u_j in a fixed rank-8 subspace.
    Its 64 sink keys and its last 1024 keys (the local band, where the
    queries sit) get +gamma*u_j; every query head gets
    +sign(w[t,h])*gamma*u_j, so positive-weight heads score high on those keys.
    """
    g = _gen(4)
    nseq, L, nq = 4, 32768, 1024
    S, T = nseq * L, nseq * nq
    q = _normal(g, (T, 32, 128))
    kv = _normal(g, (S, 128))
    sc = _scales(g, S)
    w = _weights(g, T)
    basis, _ = torch.linalg.qr(_normal(g, (128, 8)).to(torch.float64))
    coef = _normal(g, (nseq, 8)).to(torch.float64)
    coef = coef / coef.norm(dim=1, keepdim=True)
    u = (coef @ basis.T).to(torch.float32)          # [nseq, 128] unit rows
    for j in range(nseq):
        k0 = j * L
        kv[k0:k0 + 64] += gamma * u[j]
        kv[k0 + L - nq:k0 + L] += gamma * u[j]
        rows = slice(j * nq, (j + 1) * nq)
        q[rows] += torch.sign(w[rows]).unsqueeze(-1) * gamma * u[j]
    ks, ke = packed_causal_windows([nq] * nseq, [L] * nseq)
    return SelectInputs("fp8_packed", _fp8(q), _fp8(kv), sc, w, ks, ke, 2048,
                        extra={"cu_seqlens_q": [j * nq for j in range(nseq + 1)],
                               "cu_seqlens_k": [j * L for j in range(nseq + 1)]})


# ---------------------------------------------------------------------------
# Small parity cases (span several tiles, ragged tails)
# ---------------------------------------------------------------------------

def small_case(seed: int, dtype: str, T: int, S: int, topk: int,
               windows: str = "causal", scales: bool = True,
               kv_levels: int = 0, heads: int = 32) -> SelectInputs:
    """A generic small case.

    windows: "causal" | "random" | "short" | "empty_mix" | "packed".
    kv_levels > 0 rounds key entries onto that many levels (forces ties).
    heads: the indexer's head count H (q [T, H, 128], weights [T, H]).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(SEED_BASE + 1000 + seed)
    q = _normal(g, (T, heads, 128))
    kv = _normal(g, (S, 128))
    sc = _scales(g, S) if scales else None
    w = _weights(g, T, heads)
    if kv_levels:
        kv = (kv.clamp(-2, 2) * (kv_levels / 4)).round() / (kv_levels / 4)
    if windows == "causal":
        ks, ke = causal_windows(T, S)
    elif windows == "random":
        a = torch.randint(0, S + 1, (T,), generator=g)
        b = torch.randint(0, S + 1, (T,), generator=g)
        ks, ke = torch.minimum(a, b).to(torch.int32), torch.maximum(a, b).to(torch.int32)
    elif windows == "short":
        ks = torch.randint(0, max(1, S - topk), (T,), generator=g).to(torch.int32)
        ln = torch.randint(0, topk + 1, (T,), generator=g).to(torch.int32)
        ke = torch.minimum(ks + ln, torch.tensor(S, dtype=torch.int32))
    elif windows == "empty_mix":
        ks, ke = causal_windows(T, S)
        ke = ke.clone()
        ks = ks.clone()
        ke[::5] = ks[::5]                 # empty windows
        ks[1::7] = torch.clamp(ke[1::7] - 1, min=0)   # windows of one key
    elif windows == "packed":
        n = 3
        qn = [T // n] * (n - 1) + [T - (T // n) * (n - 1)]
        kn = [S // n] * (n - 1) + [S - (S // n) * (n - 1)]
        qn = [min(a, b) for a, b in zip(qn, kn)]
        ks, ke = packed_causal_windows(qn, kn)
        pad = T - ks.numel()
        if pad:
            ks = torch.cat([ks, torch.zeros(pad, dtype=torch.int32)])
            ke = torch.cat([ke, torch.zeros(pad, dtype=torch.int32)])
    else:
        raise ValueError(windows)
    cast = _fp8 if dtype == "fp8" else (lambda x: x.to(torch.bfloat16))
    return SelectInputs(f"small{seed}_{dtype}_{windows}", cast(q), cast(kv), sc, w,
                        ks.contiguous(), ke.contiguous(), topk)


def get(name: str):
    """Workload by name."""
    table = {
        "bf16_small": bf16_small, "bf16_ties": bf16_ties, "bf16_all_equal": bf16_all_equal,
        "rows_bf16": rows_bf16, "rows_f32": rows_f32, "rows_bf16_1024": rows_bf16_1024,
        "fp8_prefill": fp8_prefill, "fp8_packed": fp8_packed, "fp8_large": fp8_large,
        "fp8_prefill_64h": fp8_prefill_64h,
    }
    return table[name]()


def sample_rows(T: int, n: int, seed: int = 0) -> list[int]:
    """n seeded row indices of [0, T), always including the first and last."""
    g = torch.Generator(device="cpu")
    g.manual_seed(SEED_BASE + 7000 + seed)
    if n >= T:
        return list(range(T))
    mid = torch.randperm(T - 2, generator=g)[: n - 2] + 1
    return sorted({0, T - 1, *mid.tolist()})


def block_structured(seed: int, dtype: str, T: int, S: int, topk: int, hot_every: int = 8,
                     cold: float = 2.0 ** -7, heads: int = 32) -> SelectInputs:
    """Keys in 128-key blocks where only every hot_every-th block keeps its
    kv_scales and the others have theirs multiplied by `cold`, with causal
    windows and mostly positive weights (|N(0,1)|/sqrt(32), negated on the
    heads h % 8 == 0): the top-k lies in the hot blocks and the cold blocks'
    scores stay far below the threshold, the case score-bound pruning is for."""
    c = small_case(seed, dtype, T, S, topk, windows="causal", heads=heads)
    sc = c.kv_scales.clone()
    blk = torch.arange(S) // 128
    sc[blk % hot_every != 0] *= cold
    w = c.weights.abs()
    w[:, ::8] = -w[:, ::8]
    name = f"blocks{seed}_{dtype}" + ("" if heads == 32 else f"_{heads}h")
    return SelectInputs(name, c.q, c.kv, sc, w.contiguous(), c.ks, c.ke, topk)
