"""Seeded synthetic workloads for coarsening and compressed decode attention.

Inputs only: this module draws keys, values, queries, sequence lengths and page
assignments. It holds none of the method's arithmetic and imports neither the
GPU package nor the oracle; both consume what it produces.

Every draw comes from one ``torch.Generator`` seeded with the workload's seed on
the device the caller names (torch's CPU and CUDA generators give different
streams for the same seed, so a workload is identified by seed AND device).

Key trajectories are piecewise-smooth random walks ("regime walks"): a sequence
of T tokens is cut into R regimes at R-1 distinct uniform cut points in
[1, T-1]; regime r has a drift delta_r ~ N(0, 0.05^2 I) added every step and a
jump J_r ~ N(0, I) added at its first token (jumps accumulate); the key is the
walk plus N(0, 0.1^2 I) noise. Values and queries are N(0, 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

N_SINK = 8
N_RECENT = 48
PAGE_NODES = 16


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    R: int                      # decode query rows per sequence
    dtype: str                  # "f32" or "bf16"
    T: int = 0                  # uniform context length (0 when ragged)
    T_range: tuple = ()         # (lo, hi) log-uniform context lengths when ragged
    regimes: int = 0            # regimes per unit (0: max(8, round(T / 160)))
    N: int = 0                  # middle segments (0: floor(N_frac * T))
    N_frac: float = 0.0
    shuffle_pages: bool = False
    description: str = field(default="", compare=False)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", 0, B=1, Hq=2, Hkv=1, d=64, R=1, dtype="f32", T=1024, regimes=8, N=32,
        description="1 KV head, 2 query heads, d=64, T=1024, fp32, 8 regimes, N=32"),
    "gqa6_10k5_prefill_decode": Workload(
        "gqa6_10k5_prefill_decode", 1, B=1, Hq=12, Hkv=2, d=128, R=1, dtype="bf16", T=10500, regimes=40, N=365,
        description="1.5B-shaped: 12/2 heads, d=128, T=10,500, bf16, 40 regimes, N=365 (28.6x)"),
    "gqa7_32k_decode_3p5pct": Workload(
        "gqa7_32k_decode_3p5pct", 2, B=32, Hq=28, Hkv=4, d=128, R=1, dtype="bf16", T=32768, regimes=200, N=1091,
        description="7B-shaped decode: B=32, 28/4 heads, d=128, T=32,768, 200 regimes, N=1,091 (+8+48)"),
    "gqa7_ragged_paged_2pct": Workload(
        "gqa7_ragged_paged_2pct", 3, B=128, Hq=28, Hkv=4, d=128, R=4, dtype="bf16", T_range=(4096, 131072),
        regimes=0, N_frac=0.02, shuffle_pages=True,
        description="7B-shaped ragged paged decode: B=128, 28/4 heads, T log-uniform [4,096, 131,072], "
                    "N=floor(0.02 T), 4 query rows, 16-node pages, shuffled page table"),
    "coarsen_131k": Workload(
        "coarsen_131k", 4, B=8, Hq=28, Hkv=4, d=128, R=1, dtype="bf16", T=131072, regimes=1000, N=2621,
        description="Coarsening throughput: 8 x 4 KV heads, d=128, T=131,072, 1,000 regimes, N=2,621 (2%)"),
}


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def seq_lengths(w: Workload) -> list[int]:
    """Context length per sequence. Ragged lengths are floor(exp(U(ln lo, ln hi))) drawn on the CPU."""
    if not w.T_range:
        return [w.T] * w.B
    g = generator(w.seed, "cpu")
    lo, hi = w.T_range
    u = torch.rand(w.B, generator=g, dtype=torch.float64)
    return [int(math.floor(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo))))) for x in u]


def segment_counts(w: Workload, T_list: list[int]) -> list[int]:
    if w.N:
        return [w.N] * len(T_list)
    return [max(1, int(math.floor(w.N_frac * T))) for T in T_list]


def regimes_for(w: Workload, T: int) -> int:
    return w.regimes if w.regimes else max(8, int(round(T / 160)))


def regime_walk(g: torch.Generator, T: int, d: int, regimes: int, device,
                drift_std: float = 0.05, jump_std: float = 1.0, noise_std: float = 0.1) -> torch.Tensor:
    """Keys of one unit, fp32 [T, d] (see module docstring)."""
    if T == 0:
        return torch.zeros(0, d, device=device)
    n_cuts = max(0, min(regimes - 1, T - 1))
    cuts = (torch.randperm(T - 1, generator=g, device=device)[:n_cuts] + 1) if n_cuts else \
        torch.zeros(0, dtype=torch.long, device=device)
    starts = torch.cat([torch.zeros(1, dtype=torch.long, device=device), torch.sort(cuts).values])
    n_reg = starts.numel()
    is_start = torch.zeros(T, dtype=torch.long, device=device)
    is_start[starts] = 1
    rid = torch.cumsum(is_start, 0) - 1
    drift = torch.randn(n_reg, d, generator=g, device=device) * drift_std
    jump = torch.randn(n_reg, d, generator=g, device=device) * jump_std
    inc = drift[rid]
    inc[starts] += jump
    walk = torch.cumsum(inc, 0)
    return walk + torch.randn(T, d, generator=g, device=device) * noise_std


def make_kv(w: Workload, device, T_list: list[int] | None = None, values: str = "normal"):
    """Raw keys and values in the packed layout: sequence b is a contiguous [Hkv, T_b, d]
    block. Returns flat tensors k, v of shape [sum_b T_b * Hkv, d] in the workload dtype,
    plus the per-sequence lengths. values: "normal" (N(0,1)), "zero", or "walk" (an
    independent regime walk)."""
    T_list = seq_lengths(w) if T_list is None else T_list
    g = generator(w.seed, device)
    total = sum(T_list) * w.Hkv
    k = torch.empty(total, w.d, dtype=w.torch_dtype, device=device)
    v = torch.empty(total, w.d, dtype=w.torch_dtype, device=device)
    row = 0
    for T in T_list:
        for _ in range(w.Hkv):
            k[row:row + T] = regime_walk(g, T, w.d, regimes_for(w, T), device).to(w.torch_dtype)
            if values == "normal":
                v[row:row + T] = torch.randn(T, w.d, generator=g, device=device).to(w.torch_dtype)
            elif values == "zero":
                v[row:row + T] = 0
            elif values == "walk":
                v[row:row + T] = regime_walk(g, T, w.d, regimes_for(w, T), device).to(w.torch_dtype)
            else:
                raise ValueError(values)
            row += T
    return k, v, T_list


def make_queries(w: Workload, device) -> torch.Tensor:
    g = generator(w.seed + 1_000_003, device)
    return torch.randn(w.B, w.R, w.Hq, w.d, generator=g, device=device).to(w.torch_dtype)


def unit_rows(k: torch.Tensor, T_list: list[int], Hkv: int, b: int, h: int) -> torch.Tensor:
    """Rows [T_b, d] of unit (b, h) in the packed layout."""
    off = sum(T_list[:b]) * Hkv + h * T_list[b]
    return k[off:off + T_list[b]]


def max_entries(T: int, N: int, n_sink: int = N_SINK, n_recent: int = N_RECENT) -> int:
    s = min(n_sink, T)
    r = min(n_recent, T - s)
    return s + (N if T - s - r > 0 else 0) + r


def page_assignment(B: int, Hkv: int, pages_per_unit: list[int], shuffle: bool, seed: int):
    """Physical page ids [B, Hkv, max_pages] int32 (unused slots -1) and the pool size.
    Units take consecutive ids in (b, h) order; with shuffle the ids are permuted by a
    seeded CPU permutation (a fragmented allocator)."""
    max_pages = max(1, max(pages_per_unit))
    total = sum(pages_per_unit) * Hkv
    ids = torch.arange(total, dtype=torch.int32)
    if shuffle:
        ids = ids[torch.randperm(total, generator=generator(seed + 7, "cpu"))]
    table = torch.full((B, Hkv, max_pages), -1, dtype=torch.int32)
    pos = 0
    for b in range(B):
        for h in range(Hkv):
            n = pages_per_unit[b]
            table[b, h, :n] = ids[pos:pos + n]
            pos += n
    return table, max(total, 1)
