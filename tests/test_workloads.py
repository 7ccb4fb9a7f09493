"""The seeded input generator against the recipe it states (not gpu): regime walks (R regimes, a
N(0, 1) jump at each regime start, a per-regime N(0, 0.05^2) drift per step, N(0, 0.1^2) noise),
N(0, 1) values and queries, log-uniform ragged lengths, the N rules, the paged layout."""
import math
import os
import sys

import numpy as np
import pytest
import torch
from scipy import stats

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402


def test_regime_walk_structure():
    """Steps inside a regime are the regime's drift plus the difference of two noise draws; a regime
    start adds a N(0, I) jump. With d = 64 the jumps (norm ~8) stand far above the other steps
    (norm ~1.2), so the regime starts can be read off the walk."""
    d, T, R = 64, 20000, 25
    g = workloads.generator(123, "cpu")
    k = workloads.regime_walk(g, T, d, R, "cpu").double().numpy()
    step = np.diff(k, axis=0)
    norms = np.linalg.norm(step, axis=1)
    starts = np.flatnonzero(norms > 4.0) + 1
    assert len(starts) == R - 1                        # R regimes: R - 1 starts after token 0
    assert np.all(norms[norms <= 4.0] < 2.5)
    bounds = np.concatenate([[0], starts, [T]])
    drifts, noise_resid, jumps = [], [], []
    for r in range(R):
        lo, hi = bounds[r], bounds[r + 1]
        inner = step[lo:hi - 1]                        # steps strictly inside regime r
        if len(inner) < 50:
            continue
        delta = inner.mean(axis=0)
        drifts.append(delta)
        noise_resid.append(inner - delta)
        if r > 0:
            jumps.append(step[lo - 1] - delta)         # the step into the regime: jump + drift + noise
    drifts = np.concatenate(drifts)
    noise = np.concatenate(noise_resid).ravel()
    jumps = np.concatenate(jumps)
    assert abs(drifts.std() - 0.05) < 0.01             # per-regime drift N(0, 0.05^2)
    assert abs(noise.std() - 0.1 * math.sqrt(2)) < 0.005   # difference of two N(0, 0.1^2) draws
    assert abs(jumps.std() - math.sqrt(1.0 + 2 * 0.01)) < 0.06   # N(0, 1) jump plus the step noise
    assert stats.kstest(noise / noise.std(), "norm").pvalue > 1e-3


def test_regime_walk_degenerate_lengths():
    g = workloads.generator(1, "cpu")
    assert workloads.regime_walk(g, 0, 8, 5, "cpu").shape == (0, 8)
    one = workloads.regime_walk(g, 1, 8, 5, "cpu")        # more regimes than tokens: one regime
    assert one.shape == (1, 8) and torch.isfinite(one).all()


def test_values_queries_and_packed_layout():
    w = workloads.Workload("t", 5, B=3, Hq=6, Hkv=2, d=32, R=2, dtype="f32", T=0, regimes=4)
    T_list = [300, 0, 129]
    k, v, T_out = workloads.make_kv(w, "cpu", T_list=T_list)
    assert T_out == T_list and k.shape == v.shape == (sum(T_list) * w.Hkv, w.d)
    vv = v.double().numpy().ravel()
    assert abs(vv.mean()) < 0.03 and abs(vv.std() - 1.0) < 0.03
    # unit (b, h) is the contiguous block sum_{b' < b} Hkv T_b' + h T_b
    for b, T in enumerate(T_list):
        for h in range(w.Hkv):
            off = sum(T_list[:b]) * w.Hkv + h * T
            assert torch.equal(workloads.unit_rows(k, T_list, w.Hkv, b, h), k[off:off + T])
    q = workloads.make_queries(w, "cpu")
    assert q.shape == (w.B, w.R, w.Hq, w.d)
    assert abs(q.double().std().item() - 1.0) < 0.1
    # same seed, same inputs; another seed, other inputs
    k2, _, _ = workloads.make_kv(w, "cpu", T_list=T_list)
    assert torch.equal(k, k2)
    w3 = workloads.Workload("t", 6, B=3, Hq=6, Hkv=2, d=32, R=2, dtype="f32", T=0, regimes=4)
    assert not torch.equal(k, workloads.make_kv(w3, "cpu", T_list=T_list)[0])


def test_ragged_lengths_are_log_uniform_and_N_rules():
    w = workloads.WORKLOADS["gqa7_ragged_paged_2pct"]
    T_list = workloads.seq_lengths(w)
    lo, hi = w.T_range
    assert len(T_list) == w.B and all(lo <= T < hi for T in T_list)
    u = (np.log(T_list) - math.log(lo)) / (math.log(hi) - math.log(lo))
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    assert workloads.segment_counts(w, T_list) == [max(1, int(math.floor(0.02 * T))) for T in T_list]
    assert workloads.regimes_for(w, 16000) == 100 and workloads.regimes_for(w, 100) == 8
    w3 = workloads.WORKLOADS["gqa7_32k_decode_3p5pct"]
    assert workloads.seq_lengths(w3) == [32768] * 32 and workloads.segment_counts(w3, [32768]) == [1091]


@pytest.mark.parametrize("shuffle", [False, True])
def test_page_assignment_is_a_permutation(shuffle):
    pages = [3, 0, 5, 1]
    table, num = workloads.page_assignment(4, 2, pages, shuffle, seed=9)
    assert table.shape == (4, 2, 5) and num == sum(pages) * 2
    used = table[table >= 0]
    assert sorted(used.tolist()) == list(range(num))        # every physical page exactly once
    for b, n in enumerate(pages):
        assert (table[b, :, n:] == -1).all() and (table[b, :, :n] >= 0).all()
    if shuffle:
        assert not torch.equal(used, torch.arange(num, dtype=torch.int32))
