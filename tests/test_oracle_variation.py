"""Pins of the oracle's fixed fp32 variation recipe (not gpu).

The recipe ("Equal-Variation KV Cache", Implementation notes: z_t = P[k_t; v_t],
d_t = ||z_t - z_{t-1}||_2) is a chain of correctly rounded IEEE operations. An
exact-rational model of binary32 (tests/exact_f32.py) must reproduce the oracle
bit for bit; a dropped fma, a reordered chain or contraction would break it.
"""
import numpy as np

import exact_f32 as E


def _rand(rng, n, scale):
    return (rng.standard_normal(n) * scale).astype(np.float32)


def test_feature_matches_exact_binary32_model(orc):
    rng = np.random.default_rng(0)
    for d, scale in [(8, 1.0), (8, 100.0), (64, 3.0)]:
        P = orc.projection(3, d)
        for _ in range(3):
            k, v = _rand(rng, d, scale), _rand(rng, d, 1.0)
            got = orc.feature_f32(P, k, v)
            want = E.feature(P, k, v)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (d, got, want)


def test_quantised_step_matches_exact_model(orc):
    rng = np.random.default_rng(1)
    for scale in [1e-6, 1e-3, 1.0, 30.0, 5e3]:
        for _ in range(20):
            zp, zc = _rand(rng, 16, scale), _rand(rng, 16, scale)
            assert orc.quantised_step(zp, zc) == E.quantised_step(zp, zc)


def test_quantised_step_rounds_half_to_even(orc):
    # d = 2^-21 exactly -> d * 2^20 = 0.5 -> 0 ; d = 3 * 2^-21 -> 1.5 -> 2
    zp = np.zeros(16, np.float32)
    zc = np.zeros(16, np.float32)
    zc[0] = 2.0 ** -21
    assert orc.quantised_step(zp, zc) == 0
    zc[0] = 3 * 2.0 ** -21
    assert orc.quantised_step(zp, zc) == 2
    zc[0] = 5 * 2.0 ** -21
    assert orc.quantised_step(zp, zc) == 2


def test_quantised_step_closed_form(orc):
    # a 3-4-5 triangle: d = 5 exactly, D = 5 * 2^20
    zp = np.zeros(16, np.float32)
    zc = np.zeros(16, np.float32)
    zc[3], zc[9] = 3.0, -4.0
    assert orc.quantised_step(zp, zc) == 5 * 2 ** 20


def test_quantised_step_overflow(orc):
    import pytest
    zp = np.zeros(16, np.float32)
    zc = np.zeros(16, np.float32)
    zc[0] = 2.0 ** 20          # d * 2^20 = 2^40: largest accepted
    assert orc.quantised_step(zp, zc) == 2 ** 40
    zc[0] = 2.0 ** 20 * 1.001
    with pytest.raises(orc.OracleError):
        orc.quantised_step(zp, zc)
    zc[0] = np.inf
    with pytest.raises(orc.OracleError):
        orc.quantised_step(zp, zc)


def test_fp32_recipe_close_to_fp64(orc):
    """The fp32 variation stays within a few fp32 ulps (relative) of the fp64 one on
    workload-like tokens; the quantised codes then differ by at most a few units."""
    rng = np.random.default_rng(2)
    d = 128
    T = 300
    k = np.cumsum(rng.standard_normal((T, d)) * 0.05, 0).astype(np.float32) + 20
    v = rng.standard_normal((T, d)).astype(np.float32)
    u = orc.coarsen_unit(k, v, 0, 0, 8, orc.projection(4, d))
    d32 = u.D[1:] / 2.0 ** 20
    rel = np.abs(d32 - u.d64[1:]) / u.d64[1:]
    assert rel.max() < 2e-5


def test_fp64_variant_moves_steps_but_not_boundaries_on_the_workloads(orc):
    """Information on the fixed fp32 recipe (reading 4): on the 1.5B-shaped 10.5K-token workload's
    first unit (regime-walk keys, N = 365) the fp64 variation differs from the fp32 recipe's in the
    last digits of almost every quantised step, yet the segment boundaries computed from the fp64
    steps equal the recipe's (at most 1% may differ; none do on this unit)."""
    import workloads
    w = workloads.WORKLOADS["gqa6_10k5_prefill_decode"]
    T_list = workloads.seq_lengths(w)
    k, v, _ = workloads.make_kv(w, "cpu", T_list=T_list)
    kk = workloads.unit_rows(k, T_list, w.Hkv, 0, 0).float().numpy()
    vv = workloads.unit_rows(v, T_list, w.Hkv, 0, 0).float().numpy()
    u = orc.coarsen_unit(kk, vv, 8, 48, w.N, orc.projection(w.seed, w.d))
    d32, d64 = u.D[1:] / 2.0 ** 20, u.d64[1:]
    rel = np.abs(d32 - d64) / d64
    D64 = np.rint(u.d64 * 2.0 ** 20).astype(np.int64)
    D64[0] = 0
    b64 = orc.segment(np.cumsum(D64), w.N)
    moved = int((b64 != u.bounds).sum())
    print(f"\nmax rel |d32 - d64| / d64 = {rel.max():.2e}; steps D differing: {int((D64 != u.D).sum())} of {u.M}"
          f" (max {int(np.abs(D64 - u.D).max())} units); boundaries differing: {moved} of {w.N - 1}")
    assert rel.max() < 1e-4
    assert moved <= (w.N - 1) // 100
