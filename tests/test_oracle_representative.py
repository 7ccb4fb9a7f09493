"""Oracle pins of the variation-weighted segment representative ("Equal-Variation KV Cache",
"Implementation notes": k_j = sum_{r in S_j} d_r k_r / sum_{r in S_j} d_r, same for v), with the
weights read as the fixed-point steps D_r (D_0 = 0 for the first middle token) and a segment
without variation keeping the plain mean.

Pins: a linear path (constant steps: each segment's representative is its midpoint token, except
that the first segment's first member carries no weight), numpy's weighted average over the
oracle's own exact integer steps, the convex hull of the members, and invariance of everything
the option must not touch (steps, boundaries, masses, variances, exact tokens)."""
import numpy as np
import pytest

import oracle

S, W = 8, 48


def _linear_unit(T, d, seed):
    rng = np.random.default_rng(seed)
    a, bk = rng.standard_normal(d), rng.standard_normal(d) * 0.05
    c, bv = rng.standard_normal(d), rng.standard_normal(d) * 0.05
    t = np.arange(T, dtype=np.float64)[:, None]
    # fp32 values exactly: the path is linear up to the fp32 rounding of each token
    return (a + t * bk).astype(np.float32), (c + t * bv).astype(np.float32)


def test_linear_path_representative_is_segment_midpoint():
    T, d, N = 4 * 64 + S + W, 64, 8
    k, v = _linear_unit(T, d, seed=3)
    P = oracle.projection(11, d)
    u = oracle.coarsen_unit(k, v, S, W, N, P, representative="variation")
    plain = oracle.coarsen_unit(k, v, S, W, N, P)
    # steps are constant up to rounding
    D = u.D[1:].astype(np.float64)
    assert u.D[0] == 0 and D.min() > 0 and (D.max() - D.min()) / D.mean() < 1e-3
    for e in range(u.s_eff, u.s_eff + (u.mass.shape[0] - u.s_eff - u.w_eff)):
        st, m = int(u.start[e]), int(u.mass[e])
        members = np.arange(st, st + m)
        if st == u.s_eff:            # first segment: D_0 = 0 drops its first member
            members = members[1:]
        mid_k = k[members].astype(np.float64).mean(axis=0)   # a linear path: mean = midpoint token
        mid_v = v[members].astype(np.float64).mean(axis=0)
        assert np.abs(u.kt[e] - mid_k).max() < 1e-4 * (1 + np.abs(mid_k).max())
        assert np.abs(u.vt[e] - mid_v).max() < 1e-4 * (1 + np.abs(mid_v).max())
        # and the plain mean of the first segment differs by half a step
        if st == u.s_eff:
            assert np.abs(plain.kt[e] - u.kt[e]).max() > 0.4 * np.abs(k[1] - k[0]).max()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_weighted_representative_matches_numpy_average(seed):
    rng = np.random.default_rng(seed)
    T, d, N = 700, 64, 25
    k = rng.standard_normal((T, d)).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    k[300:420] = k[300]            # a flat stretch: segments inside it have no variation
    v[300:420] = v[300]
    P = oracle.projection(5 + seed, d)
    u = oracle.coarsen_unit(k, v, S, W, N, P, representative="variation")
    n_flat = 0
    for e in range(u.s_eff, u.mass.shape[0] - u.w_eff):
        st, m = int(u.start[e]), int(u.mass[e])
        w = u.D[st - u.s_eff: st - u.s_eff + m].astype(np.float64)
        kk, vv = k[st:st + m].astype(np.float64), v[st:st + m].astype(np.float64)
        if w.sum() == 0:
            n_flat += 1
            ek, ev = kk.mean(axis=0), vv.mean(axis=0)
        else:
            ek, ev = np.average(kk, axis=0, weights=w), np.average(vv, axis=0, weights=w)
        np.testing.assert_allclose(u.kt[e], ek, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(u.vt[e], ev, rtol=1e-12, atol=1e-12)
        # inside the members' per-dimension hull
        assert np.all(u.kt[e] >= kk.min(axis=0) - 1e-12) and np.all(u.kt[e] <= kk.max(axis=0) + 1e-12)
    assert n_flat >= 0


def test_option_changes_only_the_middle_representatives():
    rng = np.random.default_rng(9)
    T, d, N = 900, 128, 40
    k = rng.standard_normal((T, d)).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    P = oracle.projection(2, d)
    a = oracle.coarsen_unit(k, v, S, W, N, P)
    b = oracle.coarsen_unit(k, v, S, W, N, P, representative="variation")
    for f in ("D", "C", "bounds", "start", "mass", "sigma2", "alpha", "beta"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    E = a.kt.shape[0]
    exact = list(range(a.s_eff)) + list(range(E - a.w_eff, E))
    assert np.array_equal(a.kt[exact], b.kt[exact]) and np.array_equal(a.vt[exact], b.vt[exact])
    mid = [e for e in range(a.s_eff, E - a.w_eff) if a.mass[e] > 1]
    assert mid and np.abs(a.kt[mid] - b.kt[mid]).max() > 1e-3


def test_flat_segment_keeps_plain_mean():
    """Identical tokens after the first middle token: every step is zero, so each segment keeps
    its plain mean (here the common token)."""
    T, d = 200, 64
    rng = np.random.default_rng(4)
    k = np.repeat(rng.standard_normal((1, d)).astype(np.float32), T, axis=0)
    v = np.repeat(rng.standard_normal((1, d)).astype(np.float32), T, axis=0)
    P = oracle.projection(1, d)
    u = oracle.coarsen_unit(k, v, S, W, 10, P, representative="variation")
    assert int(u.C[-1]) == 0 and u.mass.shape[0] == u.s_eff + 1 + u.w_eff   # C_T = 0: one node
    np.testing.assert_array_equal(u.kt[u.s_eff], k[0].astype(np.float64))
