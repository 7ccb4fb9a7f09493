"""Pins of the oracle's whole coarsening of one unit (not gpu).

Brute force on T <= 64: an independent pure-Python pipeline (exact-rational
binary32 variation, per-j linear search for the boundaries, numpy member
statistics) must give the same entries bit for bit (integers) and to fp64
rounding (statistics). Closed forms: linear member keys have per-dimension
variance delta^2 (m^2 - 1) / 12; identical keys have zero variance.
Node statistics follow "SPICY-KV" Claims 2-3 and section 2 (alpha = log m,
beta = sigma^2 / (2 d_k)); the split and segmentation follow "Equal-Variation
KV Cache", Mathematical statement and Implementation notes.
"""
import math

import numpy as np
import pytest

import exact_f32 as E
from test_oracle_segment import brute as brute_segment


def brute_coarsen(k, v, S, W, N, P):
    T, d = k.shape
    s_eff = min(S, T)
    w_eff = min(W, T - s_eff)
    M = T - s_eff - w_eff
    D = [0] * M
    zprev = None
    for t in range(M):
        z = E.feature(P, k[s_eff + t], v[s_eff + t])
        if t > 0:
            D[t] = E.quantised_step(zprev, z)
        zprev = z
    C = np.cumsum(np.array(D, dtype=object)) if M else np.zeros(0, dtype=object)
    b = brute_segment(list(C), N)
    ents = [(t, 1) for t in range(s_eff)]
    ents += [(s_eff + b[j], b[j + 1] - b[j]) for j in range(N) if b[j + 1] > b[j]]
    ents += [(s_eff + M + t, 1) for t in range(w_eff)]
    kt, vt, s2 = [], [], []
    for st, m in ents:
        kk = k[st:st + m].astype(np.float64)
        vv = v[st:st + m].astype(np.float64)
        kt.append(kk.mean(0))
        vt.append(vv.mean(0))
        s2.append(kk.var(0).mean())                    # population variance, averaged over d
    return dict(D=D, b=b, ents=ents, kt=np.array(kt).reshape(-1, d), vt=np.array(vt).reshape(-1, d),
                s2=np.array(s2), alpha=np.log([m for _, m in ents]) if ents else np.zeros(0),
                M=M)


def _inputs(rng, T, d, kind):
    if kind == "walk":
        k = np.cumsum(rng.standard_normal((T, d)) * 0.3, 0)
        jumps = rng.random(T) < 0.1
        k[jumps] += rng.standard_normal((jumps.sum(), d)) * 3
        v = rng.standard_normal((T, d))
    elif kind == "flat":
        k = np.ones((T, d)) * 2.5
        v = np.zeros((T, d))
        if T > 20:
            k[20:] += 1.0                             # a single step: all thresholds at one token
    else:
        k = rng.standard_normal((T, d))
        v = rng.standard_normal((T, d))
    return k.astype(np.float32), v.astype(np.float32)


CASES = [(T, S, W, N, kind) for (T, S, W, N, kind) in [
    (64, 8, 8, 6, "walk"), (64, 4, 12, 13, "walk"), (48, 8, 8, 40, "walk"), (40, 8, 8, 1, "normal"),
    (64, 2, 3, 9, "flat"), (30, 0, 0, 4, "flat"), (16, 8, 8, 3, "normal"), (10, 8, 8, 3, "normal"),
    (5, 8, 48, 2, "normal"), (0, 8, 8, 3, "normal"), (64, 0, 0, 64, "normal"), (33, 1, 1, 7, "walk"),
]]


@pytest.mark.parametrize("T,S,W,N,kind", CASES)
def test_coarsen_unit_matches_brute_force(orc, T, S, W, N, kind):
    d = 8
    rng = np.random.default_rng(T * 131 + N)
    k, v = _inputs(rng, T, d, kind)
    P = orc.projection(9, d)
    u = orc.coarsen_unit(k, v, S, W, N, P)
    ref = brute_coarsen(k, v, S, W, N, P)
    assert u.M == ref["M"]
    assert [int(x) for x in u.D] == ref["D"]
    assert [int(x) for x in u.bounds] == ref["b"]
    assert list(zip(u.start.tolist(), u.mass.tolist())) == ref["ents"]
    np.testing.assert_allclose(u.kt, ref["kt"], rtol=1e-14, atol=1e-12)
    np.testing.assert_allclose(u.vt, ref["vt"], rtol=1e-14, atol=1e-12)
    np.testing.assert_allclose(u.sigma2, ref["s2"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(u.alpha, ref["alpha"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(u.beta, u.sigma2 / (2 * d), rtol=1e-15)


def test_partition_and_mass(orc):
    rng = np.random.default_rng(3)
    T, d = 700, 64
    k, v = _inputs(rng, T, d, "walk")
    u = orc.coarsen_unit(k, v, 8, 48, 37, orc.projection(1, d))
    assert u.mass.sum() == T                           # every token in exactly one entry
    ends = u.start + u.mass
    assert np.array_equal(u.start[1:], ends[:-1])      # contiguous, in token order
    assert np.all(u.mass[:8] == 1) and np.all(u.mass[-48:] == 1)
    assert u.kt.shape[0] == 8 + 48 + np.count_nonzero(np.diff(u.bounds))


def test_linear_keys_closed_form_variance(orc):
    """Keys k_t = a + t delta inside one segment: Var_i = delta_i^2 (m^2 - 1) / 12, the mean is
    the midpoint; with N = 1 the whole middle is one segment."""
    d, T = 64, 90
    a = np.linspace(-1, 1, d)
    delta = np.linspace(0.5, 2.0, d) / 64
    t = np.arange(T)[:, None]
    k = (a + t * delta).astype(np.float32)
    v = np.zeros((T, d), np.float32)
    u = orc.coarsen_unit(k, v, 0, 0, 1, orc.projection(2, d))
    m = T
    kk = k.astype(np.float64)                         # the fp32 inputs, exactly
    np.testing.assert_allclose(u.kt[0], kk.mean(0), rtol=1e-14)
    want_var = (np.diff(kk, axis=0).mean(0) ** 2) * (m * m - 1) / 12
    np.testing.assert_allclose(u.sigma2[0], want_var.mean(), rtol=1e-5)
    assert u.alpha[0] == pytest.approx(math.log(m), abs=1e-15)


def test_identical_keys_zero_variance(orc):
    d, T = 64, 40
    k = np.tile(np.linspace(-3, 3, d, dtype=np.float32), (T, 1))
    v = np.random.default_rng(0).standard_normal((T, d)).astype(np.float32)
    u = orc.coarsen_unit(k, v, 0, 0, 5, orc.projection(2, d))
    assert np.all(u.sigma2 == 0.0) and np.all(u.beta == 0.0)


def test_alternating_keys_hit_every_threshold_exactly(orc):
    """Keys alternating between two rows give every middle step the same D (the difference of the
    two projections, negated, has the same square norm), so c_t = t D; with M - 1 = N k the
    thresholds j c_T / N are hit exactly, at b_j = j k (the equality case of N c_t >= j c_T)."""
    d, S, W, N, step = 64, 8, 48, 16, 40
    M = N * step + 1
    T = S + M + W
    rng = np.random.default_rng(3)
    k = (rng.standard_normal((T, d)) * 0.3).astype(np.float32)
    v = np.zeros((T, d), np.float32)
    a = k[S].copy()
    k[S:S + M:2] = a
    k[S + 1:S + M:2] = a * np.float32(-0.5) + np.float32(0.125)
    u = orc.coarsen_unit(k, v, S, W, N, orc.projection(5, d))
    assert u.C[1] > 0 and np.array_equal(u.C, np.arange(M, dtype=np.int64) * u.C[1])
    assert np.array_equal(u.bounds, np.append(np.arange(N) * step, M))
    assert np.all(u.mass[S:S + N - 1] == step) and u.mass[S + N - 1] == step + 1   # the last also takes t = M - 1


def test_overflow_is_reported(orc):
    d, T = 64, 20
    k = np.zeros((T, d), np.float32)
    k[10:] = 1e30
    v = np.zeros((T, d), np.float32)
    with pytest.raises(orc.OracleError):
        orc.coarsen_unit(k, v, 0, 0, 3, orc.projection(2, d))


def test_planted_mistake_is_caught(orc, monkeypatch):
    """A plausible oracle bug (boundary token assigned to the previous segment) must fail
    the brute-force comparison: planted in a copy of the oracle's output on the CPU."""
    d = 8
    rng = np.random.default_rng(5)
    k, v = _inputs(rng, 64, d, "walk")
    P = orc.projection(9, d)
    u = orc.coarsen_unit(k, v, 8, 8, 6, P)
    ref = brute_coarsen(k, v, 8, 8, 6, P)
    shifted = [b + 1 if 0 < j < 6 else b for j, b in enumerate(u.bounds.tolist())]
    assert shifted != ref["b"]
