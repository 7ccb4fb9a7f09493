"""Oracle pins of the diagonal variance closure ("SPICY-KV" Independent Claim 3: the subgrid
variance may be a scalar or a diagonal vector sigma_m^2; the closure is the second cumulant of the
logit deviation): s = q.k/sqrt(d) + ln m + sum_i q_i^2 var_i / (2d).

Pins: isotropic variances reduce it to the scalar form |q|^2 sigma^2/(2d); exact tokens carry zero
variance; for Gaussian members with a diagonal covariance the closure is the exact log-moment
generating function, so Z_closure/Z_full -> 1 as the segment grows, while the scalar form misses by
the closed-form factor exp((sum_i q_i^2 s_i^2 - |q|^2 mean(s^2)) / (2d))."""
import numpy as np
import pytest

import oracle

S, W = 8, 48


def test_isotropic_variance_equals_scalar_closure():
    rng = np.random.default_rng(0)
    E, d = 40, 64
    kt, vt = rng.standard_normal((E, d)), rng.standard_normal((E, d))
    alpha = np.log(rng.integers(1, 100, E)).astype(np.float64)
    sig2 = rng.random(E) * 0.5
    var = np.repeat(sig2[:, None], d, axis=1)
    q = rng.standard_normal((5, d))
    o1, l1 = oracle.decode_rows(q, kt, vt, alpha, sig2 / (2 * d))
    o2, l2 = oracle.decode_rows(q, kt, vt, alpha, sig2 / (2 * d), var)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)


def test_exact_tokens_have_zero_variance_and_var_averages_to_sigma2():
    rng = np.random.default_rng(1)
    T, d = 500, 128
    k = rng.standard_normal((T, d)).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    u = oracle.coarsen_unit(k, v, S, W, 30, oracle.projection(3, d))
    E = u.kt.shape[0]
    exact = list(range(u.s_eff)) + list(range(E - u.w_eff, E))
    assert np.all(u.var[exact] == 0.0)
    np.testing.assert_allclose(u.var.mean(axis=1), u.sigma2, rtol=1e-12, atol=0)
    # per-dimension population variance of one segment, by numpy
    e = u.s_eff + 3
    st, m = int(u.start[e]), int(u.mass[e])
    np.testing.assert_allclose(u.var[e], k[st:st + m].astype(np.float64).var(axis=0), rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("m", [64, 1024, 16384])
def test_gaussian_members_diagonal_closure_is_exact_in_the_limit(m):
    """One middle segment (N = 1) of m Gaussian keys with per-dimension standard deviations s_i
    spread over a factor 8; q weights the high-variance dimensions."""
    rng = np.random.default_rng(m)
    d = 64
    s = np.exp(np.linspace(np.log(0.05), np.log(0.4), d))
    mu = rng.standard_normal(d) * 0.3
    T = S + m + W
    k = (mu + rng.standard_normal((T, d)) * s).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    u = oracle.coarsen_unit(k, v, S, W, 1, oracle.projection(9, d))
    e = u.s_eff
    assert int(u.mass[e]) == m
    q = (np.linspace(0.5, 3.0, d) * np.sign(rng.standard_normal(d)))[None, :]
    members = k[S:S + m].astype(np.float64)
    z_full = np.log(np.sum(np.exp(members @ q[0] / np.sqrt(d))))
    one = slice(e, e + 1)
    _, l_diag = oracle.decode_rows(q, u.kt[one], u.vt[one], u.alpha[one], u.beta[one], u.var[one])
    _, l_scal = oracle.decode_rows(q, u.kt[one], u.vt[one], u.alpha[one], u.beta[one])
    _, l_mass = oracle.decode_rows(q, u.kt[one], u.vt[one], u.alpha[one], np.zeros(1))
    bias = (np.sum(q[0] ** 2 * s ** 2) - np.sum(q[0] ** 2) * np.mean(s ** 2)) / (2 * d)
    err_diag = abs(l_diag[0] - z_full)
    err_scal = l_scal[0] - z_full
    assert err_diag < 3.0 / np.sqrt(m) * 0.05 + 1e-3          # sampling error only
    assert err_scal == pytest.approx(-bias, abs=0.25 * bias + 3.0 / np.sqrt(m) * 0.05)
    assert l_mass[0] <= z_full + 1e-12                         # Jensen gap
    assert err_diag < abs(err_scal)
