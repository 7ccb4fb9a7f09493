"""Common-mode mean removal ("SPICY-KV" Independent Claim 1(b): keys mapped into an anisotropy-
reduced space by removing their common-mode mean before coarsening) against this method.

Subtracting one vector mu from every key of a unit changes nothing the method computes, up to
rounding: the variation uses differences, d_t = |P [k_t - k_{t-1}; v_t - v_{t-1}]| (mu cancels), so
the segmentation is the same; segment means shift by mu while masses and variances do not, so every
logit of a query moves by the same q.mu/sqrt(d) and the softmax output is unchanged while lse moves
by exactly that amount. The pins: fp64 variation and decode reproduce this to rounding; the fixed
fp32 variation recipe (whose rounding depends on the operands) moves each quantised step by at most
a few units and the boundaries hardly at all."""
import numpy as np

import oracle

S, W = 8, 48


def test_mean_removal_leaves_variation_segments_and_attention_unchanged():
    rng = np.random.default_rng(21)
    T, d, N = 3000, 128, 60
    drift = np.cumsum(rng.standard_normal((T, d)) * 0.05, axis=0)
    mu = (rng.standard_normal(d) * 4.0)                     # a strong common mode
    k = (mu + drift + rng.standard_normal((T, d)) * 0.1).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    kc = (k.astype(np.float64) - k.astype(np.float64).mean(axis=0)).astype(np.float32)   # mean removed
    P = oracle.projection(4, d)
    a = oracle.coarsen_unit(k, v, S, W, N, P)
    b = oracle.coarsen_unit(kc, v, S, W, N, P)
    # variation: identical in exact arithmetic (fp64 path to rounding; fp32 recipe within a few units)
    np.testing.assert_allclose(b.d64, a.d64, rtol=1e-5, atol=1e-9)
    assert np.max(np.abs(a.D - b.D)) <= 64               # 2^-20 units; steps are ~2^20 * |d_t| ~ 1e6
    moved = np.count_nonzero(a.bounds != b.bounds)
    assert moved <= 2, moved
    if moved == 0:
        # same segments: means shift by the common mode, masses and variances do not move
        shift = (k.astype(np.float64) - kc.astype(np.float64))
        mid = slice(a.s_eff, a.kt.shape[0] - a.w_eff)
        starts, lens = a.start[mid], a.mass[mid]
        exp_shift = np.stack([shift[s:s + m].mean(axis=0) for s, m in zip(starts, lens)])
        np.testing.assert_allclose(a.kt[mid] - b.kt[mid], exp_shift, rtol=0, atol=1e-9)
        np.testing.assert_allclose(a.sigma2, b.sigma2, rtol=1e-6, atol=1e-12)
        np.testing.assert_array_equal(a.mass, b.mass)


def test_decode_is_invariant_to_a_common_key_shift():
    """Shift every stored key (exact tokens and node means alike) by mu: the output is unchanged and
    lse moves by q.mu/sqrt(d) (the closure and log-mass terms do not depend on mu)."""
    rng = np.random.default_rng(22)
    E, d = 300, 64
    kt = rng.standard_normal((E, d))
    vt = rng.standard_normal((E, d))
    alpha = np.log(rng.integers(1, 50, E)).astype(np.float64)
    beta = rng.random(E) * 0.01
    var = rng.random((E, d)) * 0.2
    mu = rng.standard_normal(d) * 3.0
    q = rng.standard_normal((6, d))
    for extra in (None, var):
        o1, l1 = oracle.decode_rows(q, kt, vt, alpha, beta, extra)
        o2, l2 = oracle.decode_rows(q, kt - mu, vt, alpha, beta, extra)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1 - l2, q @ mu / np.sqrt(d), rtol=0, atol=1e-11)
