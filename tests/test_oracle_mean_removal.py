"""Common-mode mean removal ("SPICY-KV" Independent Claim 1(b): keys mapped into a less anisotropic
space by removing their common mean before coarsening) against this method.

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


# ---------------------------------------------------------------------------
# the centring option's mean key: one fixed fp32 order (reading R8)
# ---------------------------------------------------------------------------
from fractions import Fraction  # noqa: E402

import exact_f32  # noqa: E402


def _blocked_mean_exact_model(k):
    """The R8 order evaluated with the exact-rational binary32 model: every addition and the final
    division rounded once to binary32 (ties to even)."""
    T, d = k.shape
    mu = np.zeros(d, np.float32)
    for i in range(d):
        total = 0.0
        for b0 in range(0, T, 256):
            blk = 0.0
            for t in range(b0, min(b0 + 256, T)):
                blk = exact_f32.round_f32(exact_f32.f(blk) + exact_f32.f(k[t, i]))
            total = exact_f32.round_f32(exact_f32.f(total) + exact_f32.f(blk))
        mu[i] = exact_f32.round_f32(exact_f32.f(total) / T) if T else 0.0
    return mu


def _order_sensitive_keys(T, d, seed):
    rng = np.random.default_rng(seed)
    # mixed magnitudes, so that the rounding of each partial sum depends on the summation order
    mag = 10.0 ** rng.integers(-3, 4, size=(T, d))
    return (rng.standard_normal((T, d)) * mag + 37.0).astype(np.float32)


def test_key_mean_bits_follow_the_blocked_fp32_order():
    for T, seed in ((700, 1), (256, 2), (255, 3), (1, 4), (513, 5)):
        k = _order_sensitive_keys(T, 4, seed)
        got = oracle.key_mean_f32(k)
        want = _blocked_mean_exact_model(k)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (T, got, want)
    assert np.array_equal(oracle.key_mean_f32(np.zeros((0, 3), np.float32)), np.zeros(3, np.float32))


def test_key_mean_order_is_what_the_pin_sees():
    """The data above is order sensitive: one sequential fp32 sum over all tokens (no blocks) gives
    other bits in some dimension, so the bit pin would catch a wrong order."""
    k = _order_sensitive_keys(700, 8, 1)
    seq = np.zeros(8, np.float32)
    for t in range(700):
        seq = (seq + k[t]).astype(np.float32)
    naive = (seq / np.float32(700)).astype(np.float32)
    assert not np.array_equal(naive.view(np.uint32), oracle.key_mean_f32(k).view(np.uint32))


def test_key_mean_within_the_fp32_summation_bound_and_exact_on_integers():
    k = _order_sensitive_keys(5000, 6, 7)
    mu = oracle.key_mean_f32(k).astype(np.float64)
    exact = np.array([float(sum(Fraction(float(x)) for x in k[:, i]) / 5000) for i in range(6)])
    # blocked summation: at most (256 + 20) additions on any path, each within 2^-24 relative
    bound = (256 + 20 + 1) * 2.0 ** -24 * np.abs(k.astype(np.float64)).sum(axis=0) / 5000 + 2.0 ** -24 * np.abs(exact)
    assert np.all(np.abs(mu - exact) <= bound)
    ints = np.random.default_rng(8).integers(-1000, 1000, size=(3000, 5)).astype(np.float32)
    np.testing.assert_array_equal(oracle.key_mean_f32(ints),
                                  (ints.astype(np.float64).sum(axis=0) / 3000).astype(np.float32))


def test_centred_coarsening_runs_on_the_centred_keys():
    """coarsen_unit(center=True) equals coarsen_unit on center_keys(k); the centred keys average to
    about zero; the value statistics and masses do not depend on the option."""
    rng = np.random.default_rng(23)
    T, d, N = 2000, 64, 40
    k = (rng.standard_normal(d) * 5 + np.cumsum(rng.standard_normal((T, d)) * 0.05, axis=0)).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    P = oracle.projection(9, d)
    a = oracle.coarsen_unit(k, v, S, W, N, P, center=True)
    kc = oracle.center_keys(k)
    b = oracle.coarsen_unit(kc, v, S, W, N, P)
    np.testing.assert_array_equal(a.C, b.C)
    np.testing.assert_array_equal(a.bounds, b.bounds)
    np.testing.assert_array_equal(a.kt, b.kt)
    assert np.abs(kc.astype(np.float64).mean(axis=0)).max() < 1e-4 * np.abs(k).max()
    plain = oracle.coarsen_unit(k, v, S, W, N, P)
    if np.array_equal(plain.bounds, a.bounds):
        np.testing.assert_allclose(a.vt, plain.vt, rtol=0, atol=0)
        np.testing.assert_array_equal(a.mass, plain.mass)
        np.testing.assert_allclose(a.sigma2, plain.sigma2, rtol=1e-4, atol=1e-9)
