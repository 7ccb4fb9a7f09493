"""Pins of the oracle pieces that check the tensor-core projection option stage by stage
(SKV_PROJECTION_TENSOR_BF16): the bf16 rounding of P, the exact steps of the bf16 projection and
their error bound, and the coarsening driven by given steps."""
from fractions import Fraction
import math

import numpy as np
import torch

import oracle

S, W = 8, 48


def test_bf16_round_equals_torch_conversion():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0e-39, 6.5e4], np.float32)]).astype(np.float32)
    # exact ties: the low 16 bits 0x8000 with even and odd kept halves
    ties = (np.arange(1000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32) + np.uint32(0x3F800000)
    x = np.concatenate([x, ties.view(np.float32)])
    ref = torch.from_numpy(x).bfloat16().float().numpy()
    assert np.array_equal(oracle.bf16_round(x).view(np.uint32), ref.view(np.uint32))


def test_projection_bf16_is_the_rounded_projection():
    P = oracle.projection(11, 64)
    P16 = oracle.projection_bf16(11, 64)
    assert P16.shape == P.shape and np.array_equal(P16, oracle.bf16_round(P))
    assert np.all(np.abs(P16 - P) <= np.abs(P) * 2.0 ** -8)


def test_given_steps_reproduce_the_recipe_pipeline():
    """Fed the fixed recipe's own steps, the given-steps path returns the same cumulative variation,
    boundaries, entries and statistics as coarsen_unit (both representatives, centred or not)."""
    rng = np.random.default_rng(2)
    T, d, N = 900, 64, 25
    k = (np.cumsum(rng.standard_normal((T, d)) * 0.1, axis=0) + 3).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    P = oracle.projection(5, d)
    for rep in ("mean", "variation"):
        for center in (False, True):
            a = oracle.coarsen_unit(k, v, S, W, N, P, rep, center)
            b = oracle.coarsen_unit_from_steps(k, v, S, W, N, a.D, rep, center)
            for f in ("D", "C", "bounds", "start", "mass"):
                assert np.array_equal(getattr(a, f), getattr(b, f)), (rep, center, f)
            for f in ("kt", "vt", "sigma2", "var", "alpha", "beta"):
                assert np.array_equal(getattr(a, f), getattr(b, f)), (rep, center, f)


def test_given_steps_drive_the_boundaries():
    """Steps with one large jump: every threshold at or below the jump's share falls on it."""
    rng = np.random.default_rng(3)
    T, d, N = 300, 64, 10
    k = rng.standard_normal((T, d)).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    M = T - S - W
    D = np.full(M, 100, np.int64)
    D[0] = 0
    D[50] = 100 * M * 4            # the jump holds about 80% of the variation
    u = oracle.coarsen_unit_from_steps(k, v, S, W, N, D)
    C = np.cumsum(D)
    np.testing.assert_array_equal(u.C, C)
    np.testing.assert_array_equal(u.bounds, oracle.segment(C, N))
    assert np.count_nonzero(u.bounds[1:N] == 50) >= 7


def _exact_step(P16, x0, x1):
    dz = [sum(Fraction(float(P16[i, j])) * (Fraction(float(x1[j])) - Fraction(float(x0[j])))
              for j in range(P16.shape[1])) for i in range(P16.shape[0])]
    return math.sqrt(float(sum(z * z for z in dz)))


def test_tensor_steps_reference_is_the_exact_step():
    rng = np.random.default_rng(4)
    T, d = S + W + 6, 64
    k = torch.from_numpy(rng.standard_normal((T, d)) * 5).bfloat16().float().numpy()
    v = torch.from_numpy(rng.standard_normal((T, d))).bfloat16().float().numpy()
    P16 = oracle.projection_bf16(7, d)
    dref, bound = oracle.tensor_steps_reference(k, v, S, W, P16)
    x = np.concatenate([k, v], axis=1)[S:S + 6]
    assert dref[0] == 0.0 and bound[0] == 0.0
    for t in range(1, 6):
        e = _exact_step(P16, x[t - 1], x[t]) * 2 ** 20
        assert abs(dref[t] - e) <= 1e-9 * e


def _truncate_f32(a):
    """Round toward zero to binary32 (float64 in, float64 out)."""
    f = np.float32(a)
    bad = np.abs(f.astype(np.float64)) > np.abs(a)
    f[bad] = np.nextafter(f[bad], np.float32(0))
    return f.astype(np.float64)


def test_tensor_step_bound_covers_a_truncating_blocked_accumulation():
    """A plausible tensor-core model -- exact products, 16 per accumulate step, every step truncated
    to binary32 -- followed by the fixed recipe's fp32 step stays within the bound, while a
    dropped feature does not (the bound has teeth)."""
    rng = np.random.default_rng(5)
    T, d = S + W + 200, 128
    k = torch.from_numpy(np.cumsum(rng.standard_normal((T, d)) * 0.3, axis=0)).bfloat16().float().numpy()
    v = torch.from_numpy(rng.standard_normal((T, d))).bfloat16().float().numpy()
    P16 = oracle.projection_bf16(9, d)
    dref, bound = oracle.tensor_steps_reference(k, v, S, W, P16)
    x = np.concatenate([k, v], axis=1)[S:S + 200].astype(np.float64)
    prod = x[:, None, :] * P16.astype(np.float64)[None, :, :]          # exact products [t, i, j]

    def steps(prod):
        acc = np.zeros(prod.shape[:2])
        for ks in range(prod.shape[2] // 16):
            acc = _truncate_f32(acc + prod[:, :, 16 * ks:16 * ks + 16].sum(axis=2))
        z = acc.astype(np.float32)
        return np.array([0] + [oracle.quantised_step(z[t - 1], z[t]) for t in range(1, z.shape[0])])

    Dm = steps(prod)
    assert np.all(np.abs(Dm - dref) <= bound)
    dropped = prod.copy()
    dropped[:, :, 37] = 0.0
    assert np.any(np.abs(steps(dropped) - dref) > bound)
