"""Pins of the oracle's compressed decode attention (not gpu).

"SPICY-KV" demo page, section 2: s = q.k/sqrt(d_k) + log m + |q|^2 sigma^2/(2 d_k)
followed by the standard (online) softmax; Claim 3 and the simulator text: the
mass and variance terms conserve the partition Z = sum exp(s) and close the
Jensen gap that mass-only merging leaves.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax


def _full_nodes(k, v):
    n = k.shape[0]
    return dict(kt=k, vt=v, alpha=np.zeros(n), beta=np.zeros(n))


def test_unit_mass_zero_variance_is_dense_softmax(orc):
    """All m = 1, sigma^2 = 0: the compressed logit is dense softmax attention (textbook)."""
    rng = np.random.default_rng(0)
    for d, n, rows in [(64, 1, 3), (64, 50, 2), (128, 300, 7)]:
        q = rng.standard_normal((rows, d))
        k = rng.standard_normal((n, d)) * 2
        v = rng.standard_normal((n, d))
        out, lse = orc.decode_rows(q, **_full_nodes(k, v))
        s = q @ k.T / math.sqrt(d)
        np.testing.assert_allclose(lse, logsumexp(s, axis=1), rtol=1e-13, atol=1e-12)
        np.testing.assert_allclose(out, softmax(s, axis=1) @ v, rtol=1e-11, atol=1e-12)


def test_identical_keys_conserve_partition_exactly(orc):
    """m identical tokens merged into one node (alpha = ln m, sigma^2 = 0) have the same
    partition and output as the m tokens themselves."""
    rng = np.random.default_rng(1)
    d = 64
    q = rng.standard_normal((4, d))
    key = rng.standard_normal(d)
    for m in [1, 2, 7, 1000]:
        toks_k = np.tile(key, (m, 1))
        toks_v = rng.standard_normal((m, d))
        out_f, lse_f = orc.decode_rows(q, **_full_nodes(toks_k, toks_v))
        out_c, lse_c = orc.decode_rows(q, key[None], toks_v.mean(0)[None], np.array([math.log(m)]),
                                       np.array([0.0]))
        np.testing.assert_allclose(lse_c, lse_f, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out_c, out_f, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("a", [0.25, 1.0])
def test_gaussian_closure_converges_and_mass_only_shows_jensen_gap(orc, a):
    """Member keys k = mu + eps, eps ~ N(0, sigma^2 I), |q|^2 sigma^2 / d = a. Then
    E exp(q.eps/sqrt d) = exp(a/2): the closure's Z/Z_full -> 1 as m grows while the
    mass-only logit (alpha only) stays at exp(-a/2)."""
    rng = np.random.default_rng(int(a * 100))
    d = 64
    errs = []
    for m in [16, 256, 4096]:
        ratios_c, ratios_m = [], []
        for rep in range(20):
            q = rng.standard_normal(d)
            sigma = math.sqrt(a * d) / np.linalg.norm(q)
            mu = rng.standard_normal(d)
            keys = mu + rng.standard_normal((m, d)) * sigma
            vals = rng.standard_normal((m, d))
            _, lse_full = orc.decode_rows(q[None], **_full_nodes(keys, vals))
            s2 = keys.var(0).mean()
            kt, vt = keys.mean(0)[None], vals.mean(0)[None]
            _, lse_c = orc.decode_rows(q[None], kt, vt, np.array([math.log(m)]), np.array([s2 / (2 * d)]))
            _, lse_m = orc.decode_rows(q[None], kt, vt, np.array([math.log(m)]), np.array([0.0]))
            ratios_c.append(lse_c[0] - lse_full[0])
            ratios_m.append(lse_m[0] - lse_full[0])
        errs.append(abs(np.mean(ratios_c)))
        # mass-only: log(Z/Z_full) -> -a/2 (Jensen gap)
        assert np.mean(ratios_m) == pytest.approx(-a / 2, abs=0.15 + 2.0 / math.sqrt(m))
    assert errs[-1] < 0.02
    assert errs[-1] < errs[0] + 1e-9


def test_entry_order_is_irrelevant(orc):
    rng = np.random.default_rng(2)
    d, n = 128, 60
    q = rng.standard_normal((3, d))
    kt, vt = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    al, be = np.log(rng.integers(1, 60, n)), rng.random(n) * 0.01
    o1, l1 = orc.decode_rows(q, kt, vt, al, be)
    p = rng.permutation(n)
    o2, l2 = orc.decode_rows(q, kt[p], vt[p], al[p], be[p])
    np.testing.assert_allclose(l1, l2, rtol=1e-14)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)


def test_logit_terms_closed_form(orc):
    """One entry: lse = q.k/sqrt(d) + alpha + |q|^2 beta exactly; out = v."""
    d = 64
    q = np.full((1, d), 0.5)
    kt = np.full((1, d), 2.0)
    vt = np.arange(d, dtype=np.float64)[None]
    out, lse = orc.decode_rows(q, kt, vt, np.array([math.log(5)]), np.array([0.125]))
    want = 0.5 * 2.0 * d / 8.0 + math.log(5) + (0.25 * d) * 0.125
    assert lse[0] == pytest.approx(want, abs=1e-13)
    np.testing.assert_allclose(out[0], vt[0], rtol=1e-14)


def test_empty_cache(orc):
    out, lse = orc.decode_rows(np.ones((2, 64)), np.zeros((0, 64)), np.zeros((0, 64)), np.zeros(0), np.zeros(0))
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_gqa_batch_matches_dense_attention_over_repeat_kv(orc):
    """The batched decode's head mapping: with m = 1 and sigma^2 = 0 everywhere, decoding a batch
    (several query rows per sequence, G query heads per KV head) equals dense softmax attention
    after expanding the KV heads with transformers' `repeat_kv` (the GQA expansion the Llama / Qwen
    model code applies: KV head j serves query heads j G .. j G + G - 1)."""
    import torch
    from transformers.models.llama.modeling_llama import repeat_kv

    rng = np.random.default_rng(7)
    B, R, Hkv, G, d, E = 2, 3, 3, 4, 16, 11
    Hq = Hkv * G
    K = rng.standard_normal((B, Hkv, E, d)) * 2
    V = rng.standard_normal((B, Hkv, E, d))
    q = rng.standard_normal((B, R, Hq, d))

    class U:
        pass

    units = []
    for b in range(B):
        row = []
        for h in range(Hkv):
            u = U()
            u.kt, u.vt, u.alpha, u.beta = K[b, h], V[b, h], np.zeros(E), np.zeros(E)
            row.append(u)
        units.append(row)
    out, lse = orc.decode(q, units, threads=2)

    Kx = repeat_kv(torch.from_numpy(K), G).numpy()          # [B, Hq, E, d]
    Vx = repeat_kv(torch.from_numpy(V), G).numpy()
    s = np.einsum("brhd,bhed->brhe", q, Kx) / math.sqrt(d)   # [B, R, Hq, E]
    np.testing.assert_allclose(lse, logsumexp(s, axis=-1), rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(out, np.einsum("brhe,bhed->brhd", softmax(s, axis=-1), Vx), rtol=1e-11, atol=1e-12)
