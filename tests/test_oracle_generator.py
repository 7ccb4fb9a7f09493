"""Pins of the oracle's projection generator (not gpu).

The projection P is drawn from SplitMix64 + Box-Muller ("Equal-Variation KV
Cache", Implementation notes: P is a fixed random projection; the workloads
specify Gaussian entries scaled by 1/sqrt(16)).
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return [int(x) for x in fh.read().split("\n") if x and not x.startswith("#")]


def test_splitmix64_published_vector(orc):
    want = _golden("splitmix64_seed1234567.txt")
    got = [int(x) for x in orc.splitmix64_stream(1234567, len(want))]
    assert got == want


def test_projection_shape_and_determinism(orc):
    P1 = orc.projection(11, 128)
    P2 = orc.projection(11, 128)
    assert P1.shape == (16, 256) and P1.dtype == np.float32
    assert np.array_equal(P1.view(np.uint32), P2.view(np.uint32))
    assert not np.array_equal(P1, orc.projection(12, 128))


def test_projection_uses_stream_in_order(orc):
    """Entry e consumes words 2e and 2e+1 of the seed's stream: P for d=64 is the leading
    part (row-major) of the entry sequence that d=128 also starts with."""
    a = orc.projection(5, 64).reshape(-1)
    b = orc.projection(5, 128).reshape(-1)
    assert np.array_equal(a.view(np.uint32), b[: a.size].view(np.uint32))


def test_projection_entries_are_gaussian_over_4(orc):
    """Box-Muller maps two uniforms to one N(0,1) draw; scaled by 1/sqrt(16) the entries
    must be N(0, 1/16): mean 0, variance 1/16, kurtosis 3, and pass a KS test."""
    from scipy import stats
    x = np.concatenate([orc.projection(s, 128).reshape(-1) for s in range(64)]).astype(np.float64)
    n = x.size
    assert abs(x.mean()) < 5 * 0.25 / np.sqrt(n)
    assert abs(x.var() - 1 / 16) < 5 * (1 / 16) * np.sqrt(2 / n)
    assert abs(stats.kurtosis(x, fisher=False) - 3.0) < 0.05
    assert stats.kstest(x / 0.25, "norm").pvalue > 1e-3


def test_projection_rejects_bad_args(orc):
    with pytest.raises(orc.OracleError):
        orc._check(orc._load().orc_projection(1, 0, 4, None), "projection")
