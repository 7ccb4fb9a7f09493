"""Step-reconstruction error of the equal-variation encoder (not gpu).

"Equal-Variation KV Cache", Mathematical statement and Key formulas: the
normalised minimax error of the encoder/decoder is 1/(2N); Verification: the
sharp scalar prediction matched 1/(2N) through N = 32 and burst paths decay
with slope near -1. The page's decoder pi_N(t) = pi(t_j) (left endpoint) has
worst case Var/N; the sharp 1/(2N) needs a mid-variation representative.
"""
import numpy as np
import pytest


def _linear(n=4097, scale=1000.0):
    return np.linspace(0.0, scale, n)


@pytest.mark.parametrize("N", [1, 2, 3, 5, 8, 16, 32])
def test_linear_path_midrange_error_is_var_over_2N(orc, N):
    x = _linear()
    _, err, var = orc.step_reconstruction(x, N, "midrange")
    h = var / (len(x) - 1)                            # sampling resolution
    assert abs(err / var - 1 / (2 * N)) <= h / var + 1e-9


@pytest.mark.parametrize("N", [1, 4, 16, 32])
def test_linear_path_mean_error_matches_midrange(orc, N):
    x = _linear()
    _, e_mean, var = orc.step_reconstruction(x, N, "mean")
    h = var / (len(x) - 1)
    assert abs(e_mean / var - 1 / (2 * N)) <= h / var + 1e-9


@pytest.mark.parametrize("N", [2, 8, 32])
def test_left_endpoint_error_is_var_over_N(orc, N):
    x = _linear()
    _, err, var = orc.step_reconstruction(x, N, "left")
    h = var / (len(x) - 1)
    assert abs(err / var - 1 / N) <= 2 * h / var + 1e-9


def test_smooth_and_burst_paths_decay_like_one_over_N(orc):
    t = np.linspace(0, 1, 20001)
    smooth = 300 * np.sin(2 * np.pi * 3 * t) + 100 * t
    burst = 200 * np.tanh((t - 0.5) * 80) + 20 * np.sin(12 * t)
    for path in (smooth, burst):
        Ns = np.array([4, 8, 16, 32, 64])
        errs = []
        for N in Ns:
            _, err, var = orc.step_reconstruction(path, int(N), "midrange")
            assert err <= var / (2 * N) * (1 + 1e-3) + var / 20000 * 2     # never above the sharp bound
            errs.append(err / var)
        slope = np.polyfit(np.log(Ns), np.log(errs), 1)[0]
        assert -1.4 < slope < -0.7


def test_equal_variation_is_location_insensitive(orc):
    """Moving a burst along the sequence leaves the equal-variation error unchanged while
    uniform-in-time segments degrade when the burst falls inside one segment."""
    t = np.linspace(0, 1, 8001)
    errs = []
    for c in (0.21, 0.5, 0.77):
        path = 500 * np.tanh((t - c) * 400)
        _, err, var = orc.step_reconstruction(path, 16, "midrange")
        errs.append(err / var)
    assert max(errs) - min(errs) < 2e-3
    assert max(errs) <= 1 / 32 + 1e-3
