"""Pins of the oracle's equal-variation segmentation (not gpu).

"Equal-Variation KV Cache", Mathematical statement: breakpoints satisfy
V(t_j) = j Var / N with a first-hitting convention; Implementation notes: the
boundary is the first token whose cumulative variation crosses q_j = j c_T / N.
Brute force: for each j independently, a linear search for the first t with
N c_t >= j c_T in Python's exact integers.
"""
import numpy as np
import pytest


def brute(C, N):
    M = len(C)
    b = [0] * (N + 1)
    b[N] = M
    if M == 0:
        return b
    cT = int(C[-1])
    for j in range(1, N):
        t = 0
        while N * int(C[t]) < j * cT:
            t += 1
        b[j] = t
    return b


def _cases():
    rng = np.random.default_rng(7)
    yield np.zeros(0, np.int64), 4                        # empty middle
    yield np.zeros(10, np.int64), 3                       # c_T = 0: one segment
    yield np.array([0, 5], np.int64), 1                   # N = 1
    yield np.cumsum([0, 1, 1, 1, 1]).astype(np.int64), 9  # N > M: empty segments
    yield np.cumsum([0, 0, 0, 100, 0, 0, 1]).astype(np.int64), 5  # one jump crosses several thresholds
    for _ in range(200):
        M = int(rng.integers(1, 64))
        D = rng.integers(0, 50, M)
        D[0] = 0
        if rng.random() < 0.3:
            D[rng.random(M) < 0.5] = 0                    # flat runs (first-hitting matters)
        yield np.cumsum(D).astype(np.int64), int(rng.integers(1, 2 * M + 2))
    big = np.cumsum(np.r_[0, np.full(40, 2 ** 40 - 3)]).astype(np.int64)  # c_T near 2^45.3
    yield big, (1 << 20) - 1                              # products need 128 bits


@pytest.mark.parametrize("case", list(range(206)))
def test_segment_matches_definition(orc, case):
    C, N = list(_cases())[case]
    got = orc.segment(C, N)
    assert list(got) == brute(C, N)


def test_segment_invariants(orc):
    rng = np.random.default_rng(8)
    for _ in range(100):
        M = int(rng.integers(2, 500))
        D = rng.integers(0, 1000, M)
        D[0] = 0
        C = np.cumsum(D).astype(np.int64)
        N = int(rng.integers(1, M))
        b = orc.segment(C, N)
        cT = int(C[-1])
        assert b[0] == 0 and b[N] == M
        assert all(b[j] <= b[j + 1] for j in range(N))
        for j in range(1, N):
            t = int(b[j])
            assert N * int(C[t]) >= j * cT                    # threshold reached at b_j
            assert t == 0 or N * int(C[t - 1]) < j * cT       # ... and not before


def test_segment_equal_increments_gives_uniform_cut(orc):
    # constant variation per token -> boundaries at j*M/N (M multiple of N)
    M, N = 96, 8
    D = np.ones(M, np.int64)
    D[0] = 0
    b = orc.segment(np.cumsum(D), N)
    # c_t = t, c_T = 95: first t with 8 t >= 95 j  ->  ceil(95 j / 8)
    assert list(b) == [0] + [-(-95 * j // 8) for j in range(1, N)] + [M]
