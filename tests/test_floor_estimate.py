"""The boundary kernel's fast floor, checked on the host (not gpu).

For thresholds the kernel needs q = floor(N c / c_T) with 0 <= c <= c_T exactly. It takes
x = fl(fl(c) * fl(N * fl(1 / c_T))) in IEEE double (round to nearest, the same arithmetic as
Python floats), whose error is at most N 2^-51, and keeps floor(x) when x lies farther than
N 2^-48 from every integer; c = 0 gives 0 at once; every other case goes to the exact 128-bit
path. Here the same double arithmetic runs on random and adversarial (c at and around j c_T / N)
cases with c_T up to 2^62 and N up to 2^31 - 1: whenever the guard lets the estimate through, it
equals the exact integer floor, and the guard does let most estimates through.
"""
import math
import random


def estimate(N, c, CT):
    """The kernel's floor_estimate: the floor, or None for the exact path."""
    if c == 0:
        return 0
    scale = float(N) * (1.0 / float(CT))
    guard = float(N) * 2.0 ** -48
    x = float(c) * scale
    f = math.floor(x)
    r = x - f
    return f if guard < r < 1.0 - guard else None


def _cases(rng, n):
    for _ in range(n):
        N = rng.choice([1, 2, 3, 7, 100, 1091, 2621, 65535, rng.randint(2, 2 ** 31 - 1)])
        CT = rng.choice([rng.randint(1, 2 ** 20), rng.randint(1, 2 ** 40), rng.randint(2 ** 50, 2 ** 62)])
        yield N, rng.randint(0, CT), CT
        j = rng.randint(0, N)
        c0 = j * CT // N
        for dc in (-2, -1, 0, 1, 2):        # at and around a threshold
            if 0 <= c0 + dc <= CT:
                yield N, c0 + dc, CT
        yield N, CT, CT                      # the unit's last token


def test_estimate_is_exact_whenever_taken():
    rng = random.Random(20261203)
    taken = total = 0
    for N, c, CT in _cases(rng, 60000):
        q = estimate(N, c, CT)
        total += 1
        if q is not None:
            taken += 1
            assert q == N * c // CT, (N, c, CT, q)
    assert taken > total // 2


def test_exact_hits_go_to_the_exact_path():
    """N c / c_T an integer (a threshold hit exactly, c > 0): the estimate never decides alone."""
    rng = random.Random(7)
    for _ in range(20000):
        N = rng.randint(1, 5000)
        CT = N * rng.randint(1, 2 ** 40)
        j = rng.randint(1, N)
        assert estimate(N, j * CT // N, CT) is None
