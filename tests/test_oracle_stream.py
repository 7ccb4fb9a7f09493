"""Oracle pins of streaming coarsening (oracle/stream.py, readings S1-S6): after every append the
middle nodes tile the middle span in order (masses add up, starts are contiguous), their variations
add up to c_T exactly, there are at most N of them, and each node's statistics equal numpy's direct
ones over its members (which pins the pairwise merge); N = 1 keeps one node over the whole middle;
a large jump entering the middle starts a new node exactly at the jump. The split and merge
decisions (readings S3-S5) match an independent replay over (start, m, V) after every append, on
random walks and on caches whose steps repeat exactly (ties between pair sums), and the split
rule is checked at its boundary (N (V_open + D) equal to c_T after the step, and one less)."""
import numpy as np
import pytest

import oracle
from oracle.stream import StreamUnit

S, W = 8, 48


def _walk(T, d, seed, jump_at=None):
    rng = np.random.default_rng(seed)
    k = np.cumsum(rng.standard_normal((T, d)) * 0.05, axis=0) + rng.standard_normal((T, d)) * 0.02
    v = rng.standard_normal((T, d))
    if jump_at is not None:
        k[jump_at:] += 40.0
    return k.astype(np.float32), v.astype(np.float32)


def _check_invariants(u: StreamUnit, k, v):
    M = u.T - S - W
    assert len(u.nodes) <= u.N
    assert u.nodes[0].start == S
    for a, b in zip(u.nodes, u.nodes[1:]):
        assert b.start == a.start + a.m
    assert u.nodes[-1].start + u.nodes[-1].m == S + M
    assert sum(n.V for n in u.nodes) == u.cT
    for n in u.nodes:
        kk = k[n.start:n.start + n.m].astype(np.float64)
        vv = v[n.start:n.start + n.m].astype(np.float64)
        np.testing.assert_allclose(n.mk, kk.mean(axis=0), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(n.mv, vv.mean(axis=0), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(n.M2, ((kk - kk.mean(axis=0)) ** 2).sum(), rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("N", [1, 7, 40])
def test_stream_invariants_over_many_appends(N):
    T0, extra, d = 600, 400, 64
    k, v = _walk(T0 + extra, d, seed=N)
    P = oracle.projection(3, d)
    u = StreamUnit(k[:T0], v[:T0], S, W, N, P)
    _check_invariants(u, k, v)
    for t in range(T0, T0 + extra):
        u.append(k[t], v[t])
        if t % 37 == 0 or t == T0 + extra - 1:
            _check_invariants(u, k, v)
    if N == 1:
        assert len(u.nodes) == 1 and u.nodes[0].m == T0 + extra - S - W
    else:
        assert u.splits > 0 and u.merges > 0
    # the entries are sinks, middle nodes, recents, in token order
    e = u.entries()
    assert [x[0] for x in e[:S]] == list(range(S))
    assert [x[0] for x in e[-W:]] == list(range(u.T - W, u.T))
    assert sum(x[1] for x in e) == u.T


def test_variation_steps_match_the_offline_recipe():
    """c_T after streaming equals the offline cumulative variation of the whole middle: every step
    uses the same fixed fp32 recipe on the same consecutive tokens."""
    T0, extra, d = 300, 250, 128
    k, v = _walk(T0 + extra, d, seed=5)
    P = oracle.projection(8, d)
    u = StreamUnit(k[:T0], v[:T0], S, W, 20, P)
    for t in range(T0, T0 + extra):
        u.append(k[t], v[t])
    full = oracle.coarsen_unit(k, v, S, W, 20, P)
    assert u.cT == int(full.C[-1])


def test_jump_starts_a_new_node():
    T0, d = 400, 64
    jump = T0 + 100 + W          # this token enters the middle at the 101st append... after 100 more
    k, v = _walk(T0 + 200 + W, d, seed=9, jump_at=jump)
    P = oracle.projection(2, d)
    u = StreamUnit(k[:T0], v[:T0], S, W, 30, P)
    for t in range(T0, T0 + 200 + W):
        u.append(k[t], v[t])
    assert any(n.start == jump for n in u.nodes)
    _check_invariants(u, k, v)


def _replay_decisions(nodes, cT, N, steps, first_token):
    """Readings S3-S5 restated over (start, m, V) triples alone: c_T grows by the step, the token
    opens a new segment when N (V_open + D) >= c_T and joins the open one otherwise, and while more
    than N segments remain the adjacent pair with the smallest summed variation (leftmost on ties)
    becomes one."""
    segs = [tuple(x) for x in nodes]
    for i, D in enumerate(steps):
        tok = first_token + i
        cT += D
        start, m, V = segs[-1]
        segs = segs + [(tok, 1, D)] if N * (V + D) >= cT else segs[:-1] + [(start, m + 1, V + D)]
        while len(segs) > N:
            pair = min(range(len(segs) - 1), key=lambda j: (segs[j][2] + segs[j + 1][2], j))
            (s0, m0, v0), (_, m1, v1) = segs[pair], segs[pair + 1]
            segs = segs[:pair] + [(s0, m0 + m1, v0 + v1)] + segs[pair + 2:]
    return segs, cT


@pytest.mark.parametrize("N,seed,jumps", [(1, 11, ()), (2, 12, (700,)), (5, 13, (650, 820)), (40, 14, ()),
                                          (40, 15, (620, 640, 900)), (300, 16, (700,))])
def test_split_and_merge_decisions_match_a_brute_force_replay(N, seed, jumps):
    """After every append the oracle's segments (start, m, V) and c_T equal an independent replay of
    the split and merge rules fed the same quantised steps (the steps come from the pinned fixed
    fp32 recipe). Plausible slips -- '>' for '>=', comparing V_open without the new step, c_T before
    the step, the single smallest V instead of the smallest pair, the rightmost tie -- change the
    segments on these walks."""
    T0, extra, d = 600, 420, 64
    k, v = _walk(T0 + extra, d, seed=seed)
    for j in jumps:
        k[j:] += 6.0
    P = oracle.projection(seed, d)
    u = StreamUnit(k[:T0], v[:T0], S, W, N, P)
    segs = [(n.start, n.m, n.V) for n in u.nodes]
    cT = u.cT
    first = T0 - W                                   # the token that enters the middle first
    z_prev = oracle.feature_f32(P, k[first - 1], v[first - 1])
    saw_split = saw_merge = False
    for i in range(extra):
        tok = first + i
        z = oracle.feature_f32(P, k[tok], v[tok])
        D = oracle.quantised_step(z_prev, z)
        z_prev = z
        splits, merges = u.splits, u.merges
        u.append(k[T0 + i], v[T0 + i])
        segs, cT = _replay_decisions(segs, cT, N, [D], tok)
        assert [(n.start, n.m, n.V) for n in u.nodes] == segs, f"append {i}"
        assert u.cT == cT
        saw_split |= u.splits > splits
        saw_merge |= u.merges > merges
    if N > 1:
        assert saw_split and saw_merge


def _periodic(T, d, seed, flat):
    """Tokens alternating between two fixed vectors, so every variation step is the same integer D
    (the fp32 differences of a pair are exact negatives of each other), except a run `flat` of one
    repeated token (steps 0). All c_T and V are then multiples of D: exact equalities
    N (V_open + D) = c_T and exact ties between adjacent pair sums occur throughout."""
    rng = np.random.default_rng(seed)
    a, b = rng.standard_normal((2, 2, d)).astype(np.float32)
    k = np.empty((T, d), np.float32)
    v = np.empty((T, d), np.float32)
    for t in range(T):
        src = a if (t % 2 == 0 or t in flat) else b
        k[t], v[t] = src[0], src[1]
    return k, v


@pytest.mark.parametrize("N", [2, 3, 4, 7, 12, 40])
def test_split_and_merge_decisions_on_exact_ties(N):
    """The replay above on caches whose steps repeat exactly: splits at N (V_open + D) = c_T and
    merges among equal pair sums decide the segments, so '>' for '>=', c_T taken before the step and
    the rightmost tie each give different segments."""
    T0, extra, d = 300, 500, 32
    k, v = _periodic(T0 + extra, d, seed=N, flat=range(T0 + 200, T0 + 260))
    P = oracle.projection(N + 100, d)
    u = StreamUnit(k[:T0], v[:T0], S, W, N, P)
    segs = [(n.start, n.m, n.V) for n in u.nodes]
    cT = u.cT
    first = T0 - W
    z_prev = oracle.feature_f32(P, k[first - 1], v[first - 1])
    for i in range(extra):
        tok = first + i
        z = oracle.feature_f32(P, k[tok], v[tok])
        D = oracle.quantised_step(z_prev, z)
        z_prev = z
        u.append(k[T0 + i], v[T0 + i])
        segs, cT = _replay_decisions(segs, cT, N, [D], tok)
        assert [(n.start, n.m, n.V) for n in u.nodes] == segs, f"append {i}"
        assert u.cT == cT


@pytest.mark.parametrize("N", [2, 5, 40])
def test_split_rule_at_its_boundary(N):
    """Reading S4 at its boundary, with the unit's open-node variation and c_T set so that the test
    knows the exact comparison: N (V_open + D) equal to c_T after the step splits ('>=', and c_T
    includes the step); one less does not split. D is the fixed-recipe step of the token that
    enters the middle."""
    T0, d = 300, 32
    k, v = _walk(T0 + 1, d, seed=N + 40)
    P = oracle.projection(N + 40, d)
    y = T0 - W                                            # the token that enters the middle
    D = oracle.quantised_step(oracle.feature_f32(P, k[y - 1], v[y - 1]), oracle.feature_f32(P, k[y], v[y]))
    assert D > 0
    V_open = 1_000_003
    for slack, splits in ((0, True), (1, False)):
        u = StreamUnit(k[:T0], v[:T0], S, W, N, P)
        u.nodes[-1].V = V_open
        u.cT = N * (V_open + D) - D + slack               # so that N (V_open + D) = c_T + D - slack
        u.append(k[T0], v[T0])
        assert u.splits == (1 if splits else 0), f"slack {slack}"
        assert u.cT == N * (V_open + D) + slack
