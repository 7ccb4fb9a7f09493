"""Oracle pins of streaming coarsening (oracle/stream.py, readings S1-S6): after every append the
middle nodes tile the middle span in order (masses add up, starts are contiguous), their variations
add up to c_T exactly, there are at most N of them, and each node's statistics equal numpy's direct
ones over its members (which pins the pairwise merge); N = 1 keeps one node over the whole middle;
a large jump entering the middle starts a new node exactly at the jump."""
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
