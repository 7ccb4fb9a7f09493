"""Streaming (incremental) equal-variation coarsening -- oracle (test infrastructure only).

"Equal-Variation KV Cache", "Implementation notes": in streaming inference a segment that exceeds
its variation budget is split at the first threshold crossing and adjacent low-variation segments
are merged when necessary; the page leaves the policy open. Node merges follow the law of total
variance ("SPICY-KV", dependent Claim 10). Readings this module fixes:

 S1  A unit starts from the offline coarsening of its first T tokens (T > n_sink + n_recent, so the
     middle is not empty); its middle nodes are kept in token order, the last one is "open".
 S2  Appending a token slides the recent window: the oldest recent token y enters the middle and
     the new token becomes the newest recent token (sinks never change).
 S3  y's variation step D_y uses the offline fixed fp32 recipe against the previous middle token;
     the running total c_T grows by D_y.
 S4  First hitting on the open segment's budget c_T / N: if N (V_open + D_y) >= c_T (exact
     integers), y starts a new open segment (with V = D_y); otherwise y joins the open segment.
 S5  While there are more than N middle nodes, the adjacent pair with the smallest V_j + V_{j+1}
     merges (the leftmost on ties): m, mean key, mean value and the summed squared deviations M2
     combine exactly (Chan et al.'s pairwise update), V adds; a merge with the open node stays open.
 S6  Node outputs as offline: alpha = ln m, sigma^2 = M2 / (m d), beta = sigma^2 / (2 d).

Statistics are fp64 from the fp32 values of the tokens; every decision (split, merge choice) is an
exact integer comparison."""
from __future__ import annotations

import numpy as np

from . import coarsen_unit, feature_f32, quantised_step, split


class _Node:
    __slots__ = ("start", "m", "V", "mk", "mv", "M2")

    def __init__(self, start, m, V, mk, mv, M2):
        self.start, self.m, self.V, self.mk, self.mv, self.M2 = int(start), int(m), int(V), mk, mv, float(M2)


def _merge(a: _Node, b: _Node) -> _Node:
    """Pairwise combination of two adjacent nodes (law of total variance)."""
    m = a.m + b.m
    dk = b.mk - a.mk
    mk = a.mk + dk * (b.m / m)
    mv = a.mv + (b.mv - a.mv) * (b.m / m)
    M2 = a.M2 + b.M2 + float(dk @ dk) * a.m * b.m / m
    return _Node(a.start, m, a.V + b.V, mk, mv, M2)


class StreamUnit:
    """One (sequence, KV head) unit under streaming coarsening."""

    def __init__(self, k: np.ndarray, v: np.ndarray, n_sink: int, n_recent: int, N: int, P: np.ndarray):
        k = np.ascontiguousarray(k, np.float32)
        v = np.ascontiguousarray(v, np.float32)
        T, d = k.shape
        s_eff, w_eff, M = split(T, n_sink, n_recent)
        if M < 1 or s_eff != n_sink or w_eff != n_recent:
            raise ValueError("streaming starts from a unit with a non-empty middle")
        self.S, self.W, self.N, self.d, self.P = n_sink, n_recent, int(N), d, P
        self.T = T
        u = coarsen_unit(k, v, n_sink, n_recent, N, P)
        self.nodes = []
        b = u.bounds
        for j in range(N):
            if b[j + 1] > b[j]:
                st, m = n_sink + int(b[j]), int(b[j + 1] - b[j])
                kk = k[st:st + m].astype(np.float64)
                vv = v[st:st + m].astype(np.float64)
                mk = kk.mean(axis=0)
                self.nodes.append(_Node(st, m, int(u.D[b[j]:b[j + 1]].sum()), mk, vv.mean(axis=0),
                                        float(((kk - mk) ** 2).sum())))
        self.cT = int(u.C[-1])
        self.z_last = feature_f32(P, k[n_sink + M - 1], v[n_sink + M - 1])
        self.sink_k, self.sink_v = k[:n_sink].copy(), v[:n_sink].copy()
        self.rec_k = [k[T - n_recent + r].copy() for r in range(n_recent)]
        self.rec_v = [v[T - n_recent + r].copy() for r in range(n_recent)]
        self.splits = 0
        self.merges = 0

    def append(self, k_new: np.ndarray, v_new: np.ndarray):
        ky, vy = self.rec_k.pop(0), self.rec_v.pop(0)          # S2: the oldest recent token enters
        self.rec_k.append(np.asarray(k_new, np.float32).copy())
        self.rec_v.append(np.asarray(v_new, np.float32).copy())
        y_pos = self.T - self.W
        z = feature_f32(self.P, ky, vy)                          # S3
        D = quantised_step(self.z_last, z)
        self.z_last = z
        self.cT += D
        last = self.nodes[-1]
        ky64, vy64 = ky.astype(np.float64), vy.astype(np.float64)
        if self.N * (last.V + D) >= self.cT:                     # S4: y starts a new segment
            self.nodes.append(_Node(y_pos, 1, D, ky64, vy64, 0.0))
            self.splits += 1
        else:
            grown = _merge(last, _Node(y_pos, 1, 0, ky64, vy64, 0.0))
            grown.V = last.V + D
            self.nodes[-1] = grown
        while len(self.nodes) > self.N:                          # S5
            sums = [self.nodes[j].V + self.nodes[j + 1].V for j in range(len(self.nodes) - 1)]
            j = int(np.argmin(sums))                             # first minimum: leftmost on ties
            self.nodes[j:j + 2] = [_merge(self.nodes[j], self.nodes[j + 1])]
            self.merges += 1
        self.T += 1

    def entries(self):
        """(start, m, kt, vt, alpha, beta) of every entry: sinks, middle nodes, recents (S6)."""
        d = self.d
        out = []
        for t in range(self.S):
            out.append((t, 1, self.sink_k[t].astype(np.float64), self.sink_v[t].astype(np.float64), 0.0, 0.0))
        for n in self.nodes:
            s2 = n.M2 / (n.m * d)
            out.append((n.start, n.m, n.mk.copy(), n.mv.copy(), float(np.log(n.m)), s2 / (2 * d)))
        for r in range(self.W):
            out.append((self.T - self.W + r, 1, self.rec_k[r].astype(np.float64), self.rec_v[r].astype(np.float64),
                        0.0, 0.0))
        return out

    def arrays(self):
        """The entries as arrays kt [E, d], vt [E, d], alpha [E], beta [E] (decode's inputs)."""
        e = self.entries()
        return (np.stack([x[2] for x in e]), np.stack([x[3] for x in e]), np.array([x[4] for x in e]),
                np.array([x[5] for x in e]))
