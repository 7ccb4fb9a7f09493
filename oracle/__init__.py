"""CPU oracle for equal-variation KV coarsening and compressed decode attention.

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg import this module. The GPU library never imports
it, and it imports nothing from the GPU library.

The arithmetic lives in ``skv_oracle.c`` (plain C, fp64, built with gcc
``-ffp-contract=off``); this module builds it, marshals numpy arrays and runs
units on a thread pool (ctypes releases the GIL during each call).

Sources:
  [EV] "Equal-Variation KV Cache" (synthcore idea 664): Mathematical statement,
       Key formulas, Implementation notes, Verification.
  [SK] "SPICY-KV" demo page: section 2 (online-softmax kernel fusion) and
       Independent Claims 1-3.

Parity pins: every function here is pinned by tests under ``tests/`` against
published generator vectors, closed forms, textbook softmax attention, exact
rational arithmetic and brute force on small inputs (see test_oracle_*.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "skv_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

PROJ_DIM = 16
QUANT_SCALE = 2.0 ** 20
ORC_OK, ORC_ERR_ARG, ORC_ERR_OVERFLOW = 0, -1, -4


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile skv_oracle.c into oracle/_build/liboracle.so (gcc, -ffp-contract=off)."""
    os.makedirs(_BUILD, exist_ok=True)
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        i32, i64, u64, f32, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float, ctypes.c_double
        lib.orc_splitmix64_stream.argtypes = [u64, ctypes.c_int, P(u64)]
        lib.orc_splitmix64_stream.restype = None
        lib.orc_projection.argtypes = [u64, ctypes.c_int, ctypes.c_int, P(f32)]
        lib.orc_feature_f32.argtypes = [P(f32), P(f32), P(f32), ctypes.c_int, P(f32)]
        lib.orc_feature_f32.restype = None
        lib.orc_quantised_step.argtypes = [P(f32), P(f32), P(i64)]
        lib.orc_segment.argtypes = [P(i64), ctypes.c_int, ctypes.c_int, P(i32)]
        lib.orc_key_mean_f32.argtypes = [P(f32), ctypes.c_int, ctypes.c_int, P(f32)]
        lib.orc_split.argtypes = [ctypes.c_int] * 3 + [P(ctypes.c_int)] * 3
        lib.orc_coarsen_unit.argtypes = ([P(f32), P(f32)] + [ctypes.c_int] * 5 + [P(f32), P(i64), P(i64), P(f64),
                                         P(i32), P(i32), P(i32), P(f64), P(f64), P(f64), P(f64), P(f64), P(i32)])
        lib.orc_coarsen_unit2.argtypes = ([P(f32), P(f32)] + [ctypes.c_int] * 5 + [P(f32), ctypes.c_int, P(i64),
                                          P(i64), P(f64), P(i32), P(i32), P(i32), P(f64), P(f64), P(f64), P(f64),
                                          P(f64), P(f64), P(i32)])
        lib.orc_coarsen_unit_steps.argtypes = ([P(f32), P(f32)] + [ctypes.c_int] * 6 + [P(i64), P(i64), P(i64),
                                               P(i32), P(i32), P(i32), P(f64), P(f64), P(f64), P(f64), P(f64),
                                               P(f64), P(i32)])
        lib.orc_decode_rows2.argtypes = [P(f64), ctypes.c_int, ctypes.c_int, P(f64), P(f64), P(f64), P(f64),
                                         P(f64), ctypes.c_int, P(f64), P(f64)]
        lib.orc_decode_rows.argtypes = [P(f64), ctypes.c_int, ctypes.c_int, P(f64), P(f64), P(f64), P(f64),
                                        ctypes.c_int, P(f64), P(f64)]
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(rc: int, what: str):
    if rc == ORC_ERR_OVERFLOW:
        raise OracleError(f"{what}: variation overflow (d_t * 2^20 above 2^40, not finite, or M >= 2^22)")
    if rc != ORC_OK:
        raise OracleError(f"{what}: invalid argument (rc={rc})")


# --------------------------------------------------------------------------
# generator and projection
# --------------------------------------------------------------------------
def splitmix64_stream(seed: int, n: int) -> np.ndarray:
    out = np.zeros(n, dtype=np.uint64)
    _load().orc_splitmix64_stream(ctypes.c_uint64(seed), n, _ptr(out, ctypes.c_uint64))
    return out


def projection(seed: int, d: int) -> np.ndarray:
    """P: 16 x 2d fp32, N(0,1)/4 entries from SplitMix64 + Box-Muller ([EV] Implementation notes)."""
    P = np.zeros((PROJ_DIM, 2 * d), dtype=np.float32)
    _check(_load().orc_projection(ctypes.c_uint64(seed), PROJ_DIM, 2 * d, _ptr(P, ctypes.c_float)), "projection")
    return P


def feature_f32(P: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """z = P [k; v] of one token under the fixed fp32 recipe."""
    P = np.ascontiguousarray(P, np.float32)
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    z = np.zeros(PROJ_DIM, dtype=np.float32)
    _load().orc_feature_f32(_ptr(P, ctypes.c_float), _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float),
                            k.shape[0], _ptr(z, ctypes.c_float))
    return z


def quantised_step(zp: np.ndarray, zc: np.ndarray) -> int:
    """D = rne(||zc - zp||_2 * 2^20) under the fixed fp32 recipe."""
    zp = np.ascontiguousarray(zp, np.float32)
    zc = np.ascontiguousarray(zc, np.float32)
    out = np.zeros(1, dtype=np.int64)
    _check(_load().orc_quantised_step(_ptr(zp, ctypes.c_float), _ptr(zc, ctypes.c_float),
                                      _ptr(out, ctypes.c_int64)), "quantised_step")
    return int(out[0])


def segment(C: np.ndarray, N: int) -> np.ndarray:
    """Equal-variation boundaries b[0..N] from the cumulative integer variation C[0..M-1]."""
    C = np.ascontiguousarray(C, np.int64)
    M = C.shape[0]
    b = np.zeros(N + 1, dtype=np.int32)
    Cp = C if M > 0 else np.zeros(1, np.int64)
    _check(_load().orc_segment(_ptr(Cp, ctypes.c_int64), M, N, _ptr(b, ctypes.c_int32)), "segment")
    return b


def split(T: int, S: int, W: int):
    """(S_eff, W_eff, M): sinks first, then the recent window, then the middle."""
    s, w, m = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(_load().orc_split(T, S, W, ctypes.byref(s), ctypes.byref(w), ctypes.byref(m)), "split")
    return s.value, w.value, m.value


def key_mean_f32(k: np.ndarray) -> np.ndarray:
    """The unit's mean key mu [d] in the fixed fp32 order of reading R8 (common-mode mean removal,
    [SK] Independent Claim 1(b)): per dimension, blocks of 256 tokens summed in token order, block
    sums added in block order, total divided by T; all IEEE fp32."""
    k = np.ascontiguousarray(k, np.float32)
    T, d = k.shape
    mu = np.zeros(d, np.float32)
    kk = k if T > 0 else np.zeros((1, d), np.float32)
    _check(_load().orc_key_mean_f32(_ptr(kk, ctypes.c_float), T, d, _ptr(mu, ctypes.c_float)), "key_mean_f32")
    return mu


def center_keys(k: np.ndarray) -> np.ndarray:
    """Keys with the unit's mean key removed: fl32(k_ti - mu_i) (IEEE fp32 subtraction)."""
    k = np.ascontiguousarray(k, np.float32)
    return (k - key_mean_f32(k)[None, :]).astype(np.float32)


# --------------------------------------------------------------------------
# coarsening
# --------------------------------------------------------------------------
@dataclass
class UnitNodes:
    """Coarsened cache of one (sequence, KV head) unit, entries in order:
    sinks, nonempty middle segments, recents."""
    D: np.ndarray          # [M] int64 quantised variation (D[0] = 0)
    C: np.ndarray          # [M] int64 cumulative variation
    d64: np.ndarray        # [M] fp64 variation (information only)
    bounds: np.ndarray     # [N+1] int32 middle-local boundaries
    start: np.ndarray      # [E] int32 first token (unit-local) of each entry
    mass: np.ndarray       # [E] int32 member count m
    kt: np.ndarray         # [E, d] fp64 mean key
    vt: np.ndarray         # [E, d] fp64 mean value
    sigma2: np.ndarray     # [E] fp64 per-dimension key variance averaged over d
    var: np.ndarray        # [E, d] fp64 per-dimension key variance (the diagonal closure's vector)
    alpha: np.ndarray      # [E] fp64 ln m
    beta: np.ndarray       # [E] fp64 sigma2 / (2 d)
    s_eff: int
    w_eff: int
    M: int


REPRESENTATIVES = {"mean": 0, "variation": 1}


def coarsen_unit(k: np.ndarray, v: np.ndarray, n_sink: int, n_recent: int, N: int,
                 P: np.ndarray, representative: str = "mean", center: bool = False) -> UnitNodes:
    """Coarsen one unit: k, v [T, d] (any float dtype holding fp32-representable values).
    representative: "mean" (plain member mean, SPICY-KV Claim 2) or "variation" (the
    variation-weighted average of the Equal-Variation page's implementation notes, weights D_r;
    a segment without variation keeps the plain mean). center: coarsen the keys with the unit's
    mean key removed (center_keys; SPICY-KV Claim 1(b)); every key statistic, exact tokens
    included, is then of the centred keys."""
    rep = REPRESENTATIVES[representative]
    k = center_keys(k) if center else np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    P = np.ascontiguousarray(P, np.float32)
    T, d = k.shape
    s_eff, w_eff, M = split(T, n_sink, n_recent)
    Emax = s_eff + N + w_eff
    Mb = max(M, 1)
    D = np.zeros(Mb, np.int64)
    C = np.zeros(Mb, np.int64)
    d64 = np.zeros(Mb, np.float64)
    b = np.zeros(N + 1, np.int32)
    st = np.zeros(max(Emax, 1), np.int32)
    ln = np.zeros(max(Emax, 1), np.int32)
    kt = np.zeros((max(Emax, 1), d), np.float64)
    vt = np.zeros((max(Emax, 1), d), np.float64)
    s2 = np.zeros(max(Emax, 1), np.float64)
    vv_ = np.zeros((max(Emax, 1), d), np.float64)
    al = np.zeros(max(Emax, 1), np.float64)
    be = np.zeros(max(Emax, 1), np.float64)
    E = np.zeros(1, np.int32)
    kk = k if T > 0 else np.zeros((1, d), np.float32)
    vv = v if T > 0 else np.zeros((1, d), np.float32)
    f32p, i64p, i32p, f64p = (ctypes.c_float, ctypes.c_int64, ctypes.c_int32, ctypes.c_double)
    rc = _load().orc_coarsen_unit2(_ptr(kk, f32p), _ptr(vv, f32p), T, d, n_sink, n_recent, N, _ptr(P, f32p), rep,
                                   _ptr(D, i64p), _ptr(C, i64p), _ptr(d64, f64p), _ptr(b, i32p), _ptr(st, i32p),
                                   _ptr(ln, i32p), _ptr(kt, f64p), _ptr(vt, f64p), _ptr(vv_, f64p), _ptr(s2, f64p),
                                   _ptr(al, f64p), _ptr(be, f64p), _ptr(E, i32p))
    _check(rc, "coarsen_unit")
    e = int(E[0])
    return UnitNodes(D[:M].copy(), C[:M].copy(), d64[:M].copy(), b, st[:e].copy(), ln[:e].copy(),
                     kt[:e].copy(), vt[:e].copy(), s2[:e].copy(), vv_[:e].copy(), al[:e].copy(), be[:e].copy(), s_eff, w_eff, M)


def coarsen_unit_from_steps(k: np.ndarray, v: np.ndarray, n_sink: int, n_recent: int, N: int, D: np.ndarray,
                            representative: str = "mean", center: bool = False) -> UnitNodes:
    """coarsen_unit with the middle tokens' quantised steps D [M] given (int64, D[0] = 0) instead of
    the fixed fp32 recipe: prefix sums, first-hitting boundaries and node statistics follow D. The
    stage-wise check of steps computed another way (the tensor-core projection option)."""
    rep = REPRESENTATIVES[representative]
    k = center_keys(k) if center else np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    T, d = k.shape
    s_eff, w_eff, M = split(T, n_sink, n_recent)
    D_in = np.ascontiguousarray(D, np.int64)
    if D_in.shape != (M,):
        raise ValueError(f"D must have the middle's {M} steps")
    Emax = s_eff + N + w_eff
    Mb = max(M, 1)
    Dout = np.zeros(Mb, np.int64)
    C = np.zeros(Mb, np.int64)
    b = np.zeros(N + 1, np.int32)
    E1 = max(Emax, 1)
    st, ln = np.zeros(E1, np.int32), np.zeros(E1, np.int32)
    kt, vt, vv_ = np.zeros((E1, d)), np.zeros((E1, d)), np.zeros((E1, d))
    s2, al, be = np.zeros(E1), np.zeros(E1), np.zeros(E1)
    E = np.zeros(1, np.int32)
    kk = k if T > 0 else np.zeros((1, d), np.float32)
    vv = v if T > 0 else np.zeros((1, d), np.float32)
    Dp = D_in if M > 0 else np.zeros(1, np.int64)
    f32p, i64p, i32p, f64p = (ctypes.c_float, ctypes.c_int64, ctypes.c_int32, ctypes.c_double)
    rc = _load().orc_coarsen_unit_steps(_ptr(kk, f32p), _ptr(vv, f32p), T, d, n_sink, n_recent, N, rep,
                                        _ptr(Dp, i64p), _ptr(Dout, i64p), _ptr(C, i64p), _ptr(b, i32p), _ptr(st, i32p),
                                        _ptr(ln, i32p), _ptr(kt, f64p), _ptr(vt, f64p), _ptr(vv_, f64p), _ptr(s2, f64p),
                                        _ptr(al, f64p), _ptr(be, f64p), _ptr(E, i32p))
    _check(rc, "coarsen_unit_from_steps")
    e = int(E[0])
    return UnitNodes(Dout[:M].copy(), C[:M].copy(), np.zeros(M), b, st[:e].copy(), ln[:e].copy(), kt[:e].copy(),
                     vt[:e].copy(), s2[:e].copy(), vv_[:e].copy(), al[:e].copy(), be[:e].copy(), s_eff, w_eff, M)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 (ties to even), returned as fp32 (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(np.shape(x))


def projection_bf16(seed: int, d: int) -> np.ndarray:
    """P16 = bf16(P): the projection of the tensor-core option (SKV_PROJECTION_TENSOR_BF16)."""
    return bf16_round(projection(seed, d))


def tensor_steps_reference(k: np.ndarray, v: np.ndarray, n_sink: int, n_recent: int, P16: np.ndarray,
                           mma_k_steps: int | None = None):
    """The tensor-core option's steps against the exact P16 projection. Returns (d, bound), both
    [M] fp64 in units of 2^-20: d the exact step ||P16 (x_t - x_{t-1})|| * 2^20 of the middle tokens
    (x = [k; v]; every product of a bf16 feature and a bf16 entry is exact in fp64 and 2d of them
    sum with fp64 error far below the bound), and bound a limit on |D_t - d_t| for any fp32
    accumulation of those products in at most `mma_k_steps` (default 2d/16) accumulate steps of 16
    products each, rounding or truncating every step to fp32 (error at most 18 units of 2^-23 of
    the sum of magnitudes per step), followed by the fixed recipe's fp32 difference, square sum,
    square root and rne quantisation."""
    k = np.ascontiguousarray(k, np.float32).astype(np.float64)
    v = np.ascontiguousarray(v, np.float32).astype(np.float64)
    T, d = k.shape
    s_eff, w_eff, M = split(T, n_sink, n_recent)
    x = np.concatenate([k, v], axis=1)[s_eff:s_eff + M]
    P = np.asarray(P16, np.float64)
    z = x @ P.T
    S = np.abs(x) @ np.abs(P).T                    # sum of magnitudes per token and output
    nks = mma_k_steps if mma_k_steps is not None else 2 * d // 16
    e = nks * 18.0 * 2.0 ** -23 * S                # per-output accumulation bound
    dd = np.zeros(M)
    bound = np.zeros(M)
    if M > 1:
        dz = z[1:] - z[:-1]
        dd[1:] = np.sqrt((dz * dz).sum(axis=1))
        err_z = np.sqrt(((e[1:] + e[:-1]) ** 2).sum(axis=1))
        # fp32 difference, 16 fma steps, sqrt and scaling: a few dozen units of 2^-24 of d
        bound[1:] = (err_z + 64 * 2.0 ** -24 * (dd[1:] + err_z)) * 2.0 ** 20 + 1.0
    return dd * 2.0 ** 20, bound


def _pool(threads: int | None):
    return ThreadPoolExecutor(max_workers=threads or os.cpu_count() or 1)


def coarsen(seqs, n_sink: int, n_recent: int, N_list, seed: int, threads: int | None = None,
            representative: str = "mean", center: bool = False):
    """Coarsen a batch. seqs: list over sequences b of (k_b, v_b) arrays [Hkv, T_b, d].
    Returns nested list [b][h] of UnitNodes. The projection P is drawn from ``seed``."""
    d = seqs[0][0].shape[-1]
    P = projection(seed, d)
    jobs = [(b, h) for b in range(len(seqs)) for h in range(seqs[b][0].shape[0])]
    res = {}
    with _pool(threads) as ex:
        futs = {ex.submit(coarsen_unit, seqs[b][0][h], seqs[b][1][h], n_sink, n_recent, int(N_list[b]), P,
                          representative, center): (b, h)
                for (b, h) in jobs}
        for f, key in futs.items():
            res[key] = f.result()
    return [[res[(b, h)] for h in range(seqs[b][0].shape[0])] for b in range(len(seqs))]


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------
def decode_rows(q: np.ndarray, kt: np.ndarray, vt: np.ndarray, alpha: np.ndarray, beta: np.ndarray,
                var: np.ndarray | None = None):
    """Compressed decode attention of query rows q [rows, d] against one unit's entries.
    var [E, d] (optional): per-dimension key variances for the diagonal closure
    sum_i q_i^2 var_i / (2d) in place of |q|^2 beta.
    Returns (out [rows, d] fp64, lse [rows] fp64, natural log)."""
    q = np.ascontiguousarray(q, np.float64)
    rows, d = q.shape
    E = kt.shape[0]
    if E > 0:
        kt = np.ascontiguousarray(kt, np.float64)
        vt = np.ascontiguousarray(vt, np.float64)
        al = np.ascontiguousarray(alpha, np.float64)
        be = np.ascontiguousarray(beta, np.float64)
        va = np.ascontiguousarray(var, np.float64) if var is not None else None
    else:
        kt, vt, al, be = np.zeros((1, d)), np.zeros((1, d)), np.zeros(1), np.zeros(1)
        va = np.zeros((1, d)) if var is not None else None
    out = np.zeros((max(rows, 1), d), np.float64)
    lse = np.zeros(max(rows, 1), np.float64)
    qq = q if rows > 0 else np.zeros((1, d))
    f64p = ctypes.c_double
    vp = _ptr(va, f64p) if va is not None else None
    _check(_load().orc_decode_rows2(_ptr(qq, f64p), rows, d, _ptr(kt, f64p), _ptr(vt, f64p), _ptr(al, f64p),
                                    _ptr(be, f64p), vp, E, _ptr(out, f64p), _ptr(lse, f64p)), "decode_rows")
    return out[:rows], lse[:rows]


def decode(q: np.ndarray, units, threads: int | None = None, closure: str = "scalar"):
    """Decode a batch. q [B, R, Hq, d]; units[b][h] supplies (kt, vt, alpha, beta) for KV head h
    (a UnitNodes or any object with those attributes; `var` too for closure="diagonal"). Query head
    hq reads KV head hq // G. Returns out [B, R, Hq, d] fp64 and lse [B, R, Hq] fp64."""
    if closure not in ("scalar", "diagonal"):
        raise ValueError("closure must be 'scalar' or 'diagonal'")
    B, R, Hq, d = q.shape
    Hkv = len(units[0])
    G = Hq // Hkv
    out = np.zeros((B, R, Hq, d), np.float64)
    lse = np.zeros((B, R, Hq), np.float64)

    def one(b, h):
        rows = q[b, :, h * G:(h + 1) * G, :].reshape(R * G, d)
        u = units[b][h]
        o, l = decode_rows(rows, u.kt, u.vt, u.alpha, u.beta, u.var if closure == "diagonal" else None)
        out[b, :, h * G:(h + 1) * G, :] = o.reshape(R, G, d)
        lse[b, :, h * G:(h + 1) * G] = l.reshape(R, G)

    with _pool(threads) as ex:
        list(ex.map(lambda bh: one(*bh), [(b, h) for b in range(B) for h in range(Hkv)]))
    return out, lse


# --------------------------------------------------------------------------
# step reconstruction ([EV] Mathematical statement and Key formulas)
# --------------------------------------------------------------------------
def variation_boundaries(path: np.ndarray, N: int):
    """Equal-variation breakpoints of a sampled path [n] or [n, dim] (fp64 Euclidean
    increments, quantised at 2^20 and segmented by first hitting). Returns (bounds, D)."""
    x = np.asarray(path, np.float64)
    if x.ndim == 1:
        x = x[:, None]
    inc = np.zeros(x.shape[0])
    inc[1:] = np.sqrt(((x[1:] - x[:-1]) ** 2).sum(axis=1))
    D = np.rint(inc * QUANT_SCALE).astype(np.int64)
    return segment(np.cumsum(D), N), D


def step_reconstruction(path: np.ndarray, N: int, representative: str = "left"):
    """Piecewise-constant reconstruction of a sampled path from its equal-variation segments.
    representative: 'left' = the value at the segment's first sample (the pages' decoder
    pi_N(t) = pi(t_j)); 'midrange' = centre of the segment's bounding box; 'mean' = member
    mean (the node's representative). Returns (reconstruction, sup-norm error, total variation)."""
    x = np.asarray(path, np.float64)
    flat = x.ndim == 1
    if flat:
        x = x[:, None]
    b, D = variation_boundaries(x, N)
    rec = np.empty_like(x)
    for j in range(N):
        lo, hi = int(b[j]), int(b[j + 1])
        if hi <= lo:
            continue
        seg = x[lo:hi]
        if representative == "left":
            r = seg[0]
        elif representative == "midrange":
            r = 0.5 * (seg.min(axis=0) + seg.max(axis=0))
        elif representative == "mean":
            r = seg.mean(axis=0)
        else:
            raise ValueError(representative)
        rec[lo:hi] = r
    err = float(np.sqrt(((x - rec) ** 2).sum(axis=1)).max()) if x.shape[0] else 0.0
    total = float(np.sqrt(((x[1:] - x[:-1]) ** 2).sum(axis=1)).sum()) if x.shape[0] > 1 else 0.0
    return (rec[:, 0] if flat else rec), err, total
