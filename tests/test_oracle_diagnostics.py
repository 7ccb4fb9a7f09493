"""Attention diagnostics of the compressed cache against full attention (oracle only, fp64):
output MSE, output cosine and the partition ratio Z/Z_full, for equal-variation segments with the
plain-mean representative, equal-variation segments with the variation-weighted representative
("Equal-Variation KV Cache", "Implementation notes" and "Verification": the page reports that
attention-output MSE generally favoured uniform compression), and uniform segments with the plain
mean, each with and without the variance closure ("SPICY-KV" section 2, Claim 3).

These are measurements, not parity gates. What the mathematics fixes is asserted per query row:
with plain-mean nodes the mass-only partition cannot exceed the full one (Jensen: m exp(q.mean/sqrt d)
<= sum_r exp(q.k_r/sqrt d) for every segment), and the closure (beta >= 0) can only raise it. The
numbers are printed with -s."""
import numpy as np
import pytest

import oracle
import workloads

S, W = workloads.N_SINK, workloads.N_RECENT


def _uniform_nodes(k, v, n_sink, n_recent, N):
    """Uniform segmentation of the middle into N equal-length runs (the page's baseline), plain
    member mean and population variance; exact tokens as in the method."""
    T, d = k.shape
    s_eff, w_eff, M = oracle.split(T, n_sink, n_recent)
    b = [(j * M) // N for j in range(N + 1)]
    ents = [(t, 1) for t in range(s_eff)]
    ents += [(s_eff + b[j], b[j + 1] - b[j]) for j in range(N) if b[j + 1] > b[j]]
    ents += [(s_eff + M + t, 1) for t in range(w_eff)]
    kt = np.stack([k[s:s + m].mean(axis=0) for s, m in ents])
    vt = np.stack([v[s:s + m].mean(axis=0) for s, m in ents])
    var = np.array([k[s:s + m].var(axis=0).mean() for s, m in ents])
    mass = np.array([m for _, m in ents], np.float64)
    return kt, vt, np.log(mass), var / (2 * d)


def _full(q, k, v):
    s = q @ k.T / np.sqrt(k.shape[1])
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    z = p.sum(axis=1, keepdims=True)
    return (p / z) @ v, (mx + np.log(z))[:, 0]


def _metrics(out, lse, ref_out, ref_lse):
    mse = float(np.mean((out - ref_out) ** 2))
    cos = float(np.mean(np.sum(out * ref_out, axis=1) /
                        (np.linalg.norm(out, axis=1) * np.linalg.norm(ref_out, axis=1))))
    zr = float(np.mean(np.exp(lse - ref_lse)))
    return mse, cos, zr


@pytest.mark.parametrize("values", ["normal", "walk"])
def test_attention_diagnostics_equal_variation_vs_uniform(values):
    w = workloads.WORKLOADS["gqa6_10k5_prefill_decode"]
    k_all, v_all, T_list = workloads.make_kv(w, "cpu", values=values)
    q_all = workloads.make_queries(w, "cpu").double().numpy()        # [1, R, Hq, d]
    T, N, d = T_list[0], int(workloads.segment_counts(w, T_list)[0]), w.d
    P = oracle.projection(w.seed, d)
    rows = []
    for h in range(w.Hkv):
        k = workloads.unit_rows(k_all, T_list, w.Hkv, 0, h).float().numpy().astype(np.float64)
        v = workloads.unit_rows(v_all, T_list, w.Hkv, 0, h).float().numpy().astype(np.float64)
        G = w.Hq // w.Hkv
        q = q_all[0, :, h * G:(h + 1) * G].reshape(-1, d)
        ref_out, ref_lse = _full(q, k, v)
        k32, v32 = k.astype(np.float32), v.astype(np.float32)
        ev = oracle.coarsen_unit(k32, v32, S, W, N, P)
        evw = oracle.coarsen_unit(k32, v32, S, W, N, P, representative="variation")
        uni = _uniform_nodes(k, v, S, W, N)
        cases = {"equal-variation, mean": (ev.kt, ev.vt, ev.alpha, ev.beta),
                 "equal-variation, weighted": (evw.kt, evw.vt, evw.alpha, evw.beta),
                 "uniform, mean": uni}
        for name, (kt, vt, al, be) in cases.items():
            lses = {}
            for closure in (True, False):
                out, lse = oracle.decode_rows(q, kt, vt, al, be if closure else np.zeros_like(be))
                rows.append((h, name, closure) + _metrics(out, lse, ref_out, ref_lse))
                lses[closure] = lse
            assert np.all(lses[True] >= lses[False] - 1e-12), name
            if name.endswith("mean"):
                assert np.all(lses[False] <= ref_lse + 1e-9), f"{name}: Jensen"
    print(f"\n[{values} values] T={T} N={N} entries/unit={ev.kt.shape[0]}")
    for h, name, closure, mse, cos, zr in rows:
        print(f"  head {h} {name:26s} closure={closure!s:5s} MSE {mse:.3e} cos {cos:.4f} Z/Zfull {zr:.4f}")
        assert np.isfinite(mse) and cos > 0.5 and 0.05 < zr < 20
