"""Helpers shared by the GPU parity tests: pool / page-table set-up, writing synthetic
entries into the pool layout, reading GPU nodes back for the oracle, and the
tolerance checks the parity bar fixes:
  fp32: relative L2 <= 1e-5;
  bf16: relative L2 <= 5e-3 and max-abs <= 2e-2 on outputs, |lse error| <= 1e-3.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import compressed_decode_attention_equal_b200 as skv
import workloads

TOL_F32_REL_L2 = 1e-5
TOL_BF16_REL_L2 = 5e-3
TOL_BF16_MAX_ABS = 2e-2
TOL_LSE_ABS = 1e-3


def pool_for_units(entries_per_unit, B, Hkv, d, dtype, shuffle=False, seed=0, spare_pages=0, device="cuda",
                   closure="scalar"):
    """Pool and page table with ceil(E/16) pages for each unit (entries_per_unit[b] per head)."""
    pages = [max(1, -(-int(e) // skv.PAGE_NODES)) for e in entries_per_unit]
    table, total = workloads.page_assignment(B, Hkv, pages, shuffle, seed)
    pool = skv.NodePool(total + spare_pages, d, dtype, device=device, closure=closure)
    # slots no entry uses hold NaN: a kernel that lets them leak into a result fails the checks
    pool.k.fill_(float("nan"))
    pool.v.fill_(float("nan"))
    pool.ab.fill_(float("nan"))
    if pool.var is not None:
        pool.var.fill_(float("nan"))
    return pool, table.to(device)


def write_entries(pool, table, b, h, kt, vt, alpha, beta, var=None):
    """Write entries of unit (b, h) into the pool's swizzled page layout (inverse of read_entries)."""
    E, d = kt.shape
    if E == 0:
        return
    dev = pool.k.device
    pg, sl = skv._entry_rows(pool, table, b, h, E)
    epc = 16 // pool.k.element_size()
    ch = d // epc
    phys = torch.arange(ch, device=dev)[None, :] ^ (sl[:, None] & 7)
    k4 = pool.k.view(pool.num_pages, skv.PAGE_NODES, ch, epc)
    v4 = pool.v.view(pool.num_pages, skv.PAGE_NODES, ch, epc)
    k4[pg[:, None], sl[:, None], phys] = kt.to(pool.dtype).reshape(E, ch, epc).to(dev)
    v4[pg[:, None], sl[:, None], phys] = vt.to(pool.dtype).reshape(E, ch, epc).to(dev)
    pool.ab[pg, sl, 0] = alpha.float().to(dev)
    pool.ab[pg, sl, 1] = beta.float().to(dev)
    if var is not None:
        r4 = pool.var.view(pool.num_pages, skv.PAGE_NODES, ch, epc)
        r4[pg[:, None], sl[:, None], phys] = var.to(pool.dtype).reshape(E, ch, epc).to(dev)


class GpuUnit:
    """A unit's GPU-stored entries as fp64 numpy arrays (attribute names the oracle expects)."""

    def __init__(self, kt, vt, alpha, beta, var=None):
        self.kt, self.vt, self.alpha, self.beta, self.var = kt, vt, alpha, beta, var


def gpu_unit(pool, table, lens, b, h):
    kt, vt, al, be = skv.read_entries(pool, table, lens, b, h)
    var = skv.read_variances(pool, table, lens, b, h).double().cpu().numpy() if pool.var is not None else None
    return GpuUnit(kt.double().cpu().numpy(), vt.double().cpu().numpy(), al.double().cpu().numpy(),
                   be.double().cpu().numpy(), var)


def gpu_units(pool, table, lens, B, Hkv):
    return [[gpu_unit(pool, table, lens, b, h) for h in range(Hkv)] for b in range(B)]


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def check_decode(out_gpu, lse_gpu, out_ref, lse_ref, dtype, what=""):
    og = out_gpu.double().cpu().numpy() if isinstance(out_gpu, torch.Tensor) else np.asarray(out_gpu)
    lg = lse_gpu.double().cpu().numpy() if isinstance(lse_gpu, torch.Tensor) else np.asarray(lse_gpu)
    inf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lg), inf_ref), f"{what}: empty-unit pattern differs"
    fin = ~inf_ref
    if dtype == torch.float32:
        assert rel_l2(og, out_ref) <= TOL_F32_REL_L2, f"{what}: out rel-L2 {rel_l2(og, out_ref):.3e}"
        assert rel_l2(lg[fin], lse_ref[fin]) <= TOL_F32_REL_L2, f"{what}: lse rel-L2"
    else:
        r = rel_l2(og, out_ref)
        m = float(np.abs(og - out_ref).max()) if og.size else 0.0
        assert r <= TOL_BF16_REL_L2, f"{what}: out rel-L2 {r:.3e}"
        assert m <= TOL_BF16_MAX_ABS, f"{what}: out max-abs {m:.3e}"
        if fin.any():
            le = float(np.abs(lg[fin] - lse_ref[fin]).max())
            assert le <= TOL_LSE_ABS, f"{what}: lse max-abs {le:.3e}"
    assert np.all(og[inf_ref] == 0), f"{what}: empty units must give zero output"


def bf16_ulp(x):
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(ax, 1e-38)))
    return np.exp2(e - 7)


def weighted_slack(orc_unit, k, v):
    """Absolute fp32 error allowance of the variation-weighted representatives of one unit (zero
    for entries that store a plain mean). The kernel forms sum_r w_r x_r and sum_r w_r in fp32
    (w_r = D_r 2^-20 rounded to fp32) and divides: by the standard summation bound the error is
    at most about (m + 4) 2^-24 sum_r w_r |x_r| / sum_r w_r. k, v: the unit's fp32 tokens [T, d]."""
    E, d = orc_unit.kt.shape
    sk, sv = np.zeros((E, d)), np.zeros((E, d))
    for e in range(E):
        st, m = int(orc_unit.start[e]), int(orc_unit.mass[e])
        mid = st - orc_unit.s_eff
        if m < 2 or mid < 0 or mid >= orc_unit.M:
            continue
        w = orc_unit.D[mid:mid + m].astype(np.float64)
        if w.sum() == 0:
            continue
        c = (m + 4) * 2.0 ** -24 / w.sum()
        sk[e] = c * (w[:, None] * np.abs(k[st:st + m].astype(np.float64))).sum(axis=0)
        sv[e] = c * (w[:, None] * np.abs(v[st:st + m].astype(np.float64))).sum(axis=0)
    return sk, sv


def check_nodes(gpu_unit, orc_unit, dtype, d, what="", slack=None):
    """Node statistics of one unit: GPU (stored) vs oracle fp64. slack: optional (k, v) absolute
    fp32 allowances per entry and dimension (see weighted_slack)."""
    assert gpu_unit.kt.shape == orc_unit.kt.shape, f"{what}: entry count"
    al_err = np.abs(gpu_unit.alpha - orc_unit.alpha)
    assert np.all(al_err <= 1e-6 * np.maximum(1.0, np.abs(orc_unit.alpha))), f"{what}: alpha"
    be_ref = orc_unit.beta
    be_err = np.abs(gpu_unit.beta - be_ref)
    assert np.all(be_err <= 1e-5 * np.abs(be_ref) + 1e-12), f"{what}: beta max rel {np.max(be_err / (be_ref + 1e-30)):.2e}"
    for i, name in enumerate(("kt", "vt")):
        g, o = getattr(gpu_unit, name), getattr(orc_unit, name)
        if dtype == torch.float32:
            assert rel_l2(g, o) <= TOL_F32_REL_L2, f"{what}: {name} rel-L2 {rel_l2(g, o):.2e}"
            if slack is not None:
                assert np.all(np.abs(g - o) <= slack[i] + 2.0 ** -23 * np.abs(o) + 1e-30), f"{what}: {name}"
        else:
            # the fp32 mean rounded once to bf16: within half an ulp of the fp64 mean, plus fp32 error
            err = np.abs(g - o)
            bound = 0.5 * bf16_ulp(o) + 1e-6 * np.abs(o) + 1e-30
            if slack is not None:
                bound = bound + slack[i]
            assert np.all(err <= bound), f"{what}: {name} worst excess {np.max(err / bound):.3f}"
            assert rel_l2(g, o) <= TOL_BF16_REL_L2
    if getattr(gpu_unit, "var", None) is not None:
        # per-dimension variances: an fp32 two-pass variance rounded once to the dtype
        g, o = gpu_unit.var, orc_unit.var
        err = np.abs(g - o)
        if dtype == torch.float32:
            bound = 2e-6 * np.abs(o) + 1e-12
        else:
            bound = 0.5 * bf16_ulp(o) + 2e-6 * np.abs(o) + 1e-12
        assert np.all(err <= bound), f"{what}: var worst excess {np.max(err / bound):.3f}"


def to_np32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()
