"""GPU parity at the workloads' full sizes, in the launch configuration bench.py times.

The whole batch is coarsened / decoded on the GPU; the oracle recomputes a sample of units one
by one (the shortest and longest sequences, first and last KV heads): bit-exact cumulative
variation, boundaries and entry counts, node statistics within tolerance, decode outputs within
the bf16 bar against the oracle fed the GPU's stored nodes.
"""
import numpy as np
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
import oracle
import workloads
from gpu_helpers import check_decode, check_nodes, gpu_units, to_np32, weighted_slack

pytestmark = pytest.mark.gpu

S, W = workloads.N_SINK, workloads.N_RECENT


def _coarsen_full(w, values="normal", representative="mean"):
    T_list = workloads.seq_lengths(w)
    N_list = workloads.segment_counts(w, T_list)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list, values=values)
    pages = [skv.pages_for(T, N, S, W) for T, N in zip(T_list, N_list)]
    table, num_pages = workloads.page_assignment(w.B, w.Hkv, pages, w.shuffle_pages, w.seed)
    table = table.cuda()
    pool = skv.NodePool(num_pages, w.d, w.torch_dtype)
    pool.k.fill_(float("nan"))
    pool.v.fill_(float("nan"))
    pool.ab.fill_(float("nan"))
    bnd = torch.full((w.B, w.Hkv, max(N_list) + 1), -7, dtype=torch.int32, device="cuda")
    cum = torch.full((k.shape[0],), -7, dtype=torch.int64, device="cuda")
    ws = torch.zeros(skv.coarsen_workspace_bytes(w.Hkv, w.d, T_list, N_list, S, W), dtype=torch.uint8,
                     device="cuda")
    lens = skv.coarsen(k, v, w.Hkv, T_list, N_list, S, W, w.seed, pool, table, boundaries=bnd, cumvar=cum,
                       workspace=ws, representative=representative)
    st, flags = skv.workspace_error(ws)
    assert st == 0, flags
    return dict(k=k, v=v, T=T_list, N=N_list, pool=pool, table=table, lens=lens, bnd=bnd, cum=cum)


def _check_units(w, r, units, representative="mean"):
    P = oracle.projection(w.seed, w.d)
    for (b, h) in units:
        kk = to_np32(workloads.unit_rows(r["k"], r["T"], w.Hkv, b, h))
        vv = to_np32(workloads.unit_rows(r["v"], r["T"], w.Hkv, b, h))
        u = oracle.coarsen_unit(kk, vv, S, W, r["N"][b], P, representative)
        what = f"{w.name} unit ({b},{h}) T={r['T'][b]}"
        off = sum(r["T"][:b]) * w.Hkv + h * r["T"][b]
        assert np.array_equal(r["cum"][off:off + u.M].cpu().numpy(), u.C), f"{what}: c_t"
        assert np.array_equal(r["bnd"][b, h, :r["N"][b] + 1].cpu().numpy(), u.bounds), f"{what}: boundaries"
        assert int(r["lens"][b, h]) == u.kt.shape[0], f"{what}: lens"
        kt, vt, al, be = skv.read_entries(r["pool"], r["table"], r["lens"], b, h)

        class G:
            pass

        g = G()
        g.kt, g.vt = kt.double().cpu().numpy(), vt.double().cpu().numpy()
        g.alpha, g.beta = al.double().cpu().numpy(), be.double().cpu().numpy()
        check_nodes(g, u, w.torch_dtype, w.d, what, slack=weighted_slack(u, kk, vv))


def _check_decode(w, r, sample_b):
    q = workloads.make_queries(w, "cuda")
    out, lse = skv.decode_attn(q, w.Hkv, r["pool"], r["table"], r["lens"])
    torch.cuda.synchronize()
    units = []
    for b in sample_b:
        row = []
        for h in range(w.Hkv):
            kt, vt, al, be = skv.read_entries(r["pool"], r["table"], r["lens"], b, h)

            class G:
                pass

            g = G()
            g.kt, g.vt = kt.double().cpu().numpy(), vt.double().cpu().numpy()
            g.alpha, g.beta = al.double().cpu().numpy(), be.double().cpu().numpy()
            row.append(g)
        units.append(row)
    ref_out, ref_lse = oracle.decode(q[sample_b].double().cpu().numpy(), units)
    check_decode(out[sample_b], lse[sample_b], ref_out, ref_lse, w.torch_dtype, f"{w.name} decode")
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_gqa7_32k_3p5pct_full():
    """7B-shaped decode workload: 32 x 4 units of 32,768 tokens coarsened to 1,147 entries each."""
    w = workloads.WORKLOADS["gqa7_32k_decode_3p5pct"]
    r = _coarsen_full(w)
    assert int(r["lens"].min()) <= 1147 and int(r["lens"].max()) == 1147
    _check_units(w, r, [(0, 0), (31, 3)])
    _check_decode(w, r, [0, 17, 31])


def test_gqa7_ragged_paged_2pct_full():
    """Ragged paged workload: 128 sequences, T log-uniform in [4,096, 131,072], N = floor(0.02 T),
    4 query rows per sequence, shuffled page table."""
    w = workloads.WORKLOADS["gqa7_ragged_paged_2pct"]
    r = _coarsen_full(w)
    T = np.array(r["T"])
    short, long_ = int(T.argmin()), int(T.argmax())
    _check_units(w, r, [(short, 0), (long_, 3)])
    _check_decode(w, r, sorted({short, long_, 5}))


def test_coarsen_131k_full():
    """Coarsening-throughput workload: 8 x 4 units of 131,072 tokens, N = 2,621."""
    w = workloads.WORKLOADS["coarsen_131k"]
    r = _coarsen_full(w)
    _check_units(w, r, [(0, 0), (7, 3)])


def test_gqa7_32k_3p5pct_variation_weighted_full():
    """The 7B-shaped workload coarsened with the variation-weighted representative, then decoded."""
    w = workloads.WORKLOADS["gqa7_32k_decode_3p5pct"]
    r = _coarsen_full(w, representative="variation")
    _check_units(w, r, [(3, 1), (30, 2)], representative="variation")
    _check_decode(w, r, [3, 30])


def test_coarsen_131k_tensor_projection_full():
    """The coarsening workload with the tensor-core projection option, stage by stage on sampled
    units: every step within the bound of the exact bf16 projection's step; boundaries, c_t and
    statistics as the oracle computes them from those steps."""
    w = workloads.WORKLOADS["coarsen_131k"]
    T_list = workloads.seq_lengths(w)
    N_list = workloads.segment_counts(w, T_list)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list)
    pages = [skv.pages_for(T, N, S, W) for T, N in zip(T_list, N_list)]
    table, num_pages = workloads.page_assignment(w.B, w.Hkv, pages, False, w.seed)
    table = table.cuda()
    pool = skv.NodePool(num_pages, w.d, w.torch_dtype)
    bnd = torch.full((w.B, w.Hkv, max(N_list) + 1), -7, dtype=torch.int32, device="cuda")
    cum = torch.full((k.shape[0],), -7, dtype=torch.int64, device="cuda")
    ws = torch.zeros(skv.coarsen_workspace_bytes(w.Hkv, w.d, T_list, N_list, S, W), dtype=torch.uint8, device="cuda")
    lens = skv.coarsen(k, v, w.Hkv, T_list, N_list, S, W, w.seed, pool, table, boundaries=bnd, cumvar=cum,
                       workspace=ws, projection="tensor")
    st, flags = skv.workspace_error(ws)
    assert st == 0, flags
    P16 = oracle.projection_bf16(w.seed, w.d)
    for (b, h) in [(0, 0), (3, 2), (7, 3)]:
        kk = to_np32(workloads.unit_rows(k, T_list, w.Hkv, b, h))
        vv = to_np32(workloads.unit_rows(v, T_list, w.Hkv, b, h))
        M = T_list[b] - S - W
        off = sum(T_list[:b]) * w.Hkv + h * T_list[b]
        C = cum[off:off + M].cpu().numpy()
        D = np.diff(C, prepend=0)
        dref, bound = oracle.tensor_steps_reference(kk, vv, S, W, P16)
        assert np.all(np.abs(D - dref) <= bound), f"unit ({b},{h}) steps"
        u = oracle.coarsen_unit_from_steps(kk, vv, S, W, N_list[b], D)
        assert np.array_equal(bnd[b, h, :N_list[b] + 1].cpu().numpy(), u.bounds)
        assert int(lens[b, h]) == u.kt.shape[0]
        kt, vt, al, be = skv.read_entries(pool, table, lens, b, h)

        class G:
            pass

        g = G()
        g.kt, g.vt = kt.double().cpu().numpy(), vt.double().cpu().numpy()
        g.alpha, g.beta = al.double().cpu().numpy(), be.double().cpu().numpy()
        check_nodes(g, u, w.torch_dtype, w.d, f"tensor projection unit ({b},{h})")


def test_coarsen_131k_captured_equals_direct():
    """Half the 131k coarsening workload (16 units of 131,072 tokens) captured into a CUDA graph and
    replayed gives the direct call's boundaries, lens and stored nodes bit for bit."""
    import dataclasses
    w = dataclasses.replace(workloads.WORKLOADS["coarsen_131k"], B=4)
    r = _coarsen_full(w)
    T_list, N_list = r["T"], r["N"]
    pool2 = skv.NodePool(r["pool"].num_pages, w.d, w.torch_dtype)
    lens2 = torch.full_like(r["lens"], -7)
    bnd2 = torch.full_like(r["bnd"], -7)
    ws2 = torch.zeros(skv.coarsen_workspace_bytes(w.Hkv, w.d, T_list, N_list, S, W), dtype=torch.uint8,
                      device="cuda")
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        skv.coarsen(r["k"], r["v"], w.Hkv, T_list, N_list, S, W, w.seed, pool2, r["table"], lens=lens2,
                    boundaries=bnd2, workspace=ws2)
    g.replay()
    torch.cuda.synchronize()
    assert skv.workspace_error(ws2)[0] == 0
    assert torch.equal(lens2, r["lens"]) and torch.equal(bnd2, r["bnd"])
    for b in range(w.B):
        for h in range(w.Hkv):
            one = skv.read_entries(r["pool"], r["table"], r["lens"], b, h)
            two = skv.read_entries(pool2, r["table"], lens2, b, h)
            for x, y in zip(one, two):
                assert torch.equal(x, y), f"unit ({b},{h}) differs"
    del g
