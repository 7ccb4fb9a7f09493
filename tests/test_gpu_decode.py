"""GPU parity of compressed decode attention ("SPICY-KV" section 2 logit with online softmax)
against the fp64 oracle, on synthetic entry sets written straight into the pool: GQA groups of
1..8 heads, 1..5 query rows per sequence (row passes above 32 rows), d = 64 / 128, ragged and
empty units, partial last pages, shuffled page tables and split units."""
import math

import numpy as np
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
import oracle
from gpu_helpers import check_decode, gpu_units, pool_for_units, write_entries

pytestmark = pytest.mark.gpu


def _synthetic(B, Hq, Hkv, R, d, lens_list, dtype, seed, key_scale=3.0, shuffle=True, spare=0, closure="scalar"):
    g = torch.Generator(device="cpu").manual_seed(seed)
    pool, table = pool_for_units(lens_list, B, Hkv, d, dtype, shuffle=shuffle, seed=seed, spare_pages=spare,
                                 closure=closure)
    for b in range(B):
        for h in range(Hkv):
            E = int(lens_list[b])
            kt = torch.randn(E, d, generator=g) * key_scale
            vt = torch.randn(E, d, generator=g)
            mass = torch.randint(1, 200, (E,), generator=g).double()
            alpha = torch.log(mass)
            beta = torch.rand(E, generator=g) * 0.02
            # per-dimension variances spread over two decades (diagonal pools only)
            var = torch.rand(E, d, generator=g).pow(3) * 2.0 if closure == "diagonal" else None
            write_entries(pool, table, b, h, kt, vt, alpha, beta, var)
    lens = torch.tensor([[int(lens_list[b])] * Hkv for b in range(B)], dtype=torch.int32, device="cuda")
    q = (torch.randn(B, R, Hq, d, generator=g)).to(dtype).cuda()
    return pool, table, lens, q


def _run(B, Hq, Hkv, R, d, lens_list, dtype, seed, closure="scalar", **kw):
    pool, table, lens, q = _synthetic(B, Hq, Hkv, R, d, lens_list, dtype, seed, closure=closure, **kw)
    out, lse = skv.decode_attn(q, Hkv, pool, table, lens)
    torch.cuda.synchronize()
    units = gpu_units(pool, table, lens, B, Hkv)
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), units, closure=closure)
    check_decode(out, lse, ref_out, ref_lse, dtype, what=f"B{B} Hq{Hq} Hkv{Hkv} R{R} d{d}")
    return out, lse


@pytest.mark.parametrize("Hq,Hkv,R", [(28, 4, 1), (12, 2, 1), (4, 4, 1), (16, 8, 1), (28, 4, 4), (16, 2, 5),
                                      (14, 2, 2), (8, 1, 3)])
def test_decode_bf16_gqa_shapes(Hq, Hkv, R):
    B = 3
    lens = [1147, 37, 300]
    _run(B, Hq, Hkv, R, 128, lens, torch.bfloat16, seed=Hq * 10 + R)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_bf16_ragged_and_empty(d):
    lens = [0, 1, 15, 16, 17, 31, 33, 250, 0, 2677]
    _run(len(lens), 14, 2, 1, d, lens, torch.bfloat16, seed=d)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_f32_path(d):
    lens = [88, 1, 0, 200]
    _run(len(lens), 2, 1, 1, d, lens, torch.float32, seed=5 + d, key_scale=1.0)


def test_decode_single_unit_many_ctas():
    """One long unit split across every CTA (partials merged by the combine kernel)."""
    _run(1, 7, 1, 1, 128, [20000], torch.bfloat16, seed=11)


def test_decode_peaked_softmax():
    """Large key scale: one entry dominates (online max updates across pages and CTAs)."""
    _run(4, 28, 4, 1, 128, [500, 1500, 64, 3000], torch.bfloat16, seed=12, key_scale=12.0)


def test_decode_is_deterministic():
    a, la = _run(2, 28, 4, 1, 128, [900, 2000], torch.bfloat16, seed=13)
    b, lb = _run(2, 28, 4, 1, 128, [900, 2000], torch.bfloat16, seed=13)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_decode_bad_page_id_is_flagged_not_read():
    """A page id outside the pool raises the device flag and is skipped (no out-of-bounds read)."""
    B, Hq, Hkv, d = 2, 7, 1, 128
    pool, table, lens, q = _synthetic(B, Hq, Hkv, 1, d, [64, 64], torch.bfloat16, seed=3)
    table[1, 0, 2] = pool.num_pages + 5
    ws = torch.zeros(skv.decode_workspace_bytes(B, 1, Hq, Hkv, d, table.shape[2]), dtype=torch.uint8,
                     device="cuda")
    out, lse = skv.decode_attn(q, Hkv, pool, table, lens, workspace=ws)
    st, flags = skv.workspace_error(ws)
    assert st == skv._lib.SKV_ERR_DEVICE and flags & skv._lib.FLAG_BAD_PAGE
    # unit 0 is untouched by the bad page
    units = gpu_units(pool, table, lens, 1, Hkv)
    ref_out, ref_lse = oracle.decode(q[:1].double().cpu().numpy(), units)
    check_decode(out[:1], lse[:1], ref_out, ref_lse, torch.bfloat16)
    st, flags = skv.workspace_error(ws)
    assert st == 0 and flags == 0          # read-and-clear


def test_decode_lens_above_capacity_is_clamped_and_flagged():
    B, Hq, Hkv, d = 1, 7, 1, 128
    pool, table, lens, q = _synthetic(B, Hq, Hkv, 1, d, [40], torch.bfloat16, seed=4, shuffle=False)
    ws = torch.zeros(skv.decode_workspace_bytes(B, 1, Hq, Hkv, d, table.shape[2]), dtype=torch.uint8,
                     device="cuda")
    lens_bad = lens.clone()
    lens_bad[0, 0] = table.shape[2] * 16 + 100
    skv.decode_attn(q, Hkv, pool, table, lens_bad, workspace=ws)
    st, flags = skv.workspace_error(ws)
    assert flags & skv._lib.FLAG_BAD_LENS


def test_decode_repeated_calls_at_bench_shape_are_identical():
    """The 7B-shaped 3.5% workload's launch configuration (32 x 4 units of 1,147 entries, split
    across every CTA): 24 back-to-back calls alternating two caches give bit-identical outputs,
    and sampled units match the oracle. Catches pipeline races that depend on timing."""
    B, Hq, Hkv, d = 32, 28, 4, 128
    lens = [1147] * B
    caches = [_synthetic(B, Hq, Hkv, 1, d, lens, torch.bfloat16, seed=100 + i, shuffle=False) for i in range(2)]
    ws = torch.zeros(skv.decode_workspace_bytes(B, 1, Hq, Hkv, d, caches[0][1].shape[2]), dtype=torch.uint8,
                     device="cuda")
    firsts = [None, None]
    outs = [(torch.empty_like(c[3]), torch.empty(B, 1, Hq, dtype=torch.float32, device="cuda")) for c in caches]
    for it in range(24):
        pool, table, ln, q = caches[it % 2]
        out, lse = outs[it % 2]
        skv.decode_attn(q, Hkv, pool, table, ln, out=out, lse=lse, workspace=ws)
        if firsts[it % 2] is None:
            torch.cuda.synchronize()
            firsts[it % 2] = (out.clone(), lse.clone())
        elif it >= 22:
            torch.cuda.synchronize()
            assert torch.equal(out, firsts[it % 2][0]) and torch.equal(lse, firsts[it % 2][1])
    st, flags = skv.workspace_error(ws)
    assert st == 0, flags
    pool, table, ln, q = caches[0]
    sample = [0, 13, 31]
    units = gpu_units(pool, table, ln, B, Hkv)
    ref_out, ref_lse = oracle.decode(q[sample].double().cpu().numpy(), [units[b] for b in sample])
    check_decode(firsts[0][0][sample], firsts[0][1][sample], ref_out, ref_lse, torch.bfloat16, "bench shape")


def _widen_table(table, extra, fill):
    """The same page table with `extra` more columns holding `fill` (ids past every unit's pages)."""
    B, Hkv, P = table.shape
    wide = torch.full((B, Hkv, P + extra), fill, dtype=table.dtype, device=table.device)
    wide[:, :, :P] = table
    return wide


def test_decode_uniform_lens_table_wider_than_units():
    """Equal-length units in a page table wider than they need, its spare columns holding ids
    outside the pool: pages read ahead for a full-width table are discarded, no flag is raised,
    and the outputs match the oracle."""
    B, Hq, Hkv, d = 16, 28, 4, 128
    pool, table, lens, q = _synthetic(B, Hq, Hkv, 1, d, [700] * B, torch.bfloat16, seed=21)
    wide = _widen_table(table, 13, pool.num_pages + 1000)
    ws = torch.zeros(skv.decode_workspace_bytes(B, 1, Hq, Hkv, d, wide.shape[2]), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        out, lse = skv.decode_attn(q, Hkv, pool, wide, lens, workspace=ws)
        st, flags = skv.workspace_error(ws)
        assert st == 0 and flags == 0, flags
    units = gpu_units(pool, table, lens, B, Hkv)
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), units)
    check_decode(out, lse, ref_out, ref_lse, torch.bfloat16, "wide table")


def test_decode_ragged_lens_few_units():
    """Few units of different lengths (the launch a uniform batch of this size would use, with the
    read-ahead discarded and the flat split taking over)."""
    lens = [700, 1147, 33, 512, 900, 1, 0, 640, 16, 17, 300, 1147, 64, 65, 999, 250]
    _run(len(lens), 28, 4, 1, 128, lens, torch.bfloat16, seed=22)


def test_decode_bad_page_in_first_pages_is_flagged():
    """A bad page id among the first pages of a full-width, equal-length batch (read before the
    lens are known) raises the flag once the lens confirm the split; other units are exact."""
    B, Hq, Hkv, d = 16, 28, 4, 128
    pool, table, lens, q = _synthetic(B, Hq, Hkv, 1, d, [700] * B, torch.bfloat16, seed=23)
    bad = table.clone()
    bad[5, 1, 0] = pool.num_pages + 9
    ws = torch.zeros(skv.decode_workspace_bytes(B, 1, Hq, Hkv, d, table.shape[2]), dtype=torch.uint8,
                     device="cuda")
    out, lse = skv.decode_attn(q, Hkv, pool, bad, lens, workspace=ws)
    st, flags = skv.workspace_error(ws)
    assert st == skv._lib.SKV_ERR_DEVICE and flags & skv._lib.FLAG_BAD_PAGE
    keep = [b for b in range(B) if b != 5]
    units = gpu_units(pool, table, lens, B, Hkv)
    ref_out, ref_lse = oracle.decode(q[keep].double().cpu().numpy(), [units[b] for b in keep])
    check_decode(out[keep], lse[keep], ref_out, ref_lse, torch.bfloat16, "bad first page")
    out2, lse2 = skv.decode_attn(q, Hkv, pool, table, lens, workspace=ws)
    st, flags = skv.workspace_error(ws)
    assert st == 0 and flags == 0
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), units)
    check_decode(out2, lse2, ref_out, ref_lse, torch.bfloat16, "after bad page")


@pytest.mark.parametrize("B,Hq,Hkv,R,d,E", [
    (24, 28, 4, 1, 128, 700),   # 96 virtual units: clusters of 3 CTAs
    (16, 28, 4, 1, 64, 1147),   # 64 units, d = 64: clusters of 4
    (16, 16, 2, 2, 128, 500),   # 16 query rows per unit (two row tiles)
    (8, 32, 4, 4, 64, 900),     # 32 query rows per unit (four row tiles), d = 64
    (8, 16, 4, 5, 128, 333),    # 20 query rows
    (4, 32, 4, 5, 128, 640),    # 40 query rows: two row passes per unit
    (64, 28, 4, 1, 128, 300),   # 256 units: one CTA owns each whole unit (no merge)
])
def test_decode_equal_lengths_cluster_split(B, Hq, Hkv, R, d, E):
    """Equal-length units in a full-width page table (the read-ahead and cluster-merge path when a
    cluster size fits), across GQA group sizes, query-row counts and head dims."""
    _run(B, Hq, Hkv, R, d, [E] * B, torch.bfloat16, seed=B * 100 + R * 10 + d // 64, shuffle=True)


@pytest.mark.parametrize("B,Hq,Hkv,R,d,lens", [
    (1, 12, 2, 1, 128, [421]),              # the 1.5B 10.5K shape: 2 units x 27 pages, clusters of 8
    (3, 12, 2, 1, 128, [421, 37, 0]),       # unequal and empty units: stream-K over the small grid
    (2, 28, 4, 4, 64, [100, 100]),          # 28 query rows, d = 64, 7 pages per unit: clusters of 7
    (1, 7, 1, 1, 128, [17]),                # two pages: a cluster of 2
])
def test_decode_few_pages(B, Hq, Hkv, R, d, lens):
    """Fewer pages in all units than the grid has CTAs: one cluster of up to 8 CTAs per unit and a
    grid of exactly those clusters (equal lengths), or the stream-K split over that grid."""
    _run(B, Hq, Hkv, R, d, lens, torch.bfloat16, seed=sum(lens) + Hq + d, shuffle=True)


def test_decode_equal_lengths_wide_table_two_row_passes():
    """Equal lengths, 40 query rows (two row passes), page table wider than the units."""
    B, Hq, Hkv, R, d = 4, 32, 4, 5, 128
    pool, table, lens, q = _synthetic(B, Hq, Hkv, R, d, [640] * B, torch.bfloat16, seed=31)
    wide = _widen_table(table, 7, -1)
    ws = torch.zeros(skv.decode_workspace_bytes(B, R, Hq, Hkv, d, wide.shape[2]), dtype=torch.uint8, device="cuda")
    out, lse = skv.decode_attn(q, Hkv, pool, wide, lens, workspace=ws)
    st, flags = skv.workspace_error(ws)
    assert st == 0 and flags == 0, flags
    units = gpu_units(pool, table, lens, B, Hkv)
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), units)
    check_decode(out, lse, ref_out, ref_lse, torch.bfloat16, "wide table, two row passes")


@pytest.mark.parametrize("B,Hq,Hkv,R,d,lens,dtype", [
    (32, 28, 4, 1, 128, [1147] * 32, torch.bfloat16),        # the 7B 3.5% shape
    (3, 28, 4, 1, 128, [1147, 37, 300], torch.bfloat16),
    (10, 14, 2, 1, 64, [0, 1, 15, 16, 17, 31, 33, 250, 0, 2677], torch.bfloat16),
    (4, 32, 4, 4, 128, [640, 17, 900, 64], torch.bfloat16),  # 32 query rows per unit
    (4, 32, 4, 5, 64, [333] * 4, torch.bfloat16),            # two row passes
    (4, 2, 1, 1, 128, [88, 1, 0, 200], torch.float32),
    (2, 4, 2, 1, 64, [300, 45], torch.float32),
])
def test_decode_diagonal_closure(B, Hq, Hkv, R, d, lens, dtype):
    """Diagonal-closure pools: logit q.k/sqrt(d) + alpha + sum_i q_i^2 var_i/(2d) against the oracle
    fed the GPU's stored nodes and variances."""
    kw = {"key_scale": 1.0} if dtype == torch.float32 else {}
    _run(B, Hq, Hkv, R, d, lens, dtype, seed=B * 7 + d + R, closure="diagonal", **kw)
