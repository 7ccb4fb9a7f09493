"""GPU parity of equal-variation coarsening against the oracle.

Bit-exact: the projection P, every unit's cumulative quantised variation c_t, the segment
boundaries, the entry counts. Within tolerance: node statistics (mean key / value, alpha = ln m,
beta = sigma^2 / (2d)). Sizes span several projection tiles (511 middle tokens each) with ragged tails,
plus the degenerate cases: T <= n_sink + n_recent, empty middle, M < N (empty segments dropped),
constant middle (c_T = 0), N = 1, one jump crossing many thresholds, d = 64 / 128, fp32 / bf16;
every case also with the variation-weighted segment representative."""
import numpy as np
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
import oracle
import workloads
from gpu_helpers import check_decode, check_nodes, gpu_unit, gpu_units, pool_for_units, to_np32, weighted_slack

pytestmark = pytest.mark.gpu

S, W = workloads.N_SINK, workloads.N_RECENT


def run_coarsen(k, v, Hkv, T_list, N_list, seed, n_sink=S, n_recent=W, shuffle=True, representative="mean",
                closure="scalar", center_keys=False, projection="fixed"):
    B = len(T_list)
    d = k.shape[-1]
    ent = [skv.entries_bound(T, N, n_sink, n_recent) for T, N in zip(T_list, N_list)]
    pool, table = pool_for_units(ent, B, Hkv, d, k.dtype, shuffle=shuffle, seed=seed, closure=closure)
    Nmax = max(N_list)
    bnd = torch.full((B, Hkv, Nmax + 1), -7, dtype=torch.int32, device="cuda")
    cum = torch.full((k.shape[0],), -7, dtype=torch.int64, device="cuda")
    ws = torch.zeros(skv.coarsen_workspace_bytes(Hkv, d, T_list, N_list, n_sink, n_recent), dtype=torch.uint8,
                     device="cuda")
    lens = skv.coarsen(k, v, Hkv, T_list, N_list, n_sink, n_recent, seed, pool, table, boundaries=bnd, cumvar=cum,
                       workspace=ws, representative=representative, center_keys=center_keys,
                       projection=projection)
    st, flags = skv.workspace_error(ws)
    return dict(pool=pool, table=table, lens=lens, bnd=bnd, cum=cum, status=st, flags=flags)


def oracle_units(k, v, Hkv, T_list, N_list, seed, units=None, n_sink=S, n_recent=W, representative="mean",
                 center=False):
    d = k.shape[-1]
    P = oracle.projection(seed, d)
    res = {}
    for b, T in enumerate(T_list):
        for h in range(Hkv):
            if units is not None and (b, h) not in units:
                continue
            kk = to_np32(workloads.unit_rows(k, T_list, Hkv, b, h))
            vv = to_np32(workloads.unit_rows(v, T_list, Hkv, b, h))
            res[(b, h)] = oracle.coarsen_unit(kk, vv, n_sink, n_recent, int(N_list[b]), P, representative, center)
    return res


def compare_units(r, orc, k, v, T_list, Hkv, N_list, dtype, center=False):
    d = k.shape[-1]
    for (b, h), u in orc.items():
        what = f"unit ({b},{h}) T={T_list[b]} N={N_list[b]}"
        # cumulative variation, bit for bit
        off = sum(T_list[:b]) * Hkv + h * T_list[b]
        cg = r["cum"][off:off + u.M].cpu().numpy()
        assert np.array_equal(cg, u.C), f"{what}: c_t differs at {np.flatnonzero(cg != u.C)[:5]}"
        # boundaries and entry counts, bit for bit
        bg = r["bnd"][b, h, :N_list[b] + 1].cpu().numpy()
        assert np.array_equal(bg, u.bounds), f"{what}: boundaries differ"
        assert int(r["lens"][b, h]) == u.kt.shape[0], f"{what}: lens"
        gu = gpu_unit(r["pool"], r["table"], r["lens"], b, h)
        kk = to_np32(workloads.unit_rows(k, T_list, Hkv, b, h))
        if center:
            kk = oracle.center_keys(kk)
        vv = to_np32(workloads.unit_rows(v, T_list, Hkv, b, h))
        check_nodes(gu, u, dtype, d, what, slack=weighted_slack(u, kk, vv))


def test_projection_matches_oracle_bitwise():
    for seed in (0, 1, 2, 3, 4, 12345678901234):
        for d in (64, 128):
            a = skv.projection_matrix(seed, d).numpy()
            b = oracle.projection(seed, d)
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


CASES = [
    # name, dtype, d, Hkv, T_list, N_list, values
    ("bf16_d128_multi_tile", torch.bfloat16, 128, 2, [1000, 777], [37, 20], "normal"),
    ("bf16_d64", torch.bfloat16, 64, 3, [600, 256, 1301], [11, 5, 40], "normal"),
    ("f32_d64", torch.float32, 64, 1, [1024, 511], [32, 9], "normal"),
    ("f32_d128", torch.float32, 128, 2, [700], [21], "walk"),
    ("key_only_variation", torch.bfloat16, 128, 2, [2000, 900], [50, 30], "zero"),
    ("short_sequences", torch.bfloat16, 128, 2, [0, 1, 8, 55, 56, 57, 60, 63], [4, 4, 4, 4, 4, 4, 4, 4], "normal"),
    # no unit of the batch has a middle token (no projection tile anywhere)
    ("no_middle_anywhere", torch.bfloat16, 128, 2, [0, 8, 56], [4, 4, 4], "normal"),
    ("more_segments_than_tokens", torch.bfloat16, 128, 1, [70, 200], [40, 500], "normal"),
    ("single_segment", torch.bfloat16, 128, 2, [3000], [1], "normal"),
    ("tile_edges", torch.bfloat16, 128, 1, [56 + 255, 56 + 510, 56 + 511, 56 + 512, 56 + 1022, 56 + 1023],
     [7, 7, 7, 7, 7, 7], "normal"),
    # 21 units of ragged lengths: one sequence empty, one without a middle, one with N = 1
    ("many_units_ragged", torch.bfloat16, 128, 3, [900, 40, 1500, 0, 700, 2100, 333], [30, 4, 60, 4, 1, 80, 9],
     "normal"),
]


@pytest.mark.parametrize("representative", ["mean", "variation"])
@pytest.mark.parametrize("name,dtype,d,Hkv,T_list,N_list,values", CASES, ids=[c[0] for c in CASES])
def test_coarsen_matches_oracle(name, dtype, d, Hkv, T_list, N_list, values, representative):
    seed = sum(T_list) + d
    w = workloads.Workload(name, seed, B=len(T_list), Hq=Hkv, Hkv=Hkv, d=d, R=1,
                           dtype="bf16" if dtype == torch.bfloat16 else "f32", T=0, regimes=12)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list, values=values)
    r = run_coarsen(k, v, Hkv, T_list, N_list, seed, representative=representative)
    assert r["status"] == 0, f"device flags {r['flags']}"
    orc = oracle_units(k, v, Hkv, T_list, N_list, seed, representative=representative)
    compare_units(r, orc, k, v, T_list, Hkv, N_list, dtype)


DIAG_CASES = [c for c in CASES if c[0] in ("bf16_d128_multi_tile", "bf16_d64", "f32_d64", "short_sequences",
                                           "tile_edges", "single_segment")]


@pytest.mark.parametrize("name,dtype,d,Hkv,T_list,N_list,values", DIAG_CASES, ids=[c[0] for c in DIAG_CASES])
def test_coarsen_diagonal_closure_matches_oracle(name, dtype, d, Hkv, T_list, N_list, values):
    """A pool for the diagonal closure: the same boundaries and statistics plus every node's
    per-dimension key variances (zero for exact tokens)."""
    seed = sum(T_list) + d + 1
    w = workloads.Workload(name, seed, B=len(T_list), Hq=Hkv, Hkv=Hkv, d=d, R=1,
                           dtype="bf16" if dtype == torch.bfloat16 else "f32", T=0, regimes=12)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list, values=values)
    r = run_coarsen(k, v, Hkv, T_list, N_list, seed, closure="diagonal")
    assert r["status"] == 0, f"device flags {r['flags']}"
    orc = oracle_units(k, v, Hkv, T_list, N_list, seed)
    compare_units(r, orc, k, v, T_list, Hkv, N_list, dtype)


def test_tiny_f32_diagonal_closure_end_to_end():
    """tiny_f32 coarsened into a diagonal pool and decoded with the diagonal closure, against the
    oracle's own nodes (fp32 bar)."""
    w = workloads.WORKLOADS["tiny_f32"]
    k, v, T_list = workloads.make_kv(w, "cuda")
    N_list = workloads.segment_counts(w, T_list)
    r = run_coarsen(k, v, w.Hkv, T_list, N_list, w.seed, closure="diagonal")
    assert r["status"] == 0
    orc = oracle_units(k, v, w.Hkv, T_list, N_list, w.seed)
    compare_units(r, orc, k, v, T_list, w.Hkv, N_list, torch.float32)
    q = workloads.make_queries(w, "cuda")
    out, lse = skv.decode_attn(q, w.Hkv, r["pool"], r["table"], r["lens"])
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), [[orc[(0, 0)]]], closure="diagonal")
    check_decode(out, lse, ref_out, ref_lse, torch.float32, "tiny_f32 diagonal end to end")
    scal_out, _ = oracle.decode(q.double().cpu().numpy(), [[orc[(0, 0)]]])
    assert np.abs(ref_out - scal_out).max() > 1e-5      # the two closures differ on this cache


def test_weighted_representative_on_flat_and_jump_segments():
    """Piecewise-constant keys and values with jumps: a segment's steps sit on its jump tokens, so
    the weighted key differs from the plain mean, and segments inside a flat run (no steps) keep
    the plain mean; both against the oracle."""
    T, d = 1500, 128
    g = torch.Generator(device="cuda").manual_seed(5)
    levels = torch.randn(12, 2, d, device="cuda", generator=g)
    idx = torch.div(torch.arange(T, device="cuda") * 12, T, rounding_mode="floor")
    k = (levels[idx, 0] + 0.02 * torch.randn(T, d, device="cuda", generator=g)).bfloat16()
    v = levels[idx, 1].bfloat16()
    k[600:900] = k[600]
    r = run_coarsen(k, v, 1, [T], [40], seed=7, representative="variation")
    assert r["status"] == 0
    orc = oracle_units(k, v, 1, [T], [40], seed=7, representative="variation")
    plain = oracle_units(k, v, 1, [T], [40], seed=7)
    assert np.abs(orc[(0, 0)].kt - plain[(0, 0)].kt).max() > 1e-2
    compare_units(r, orc, k, v, [T], 1, [40], torch.bfloat16)


def test_constant_middle_gives_one_node():
    """c_T = 0: every threshold is hit at the first middle token; one node holds the middle."""
    T, d, Hkv = 700, 128, 1
    k = torch.ones(T, d, dtype=torch.bfloat16, device="cuda") * 0.5
    v = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    k[:S] = torch.randn(S, d, device="cuda").bfloat16()
    r = run_coarsen(k, v, Hkv, [T], [16], seed=1)
    assert int(r["lens"][0, 0]) == S + 1 + W
    orc = oracle_units(k, v, Hkv, [T], [16], seed=1)
    compare_units(r, orc, k, v, [T], Hkv, [16], torch.bfloat16)


def test_jump_crosses_many_thresholds():
    """One huge step takes several thresholds at once: their segments are empty and dropped."""
    T, d = 400, 128
    g = torch.Generator(device="cuda").manual_seed(3)
    k = (torch.randn(T, d, device="cuda", generator=g) * 0.01).bfloat16()
    v = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    k[200:] += 50.0
    r = run_coarsen(k, v, 1, [T], [30], seed=2)
    orc = oracle_units(k, v, 1, [T], [30], seed=2)
    assert orc[(0, 0)].kt.shape[0] < S + 30 + W
    compare_units(r, orc, k, v, [T], 1, [30], torch.bfloat16)


@pytest.mark.parametrize("projection", ["fixed", "tensor"])
def test_thresholds_hit_exactly(projection):
    """Keys alternating between two rows make every middle step the same D (fl(x - y) = -fl(y - x)),
    so c_t = t D. With M - 1 = N k the ratio N c_t / c_T = t / k is an integer at every threshold:
    the double estimate of each floor lies within its guard band of an integer and the exact
    128-bit path decides. Closed form: b_j = j k, and (fixed recipe) bit-exact with the oracle."""
    N, kstep, d = 16, 40, 128
    M = N * kstep + 1                      # two projection tiles
    T = S + M + W
    g = torch.Generator(device="cuda").manual_seed(11)
    k = (torch.randn(T, d, device="cuda", generator=g) * 0.3).bfloat16()
    v = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    a, b = k[S].clone(), (k[S] * -0.5 + 0.125).bfloat16()
    k[S:S + M:2] = a
    k[S + 1:S + M:2] = b
    r = run_coarsen(k, v, 1, [T], [N], seed=5, projection=projection)
    assert r["status"] == 0, r["flags"]
    C = r["cum"][:M].cpu().numpy()        # c_t of the middle tokens t = 0 .. M - 1
    D = int(C[1])
    assert D > 0 and np.array_equal(C, np.arange(M, dtype=np.int64) * D), "steps are not all equal"
    bnd = r["bnd"][0, 0, :N + 1].cpu().numpy()
    assert np.array_equal(bnd, np.append(np.arange(N) * kstep, M)), bnd
    if projection == "fixed":
        orc = oracle_units(k, v, 1, [T], [N], seed=5)
        compare_units(r, orc, k, v, [T], 1, [N], torch.bfloat16)


@pytest.mark.parametrize("projection", ["fixed", "tensor"])
def test_long_unit_over_512_tiles(projection):
    """One unit of 600 full projection tiles plus a ragged tail (306,677 middle tokens): the
    boundary kernel sums more than 512 tile totals per unit (two rounds of its CTA) for c_T and
    each tile's start. Fixed recipe: c_t, boundaries and statistics against the oracle. Both
    projections: the boundaries are the first hits of N c_t >= j c_T on the GPU's own c_t, in
    exact integers."""
    d, N = 64, 64
    M = 600 * 511 + 77
    T = S + M + W
    g = torch.Generator(device="cuda").manual_seed(21)
    k = (torch.randn(T, d, device="cuda", generator=g) * 0.05).cumsum(0).bfloat16()
    v = (torch.randn(T, d, device="cuda", generator=g) * 0.5).bfloat16()
    r = run_coarsen(k, v, 1, [T], [N], seed=3, projection=projection)
    assert r["status"] == 0, r["flags"]
    C = r["cum"][:M].cpu().numpy()
    CT = int(C[-1])
    assert CT > 0 and np.all(np.diff(C) >= 0)
    # N c_t >= j c_T  <=>  c_t >= ceil(j c_T / N) for integer c_t: the first such t by bisection
    thr = np.array([-(-j * CT // N) for j in range(1, N)], dtype=np.int64)
    want = np.concatenate([[0], np.searchsorted(C, thr, side="left"), [M]])
    assert np.array_equal(r["bnd"][0, 0, :N + 1].cpu().numpy(), want)
    if projection == "fixed":
        orc = oracle_units(k, v, 1, [T], [N], seed=3)
        compare_units(r, orc, k, v, [T], 1, [N], torch.bfloat16)


def test_more_than_4096_segments():
    """N = 6,000 over 20,000 middle tokens: the entry planner runs two rounds of 4,096 segments
    (the entry offset carried between them) and drops the empty segments of both (two jumps, each
    crossing several thresholds at once); entries and statistics against the oracle."""
    rows = _jump_walk()
    T, d, N = rows.shape[0], rows.shape[1], 6000
    k = rows.bfloat16().cuda()
    v = (torch.randn(T, d, generator=torch.Generator().manual_seed(32)) * 0.5).bfloat16().cuda()
    r = run_coarsen(k, v, 1, [T], [N], seed=4)
    assert r["status"] == 0, r["flags"]
    orc = oracle_units(k, v, 1, [T], [N], seed=4)
    empty = np.diff(orc[(0, 0)].bounds) == 0
    assert empty[:4096].any() and empty[4096:].any()   # empty segments in both rounds
    compare_units(r, orc, k, v, [T], 1, [N], torch.bfloat16)


def _jump_walk(M=20000, d=64):
    """A random walk over S + M + W rows (CPU generator) with +30 jumps at middle tokens 3,000 and
    17,000."""
    g = torch.Generator().manual_seed(31)
    k = (torch.randn(S + M + W, d, generator=g) * 0.05).cumsum(0)
    k[S + 3000:] += 30.0
    k[S + 17000:] += 30.0
    return k


def test_overflow_is_flagged():
    T, d = 300, 128
    k = torch.zeros(T, d, dtype=torch.float32, device="cuda")
    v = torch.zeros(T, d, dtype=torch.float32, device="cuda")
    k[150:] = 1e30
    r = run_coarsen(k, v, 1, [T], [8], seed=2)
    assert r["status"] == skv._lib.SKV_ERR_OVERFLOW and r["flags"] & skv._lib.FLAG_OVERFLOW


def test_tiny_f32_end_to_end():
    """The tiny fp32 workload: 1 KV head, 2 query heads, d=64, T=1024, N=32; nodes and decode
    against the oracle's own nodes (fp32 bar: relative L2 <= 1e-5)."""
    w = workloads.WORKLOADS["tiny_f32"]
    k, v, T_list = workloads.make_kv(w, "cuda")
    N_list = workloads.segment_counts(w, T_list)
    r = run_coarsen(k, v, w.Hkv, T_list, N_list, w.seed)
    assert r["status"] == 0
    orc = oracle_units(k, v, w.Hkv, T_list, N_list, w.seed)
    compare_units(r, orc, k, v, T_list, w.Hkv, N_list, torch.float32)
    q = workloads.make_queries(w, "cuda")
    out, lse = skv.decode_attn(q, w.Hkv, r["pool"], r["table"], r["lens"])
    units = [[orc[(0, 0)]]]
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), units)
    check_decode(out, lse, ref_out, ref_lse, torch.float32, "tiny_f32 end to end")


def test_gqa6_10k5_prefill_then_decode():
    """1.5B-shaped: 12/2 heads, d=128, T=10,500, N=365: bit-exact segmentation of both heads,
    node statistics, then decode over the GPU nodes."""
    w = workloads.WORKLOADS["gqa6_10k5_prefill_decode"]
    k, v, T_list = workloads.make_kv(w, "cuda")
    N_list = workloads.segment_counts(w, T_list)
    r = run_coarsen(k, v, w.Hkv, T_list, N_list, w.seed)
    assert r["status"] == 0
    orc = oracle_units(k, v, w.Hkv, T_list, N_list, w.seed)
    compare_units(r, orc, k, v, T_list, w.Hkv, N_list, torch.bfloat16)
    q = workloads.make_queries(w, "cuda")
    out, lse = skv.decode_attn(q, w.Hkv, r["pool"], r["table"], r["lens"])
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), gpu_units(r["pool"], r["table"], r["lens"], 1, 2))
    check_decode(out, lse, ref_out, ref_lse, torch.bfloat16, "gqa6 decode")


def test_captured_coarsen_matches_direct_call_bitwise():
    """A coarsening call captured into a CUDA graph and replayed gives, bit for bit, the c_t,
    boundaries, lens and stored nodes of a direct call (the launches carry every host-side plan
    value with them), for both segment representatives."""
    T_list, N_list, Hkv, d, seed = [900, 40, 1500, 0, 700, 2100, 333, 1200], [30, 4, 60, 4, 1, 80, 9, 44], 3, 128, 31
    w = workloads.Workload("captured", seed, B=len(T_list), Hq=Hkv, Hkv=Hkv, d=d, R=1, dtype="bf16", T=0, regimes=12)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list)
    for representative in ("mean", "variation"):
        r = run_coarsen(k, v, Hkv, T_list, N_list, seed, representative=representative)
        assert r["status"] == 0, r["flags"]
        pool2 = skv.NodePool(r["pool"].num_pages, d, torch.bfloat16)
        lens2 = torch.full_like(r["lens"], -7)
        bnd2 = torch.full_like(r["bnd"], -7)
        cum2 = torch.full_like(r["cum"], -7)
        ws2 = torch.zeros(skv.coarsen_workspace_bytes(Hkv, d, T_list, N_list, S, W), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            skv.coarsen(k, v, Hkv, T_list, N_list, S, W, seed, pool2, r["table"], lens=lens2, boundaries=bnd2,
                        cumvar=cum2, workspace=ws2, representative=representative)
        g.replay()
        torch.cuda.synchronize()
        assert skv.workspace_error(ws2)[0] == 0
        assert torch.equal(lens2, r["lens"]) and torch.equal(bnd2, r["bnd"])
        for b, T in enumerate(T_list):
            for h in range(Hkv):
                off = sum(T_list[:b]) * Hkv + h * T
                M = max(0, T - S - W)
                assert torch.equal(cum2[off:off + M], r["cum"][off:off + M])
                one = skv.read_entries(r["pool"], r["table"], r["lens"], b, h)
                two = skv.read_entries(pool2, r["table"], lens2, b, h)
                for x, y in zip(one, two):
                    assert torch.equal(x, y), f"{representative}: unit ({b},{h}) differs"
        del g


def test_coarsen_is_deterministic():
    w = workloads.Workload("det", 9, B=2, Hq=4, Hkv=2, d=128, R=1, dtype="bf16", T=0, regimes=20)
    k, v, T_list = workloads.make_kv(w, "cuda", T_list=[3000, 1700])
    a = run_coarsen(k, v, 2, T_list, [90, 40], seed=9, shuffle=False)
    b = run_coarsen(k, v, 2, T_list, [90, 40], seed=9, shuffle=False)
    assert torch.equal(a["cum"], b["cum"]) and torch.equal(a["bnd"], b["bnd"])
    # bit patterns (unused slots hold NaN in both pools)
    assert torch.equal(a["pool"].k.view(torch.int16), b["pool"].k.view(torch.int16))
    assert torch.equal(a["pool"].v.view(torch.int16), b["pool"].v.view(torch.int16))
    assert torch.equal(a["pool"].ab.view(torch.int32), b["pool"].ab.view(torch.int32))


CENTER_CASES = [c for c in CASES if c[0] in ("bf16_d128_multi_tile", "bf16_d64", "f32_d64", "f32_d128",
                                             "short_sequences", "tile_edges", "many_units_ragged")]


@pytest.mark.parametrize("representative", ["mean", "variation"])
@pytest.mark.parametrize("name,dtype,d,Hkv,T_list,N_list,values", CENTER_CASES, ids=[c[0] for c in CENTER_CASES])
def test_coarsen_centred_keys_matches_oracle(name, dtype, d, Hkv, T_list, N_list, values, representative):
    """Common-mode mean removal ("SPICY-KV" Claim 1(b)): the GPU's centred keys, built from its own
    fixed-order mean key, give c_t and boundaries bit-exact with the oracle's pipeline on the
    oracle's centred keys (a single differing bit of mu would move the fixed fp32 steps), and node
    statistics of the centred keys within tolerance. Keys carry a strong common mode."""
    seed = sum(T_list) + d + 5
    w = workloads.Workload(name, seed, B=len(T_list), Hq=Hkv, Hkv=Hkv, d=d, R=1,
                           dtype="bf16" if dtype == torch.bfloat16 else "f32", T=0, regimes=12)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list, values=values)
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = (k.float() + 6.0 * torch.randn(1, d, device="cuda", generator=g)).to(dtype)
    r = run_coarsen(k, v, Hkv, T_list, N_list, seed, representative=representative, center_keys=True)
    assert r["status"] == 0, f"device flags {r['flags']}"
    orc = oracle_units(k, v, Hkv, T_list, N_list, seed, representative=representative, center=True)
    compare_units(r, orc, k, v, T_list, Hkv, N_list, dtype, center=True)
    # the stored keys are centred: per unit the plain means average to about zero, weighted by mass
    for (b, h), u in orc.items():
        if representative == "mean" and u.kt.shape[0] and T_list[b] > 0:
            centre = (u.kt * u.mass[:, None]).sum(axis=0) / u.mass.sum()
            assert np.abs(centre).max() < 1e-3 * (1 + np.abs(to_np32(workloads.unit_rows(k, T_list, Hkv, b, h))).max())


def test_centred_tiny_f32_decode_keeps_outputs_and_shifts_lse():
    """tiny_f32 with a common mode added to the keys, coarsened with and without centring: the
    centred pool decodes to the same outputs (fp32 bar) and lse lower by q.mu/sqrt(d), mu the
    oracle's fixed-order mean key, whenever the two segmentations agree; and the centred pool's
    decode matches the oracle on the oracle's centred nodes."""
    w = workloads.WORKLOADS["tiny_f32"]
    k, v, T_list = workloads.make_kv(w, "cuda")
    k = k + 4.0 * torch.randn(1, w.d, device="cuda", generator=torch.Generator(device="cuda").manual_seed(3))
    N_list = workloads.segment_counts(w, T_list)
    plain = run_coarsen(k, v, w.Hkv, T_list, N_list, w.seed)
    cent = run_coarsen(k, v, w.Hkv, T_list, N_list, w.seed, center_keys=True)
    assert plain["status"] == 0 and cent["status"] == 0
    orc = oracle_units(k, v, w.Hkv, T_list, N_list, w.seed, center=True)
    compare_units(cent, orc, k, v, T_list, w.Hkv, N_list, torch.float32, center=True)
    q = workloads.make_queries(w, "cuda")
    out_c, lse_c = skv.decode_attn(q, w.Hkv, cent["pool"], cent["table"], cent["lens"])
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), [[orc[(0, 0)]]])
    check_decode(out_c, lse_c, ref_out, ref_lse, torch.float32, "centred tiny_f32")
    if torch.equal(plain["bnd"], cent["bnd"]):
        out_p, lse_p = skv.decode_attn(q, w.Hkv, plain["pool"], plain["table"], plain["lens"])
        mu = oracle.key_mean_f32(to_np32(k)).astype(np.float64)
        qq = q.double().cpu().numpy()
        shift = (qq @ mu) / np.sqrt(w.d)
        np.testing.assert_allclose(out_c.double().cpu().numpy(), out_p.double().cpu().numpy(), rtol=0, atol=2e-5)
        np.testing.assert_allclose(lse_p.double().cpu().numpy() - lse_c.double().cpu().numpy(), shift, rtol=0,
                                   atol=2e-4 * (1 + np.abs(shift).max()))


def tensor_units(r, k, v, Hkv, T_list, N_list, seed, representative="mean", center=False):
    """The stage-wise oracle of the tensor-core projection: every step within the bound of the exact
    bf16 projection's step, then the oracle's integer stages and statistics driven by the GPU's own
    steps (recovered from its cumulative variation)."""
    d = k.shape[-1]
    P16 = oracle.projection_bf16(seed, d)
    res = {}
    for b, T in enumerate(T_list):
        for h in range(Hkv):
            kk = to_np32(workloads.unit_rows(k, T_list, Hkv, b, h))
            vv = to_np32(workloads.unit_rows(v, T_list, Hkv, b, h))
            M = max(0, T - min(S, T) - min(W, T - min(S, T)))
            off = sum(T_list[:b]) * Hkv + h * T
            C = r["cum"][off:off + M].cpu().numpy()
            D = np.diff(C, prepend=0)
            dref, bound = oracle.tensor_steps_reference(kk, vv, S, W, P16)
            bad = np.flatnonzero(np.abs(D - dref) > bound)
            assert bad.size == 0, f"unit ({b},{h}): steps outside the bound at {bad[:5]}"
            assert M == 0 or D[0] == 0
            res[(b, h)] = oracle.coarsen_unit_from_steps(kk, vv, S, W, int(N_list[b]), D, representative, center)
    return res


TC_CASES = [c for c in CASES if c[1] == torch.bfloat16]


@pytest.mark.parametrize("name,dtype,d,Hkv,T_list,N_list,values", TC_CASES, ids=[c[0] for c in TC_CASES])
def test_coarsen_tensor_projection_stagewise(name, dtype, d, Hkv, T_list, N_list, values):
    """SKV_PROJECTION_TENSOR_BF16: steps within the fp32 accumulation bound of the exact bf16
    projection; given those steps, c_t, boundaries and entry counts bit-exact and node statistics
    within tolerance (the oracle's integer stages and statistics fed the GPU's steps)."""
    seed = sum(T_list) + d + 9
    w = workloads.Workload(name, seed, B=len(T_list), Hq=Hkv, Hkv=Hkv, d=d, R=1, dtype="bf16", T=0, regimes=12)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list, values=values)
    r = run_coarsen(k, v, Hkv, T_list, N_list, seed, projection="tensor")
    assert r["status"] == 0, f"device flags {r['flags']}"
    orc = tensor_units(r, k, v, Hkv, T_list, N_list, seed)
    compare_units(r, orc, k, v, T_list, Hkv, N_list, dtype)


def test_tensor_projection_with_centred_keys_and_weighted_representative():
    """The option composes with centring (the projection reads the raw keys; statistics are of the
    centred keys) and with the variation-weighted representative (weights are the GPU's steps)."""
    T_list, N_list, Hkv, d = [1300, 700], [40, 20], 2, 128
    seed = 77
    w = workloads.Workload("tc_combo", seed, B=2, Hq=Hkv, Hkv=Hkv, d=d, R=1, dtype="bf16", T=0, regimes=12)
    k, v, _ = workloads.make_kv(w, "cuda", T_list=T_list)
    k = (k.float() + 5.0).bfloat16()
    r = run_coarsen(k, v, Hkv, T_list, N_list, seed, projection="tensor", center_keys=True,
                    representative="variation")
    assert r["status"] == 0
    orc = tensor_units(r, k, v, Hkv, T_list, N_list, seed, representative="variation", center=True)
    compare_units(r, orc, k, v, T_list, Hkv, N_list, torch.bfloat16, center=True)


def test_tensor_projection_rejects_fp32_inputs():
    k = torch.zeros(200, 64, device="cuda")
    with pytest.raises(skv.SkvError):
        run_coarsen(k, k.clone(), 1, [200], [4], 1, projection="tensor")
