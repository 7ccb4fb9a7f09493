"""GPU parity of streaming coarsening (skv_stream_init / skv_stream_append) against oracle/stream.py.

After initialisation and after every block of appends, each unit's entries are matched with the
oracle's by first token: exact tokens exactly, middle nodes with bit-exact mass and variation V,
mean key / value within the node bar, alpha, beta; c_T bit-exact. Then decode attention over the
streamed pool (entries in no particular order) is compared with the oracle fed the GPU's entries."""
import numpy as np
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
import oracle
import workloads
from gpu_helpers import bf16_ulp, check_decode, gpu_units
from oracle.stream import StreamUnit

pytestmark = pytest.mark.gpu

S, W = workloads.N_SINK, workloads.N_RECENT
PROJ_BYTES = 2 * 128 * 16 * 4   # the state buffer starts with the projection P^T


def _layout(d, Ecap, W_):
    """Byte offsets of one unit's streaming state (the library's documented layout)."""
    up = lambda x: (x + 255) & ~255
    o, off = {}, up(128)
    for name, size in (("order", 4 * Ecap), ("recent", 4 * max(W_, 1)), ("owner", 4 * Ecap), ("m", 4 * Ecap),
                       ("start", 4 * Ecap), ("V", 8 * Ecap), ("M2", 8 * Ecap), ("mk", 8 * Ecap * d),
                       ("mv", 8 * Ecap * d), ("vord", 8 * Ecap), ("rpage", 4 * max(W_, 1)),
                       ("ring", 4 * 2 * max(W_, 1) * d)):
        o[name] = off
        off = up(off + size)
    o["unit"] = off
    return o


def _walk_units(B, Hkv, T_full, d, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = {}
    for b in range(B):
        for h in range(Hkv):
            T = T_full[b]
            k = torch.cumsum(torch.randn(T, d, generator=g) * 0.05, 0) + torch.randn(T, d, generator=g) * 0.02
            k[T // 3:] += torch.randn(1, d, generator=g) * 2.0          # a regime jump
            v = torch.randn(T, d, generator=g)
            out[(b, h)] = (k.bfloat16(), v.bfloat16())
    return out


def _gpu_entries(state, st_lay, unit, pool, table, lens, d):
    """{token: (m, V, kt, vt, alpha, beta)} of one unit, read back from the pool and the state."""
    base = PROJ_BYTES + unit * st_lay["unit"]
    raw = state[base:base + st_lay["unit"]].cpu().numpy()
    hdr = raw[:128]
    cT = int(hdr[0:8].view(np.int64)[0])
    T = int(hdr[12:16].view(np.int32)[0])
    ring = int(hdr[16:20].view(np.int32)[0])
    n_ent = int(hdr[20:24].view(np.int32)[0])
    Ecap = (st_lay["recent"] - st_lay["order"]) // 4
    owner = raw[st_lay["owner"]:st_lay["owner"] + 4 * Ecap].view(np.int32)
    m = raw[st_lay["m"]:st_lay["m"] + 4 * Ecap].view(np.int32)
    start = raw[st_lay["start"]:st_lay["start"] + 4 * Ecap].view(np.int32)
    V = raw[st_lay["V"]:st_lay["V"] + 8 * Ecap].view(np.int64)
    b, h = unit // lens.shape[1], unit % lens.shape[1]
    assert int(lens[b, h]) == n_ent
    kt, vt, al, be = skv.read_entries(pool, table, lens, b, h)
    kt, vt = kt.double().cpu().numpy(), vt.double().cpu().numpy()
    al, be = al.double().cpu().numpy(), be.double().cpu().numpy()
    ents = {}
    for e in range(n_ent):
        if owner[e] == -1:
            tok, mm, vv = e, 1, 0
        elif owner[e] <= -2:
            r = -2 - owner[e]
            tok, mm, vv = T - W + (r - ring) % W, 1, 0
        else:
            tok, mm, vv = int(start[e]), int(m[e]), int(V[e])
        assert tok not in ents, f"two entries start at token {tok}"
        ents[tok] = (mm, vv, kt[e], vt[e], al[e], be[e])
    return ents, cT


def _compare(ou: StreamUnit, ents, cT, what):
    assert cT == ou.cT, f"{what}: c_T"
    exp = ou.entries()
    assert len(exp) == len(ents), f"{what}: entry count {len(ents)} vs {len(exp)}"
    Vs = {n.start: n.V for n in ou.nodes}
    for tok, m, ekt, evt, eal, ebe in exp:
        assert tok in ents, f"{what}: no entry starts at token {tok}"
        gm, gV, gkt, gvt, gal, gbe = ents[tok]
        assert gm == m, f"{what}: mass at {tok}"
        assert gV == Vs.get(tok, 0), f"{what}: variation at {tok}"
        for g, o, name in ((gkt, ekt, "k"), (gvt, evt, "v")):
            bound = 0.5 * bf16_ulp(o) + 1e-6 * np.abs(o) + 1e-30
            assert np.all(np.abs(g - o) <= bound), f"{what}: {name} at {tok}"
        assert abs(gal - eal) <= 1e-6 * max(1.0, abs(eal)), f"{what}: alpha at {tok}"
        assert abs(gbe - ebe) <= 1e-5 * abs(ebe) + 1e-12, f"{what}: beta at {tok}"


@pytest.mark.parametrize("d,N_list,T0,steps", [
    (128, [20, 31], [700, 905], 170),
    (64, [1, 9], [200, 333], 120),
])
def test_stream_matches_oracle(d, N_list, T0, steps):
    B, Hkv = len(T0), 2
    T_full = [t + steps for t in T0]
    units = _walk_units(B, Hkv, T_full, d, seed=d + steps)
    seed = 77
    # the prompts in the packed layout: sequence b = [Hkv][T0_b][d]
    k0 = torch.cat([torch.cat([units[(b, h)][0][:T0[b]] for h in range(Hkv)]) for b in range(B)]).cuda()
    v0 = torch.cat([torch.cat([units[(b, h)][1][:T0[b]] for h in range(Hkv)]) for b in range(B)]).cuda()
    cap = skv.stream_capacity(N_list, S, W)
    pages = [-(-cap // 16)] * B
    table, num_pages = workloads.page_assignment(B, Hkv, pages, True, seed)
    table = table.cuda()
    pool = skv.NodePool(num_pages, d, torch.bfloat16)
    pool.k.fill_(float("nan"))
    pool.v.fill_(float("nan"))
    pool.ab.fill_(float("nan"))
    lens, state, ws = skv.stream_init(k0, v0, Hkv, T0, N_list, S, W, seed, pool, table)
    st_lay = _layout(d, cap, W)
    assert PROJ_BYTES + st_lay["unit"] * B * Hkv == state.numel()
    P = oracle.projection(seed, d)
    ous = {(b, h): StreamUnit(units[(b, h)][0][:T0[b]].float().numpy(), units[(b, h)][1][:T0[b]].float().numpy(),
                              S, W, N_list[b], P) for b in range(B) for h in range(Hkv)}
    for step in range(steps + 1):
        if step % 40 == 0 or step == steps:
            torch.cuda.synchronize()
            for (b, h), ou in ous.items():
                ents, cT = _gpu_entries(state, st_lay, b * Hkv + h, pool, table, lens, d)
                _compare(ou, ents, cT, f"unit ({b},{h}) after {step} appends")
        if step == steps:
            break
        k_new = torch.stack([torch.stack([units[(b, h)][0][T0[b] + step] for h in range(Hkv)]) for b in range(B)])
        v_new = torch.stack([torch.stack([units[(b, h)][1][T0[b] + step] for h in range(Hkv)]) for b in range(B)])
        skv.stream_append(k_new.cuda(), v_new.cuda(), N_list, S, W, pool, table, lens, state, ws)
        for (b, h), ou in ous.items():
            ou.append(units[(b, h)][0][T0[b] + step].float().numpy(), units[(b, h)][1][T0[b] + step].float().numpy())
    st, flags = skv.workspace_error(ws)
    assert st == 0, flags
    assert sum(ou.splits for ou in ous.values()) > 0 and sum(ou.merges for ou in ous.values()) > 0 or 1 in N_list
    # decode over the streamed pool (entries unordered) against the oracle fed the GPU's entries
    Hq = 4 * Hkv
    q = torch.randn(B, 1, Hq, d, generator=torch.Generator(device="cpu").manual_seed(5)).bfloat16().cuda()
    out, lse = skv.decode_attn(q, Hkv, pool, table, lens)
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), gpu_units(pool, table, lens, B, Hkv))
    check_decode(out, lse, ref_out, ref_lse, torch.bfloat16, "decode over the streamed pool")
