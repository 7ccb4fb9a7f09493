"""skv_decode_attn_noalloc: decode attention for callers that cannot allocate device memory (a
plugin handed only its buffers, a runtime with a fixed allocator, a path where cudaMalloc may not
run). It keeps its scratch in an array the library defines at file scope instead of a caller
workspace, and launches the same kernel with the same grid as skv_decode_attn. These tests call it
through the C ABI on two calls in a row with different caches (the shared array keeps the previous
call's contents): its out and lse must equal skv_decode_attn's bit for bit, and one call is also
checked against the oracle fed the stored nodes, within the bf16 / fp32 parity bars."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
import oracle
from compressed_decode_attention_equal_b200 import _lib
from gpu_helpers import check_decode, gpu_units, pool_for_units, write_entries

pytestmark = pytest.mark.gpu


def _cache(B, Hq, Hkv, d, lens_list, seed, dtype=torch.bfloat16, R=1):
    g = torch.Generator(device="cpu").manual_seed(seed)
    pool, table = pool_for_units(lens_list, B, Hkv, d, dtype, shuffle=True, seed=seed)
    for b in range(B):
        for h in range(Hkv):
            E = int(lens_list[b])
            write_entries(pool, table, b, h, torch.randn(E, d, generator=g) * 3, torch.randn(E, d, generator=g),
                          torch.log(torch.randint(1, 200, (E,), generator=g).double()),
                          torch.rand(E, generator=g) * 0.02)
    lens = torch.tensor([[int(x)] * Hkv for x in lens_list], dtype=torch.int32, device="cuda")
    q = torch.randn(B, R, Hq, d, generator=g).to(dtype).cuda()
    return pool, table, lens, q


def _noalloc(q, Hkv, pool, table, lens):
    B, R, Hq, d = q.shape
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, R, Hq), float("nan"), dtype=torch.float32, device="cuda")
    ps = pool.struct()
    code = _lib.SKV_BF16 if q.dtype == torch.bfloat16 else _lib.SKV_F32
    st = _lib.load().skv_decode_attn_noalloc(
        ctypes.c_void_p(q.data_ptr()), code, B, R, Hq, Hkv, d, ctypes.byref(ps),
        ctypes.c_void_p(table.data_ptr()), table.shape[2], ctypes.c_void_p(lens.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_equals_workspace_entry_point_bit_for_bit_on_two_calls(dtype):
    B, Hq, Hkv, d = 8, 28, 4, 128
    caches = [_cache(B, Hq, Hkv, d, [1147, 37, 300, 1, 0, 700, 16, 2000], seed=s, dtype=dtype) for s in (41, 42)]
    for i, (pool, table, lens, q) in enumerate(caches):   # two calls in a row, different caches
        st, out_n, lse_n = _noalloc(q, Hkv, pool, table, lens)
        assert st == _lib.SKV_OK, _lib.status_string(st)
        out_w, lse_w = skv.decode_attn(q, Hkv, pool, table, lens)
        torch.cuda.synchronize()
        assert _same_bits(out_n, out_w), "out differs from skv_decode_attn"
        assert _same_bits(lse_n, lse_w), "lse differs from skv_decode_attn"
        if i == 1:   # the second call (scratch reused) against the oracle fed the stored nodes
            units = gpu_units(pool, table, lens, B, Hkv)
            ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), units)
            check_decode(out_n, lse_n, ref_out, ref_lse, dtype, "noalloc")


def test_noalloc_many_rows_stream_k_split():
    """14 query rows per KV head (2 rows x 7 heads) over ragged units: the stream-K split with
    global partials and merges in the scratch array, twice, against skv_decode_attn bit for bit
    (16-row passes at d = 64 keep the partials of the whole grid inside the 4 MiB array)."""
    B, Hq, Hkv, d = 6, 28, 4, 64
    for seed in (5, 6):
        pool, table, lens, q = _cache(B, Hq, Hkv, d, [900, 17, 400, 1500, 3, 260], seed=seed, R=2)
        st, out_n, lse_n = _noalloc(q, Hkv, pool, table, lens)
        assert st == _lib.SKV_OK, _lib.status_string(st)
        out_w, lse_w = skv.decode_attn(q, Hkv, pool, table, lens)
        torch.cuda.synchronize()
        assert _same_bits(out_n, out_w) and _same_bits(lse_n, lse_w)
        assert np.isfinite(lse_n.cpu().numpy()).all()


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 40 query rows per unit (two row passes of 32) over 16 units: the split partials exceed 4 MiB
    B, Hq, Hkv, d = 4, 32, 4, 128
    pool, table, lens, _ = _cache(B, Hq, Hkv, d, [64] * B, seed=7)
    q = torch.randn(B, 5, Hq, d).bfloat16().cuda()
    st, _, _ = _noalloc(q, Hkv, pool, table, lens)
    assert st == _lib.SKV_ERR_WORKSPACE
