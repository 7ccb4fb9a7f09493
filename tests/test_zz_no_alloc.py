"""skv_decode_attn_noalloc: decode attention for callers that cannot allocate device memory (for
example code recorded into someone else's CUDA graph, or a plugin given only its buffers). It keeps
its scratch in an array the library defines at file scope instead of a caller workspace. These
tests call it through the C ABI and compare it with skv_decode_attn on the same inputs, on two
calls in a row with different caches (the shared array keeps the previous call's contents)."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
from compressed_decode_attention_equal_b200 import _lib
from gpu_helpers import TOL_BF16_MAX_ABS, TOL_BF16_REL_L2, TOL_LSE_ABS, pool_for_units, rel_l2, write_entries

pytestmark = pytest.mark.gpu


def _cache(B, Hq, Hkv, d, lens_list, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    pool, table = pool_for_units(lens_list, B, Hkv, d, torch.bfloat16, shuffle=True, seed=seed)
    for b in range(B):
        for h in range(Hkv):
            E = int(lens_list[b])
            write_entries(pool, table, b, h, torch.randn(E, d, generator=g) * 3, torch.randn(E, d, generator=g),
                          torch.log(torch.randint(1, 200, (E,), generator=g).double()),
                          torch.rand(E, generator=g) * 0.02)
    lens = torch.tensor([[int(x)] * Hkv for x in lens_list], dtype=torch.int32, device="cuda")
    q = torch.randn(B, 1, Hq, d, generator=g).bfloat16().cuda()
    return pool, table, lens, q


def _noalloc(q, Hkv, pool, table, lens):
    B, R, Hq, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, R, Hq, dtype=torch.float32, device="cuda")
    ps = pool.struct()
    st = _lib.load().skv_decode_attn_noalloc(
        ctypes.c_void_p(q.data_ptr()), _lib.SKV_BF16, B, R, Hq, Hkv, d, ctypes.byref(ps),
        ctypes.c_void_p(table.data_ptr()), table.shape[2], ctypes.c_void_p(lens.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    B, Hq, Hkv, d = 8, 28, 4, 128
    caches = [_cache(B, Hq, Hkv, d, [1147, 37, 300, 1, 0, 700, 16, 2000], seed=s) for s in (41, 42)]
    for pool, table, lens, q in caches:           # two calls in a row, different caches
        st, out_n, lse_n = _noalloc(q, Hkv, pool, table, lens)
        assert st == _lib.SKV_OK, _lib.status_string(st)
        out_w, lse_w = skv.decode_attn(q, Hkv, pool, table, lens)
        torch.cuda.synchronize()
        og, ow = out_n.double().cpu().numpy(), out_w.double().cpu().numpy()
        assert rel_l2(og, ow) <= TOL_BF16_REL_L2
        assert np.abs(og - ow).max() <= TOL_BF16_MAX_ABS
        ln, lw = lse_n.double().cpu().numpy(), lse_w.double().cpu().numpy()
        assert np.array_equal(np.isneginf(ln), np.isneginf(lw))
        fin = np.isfinite(lw)
        assert np.abs(ln[fin] - lw[fin]).max() <= TOL_LSE_ABS


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 40 query rows per unit (two row passes of 32) over 16 units: the split partials exceed 4 MiB
    B, Hq, Hkv, d = 4, 32, 4, 128
    pool, table, lens, _ = _cache(B, Hq, Hkv, d, [64] * B, seed=7)
    q = torch.randn(B, 5, Hq, d).bfloat16().cuda()
    st, _, _ = _noalloc(q, Hkv, pool, table, lens)
    assert st == _lib.SKV_ERR_WORKSPACE
