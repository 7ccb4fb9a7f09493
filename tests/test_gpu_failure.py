"""Failure reporting on the GPU without a GPU fault. A bounded device wait that runs out must be
reported to the host as SKV_ERR_TIMEOUT (flag bit 8) and leave the context usable: the check
launches one thread that waits on an mbarrier nothing arrives at (no copy outstanding), with a
short poll limit; the next decode call then still matches the oracle."""
import ctypes

import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
import oracle
from compressed_decode_attention_equal_b200 import _lib
from gpu_helpers import check_decode, gpu_units, pool_for_units, write_entries

pytestmark = pytest.mark.gpu


def _selftest(ws, polls):
    return _lib.load().skv_wait_selftest(ctypes.c_void_p(ws.data_ptr()), ws.numel(), polls,
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("polls", [0, 1000, 1 << 20])
def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable(polls):
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert _selftest(ws, polls) == _lib.SKV_OK
    st, flags = skv.workspace_error(ws)
    assert st == _lib.SKV_ERR_TIMEOUT and flags == _lib.FLAG_TIMEOUT
    st, flags = skv.workspace_error(ws)            # read-and-clear: the flag is gone
    assert st == _lib.SKV_OK and flags == 0

    # the same context decodes correctly afterwards
    B, Hq, Hkv, d = 2, 14, 2, 128
    lens_list = [300, 41]
    g = torch.Generator(device="cpu").manual_seed(polls & 0xffff)
    pool, table = pool_for_units(lens_list, B, Hkv, d, torch.bfloat16, shuffle=True, seed=3)
    for b in range(B):
        for h in range(Hkv):
            E = lens_list[b]
            write_entries(pool, table, b, h, torch.randn(E, d, generator=g) * 3, torch.randn(E, d, generator=g),
                          torch.log(torch.randint(1, 50, (E,), generator=g).double()),
                          torch.rand(E, generator=g) * 0.02)
    lens = torch.tensor([[x] * Hkv for x in lens_list], dtype=torch.int32, device="cuda")
    q = torch.randn(B, 1, Hq, d, generator=g).bfloat16().cuda()
    dws = torch.zeros(skv.decode_workspace_bytes(B, 1, Hq, Hkv, d, table.shape[2]), dtype=torch.uint8, device="cuda")
    out, lse = skv.decode_attn(q, Hkv, pool, table, lens, workspace=dws)
    st, flags = skv.workspace_error(dws)
    assert st == _lib.SKV_OK and flags == 0
    ref_out, ref_lse = oracle.decode(q.double().cpu().numpy(), gpu_units(pool, table, lens, B, Hkv))
    check_decode(out, lse, ref_out, ref_lse, torch.bfloat16, "decode after a timed-out wait")
