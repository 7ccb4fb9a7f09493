"""The many-row decode's speculative set-up: without the aligned guess, the page prefix, the
stream-K split and the CTA's range are computed before the dependency wait from lens that a
preceding grid may still be writing, and rebuilt after the wait if the lens read then differ. A
helper kernel (tests/pdl_lens_writer.cu) lets the decode launch at once and overwrites the lens
only after a bounded sleep, so the decode's early read sees the old lens; the call must equal, bit
for bit, a call made with the final lens from the start (and likewise when the lens do not change)."""
import ctypes
import os
import subprocess

import pytest
import torch

import compressed_decode_attention_equal_b200 as skv
from gpu_helpers import pool_for_units

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def writer(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("pdl") / "libpdl_lens_writer.so")
    subprocess.run([os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc"), "-gencode", "arch=compute_100a,code=sm_100a",
                    "-O2", "-shared", "-Xcompiler", "-fPIC", "-o", so, os.path.join(HERE, "pdl_lens_writer.cu")],
                   check=True)
    lib = ctypes.CDLL(so)
    lib.launch_late_lens.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_void_p]
    lib.launch_late_lens.restype = ctypes.c_int
    return lib


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


@pytest.mark.parametrize("change", [True, False])
def test_speculative_setup_survives_lens_written_by_the_preceding_grid(writer, change):
    # 80 x 4 = 320 units (more than the grid's CTAs: the stream-K split, no aligned guess), 28 query
    # rows per KV head (rows as the MMA's M dimension)
    B, R, Hq, Hkv, d = 80, 4, 28, 4, 128
    g = torch.Generator(device="cpu").manual_seed(11)
    final = torch.randint(17, 400, (B, Hkv), generator=g, dtype=torch.int32)
    old = torch.randint(17, 400, (B, Hkv), generator=g, dtype=torch.int32) if change else final.clone()
    cap = torch.maximum(final, old).max(dim=1).values
    pool, table = pool_for_units(cap.tolist(), B, Hkv, d, torch.bfloat16, shuffle=True, seed=3)
    gd = torch.Generator(device="cuda").manual_seed(5)
    pool.k.copy_(torch.randn(pool.k.shape, generator=gd, device="cuda") * 3)
    pool.v.copy_(torch.randn(pool.v.shape, generator=gd, device="cuda"))
    pool.ab[..., 0] = torch.log(torch.randint(1, 60, pool.ab.shape[:2], generator=gd, device="cuda").float())
    pool.ab[..., 1] = torch.rand(pool.ab.shape[:2], generator=gd, device="cuda") * 1e-3
    q = torch.randn(B, R, Hq, d, generator=gd, device="cuda").bfloat16()
    final_d = final.cuda()
    ref_out, ref_lse = skv.decode_attn(q, Hkv, pool, table, final_d)
    torch.cuda.synchronize()
    # every buffer allocated up front: nothing but the writer runs between it and the decode
    out, lse = torch.empty_like(ref_out), torch.empty_like(ref_lse)
    ws = torch.zeros(skv.decode_workspace_bytes(B, R, Hq, Hkv, d, table.shape[2]), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        lens = old.cuda()
        out.fill_(float("nan"))
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream().cuda_stream
        st = writer.launch_late_lens(ctypes.c_void_p(lens.data_ptr()), ctypes.c_void_p(final_d.data_ptr()),
                                     lens.numel(), 1000, ctypes.c_void_p(stream))
        assert st == 0
        # may start while the writer sleeps
        skv.decode_attn(q, Hkv, pool, table, lens, out=out, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        st, flags = skv.workspace_error(ws)
        assert st == 0, flags
        assert torch.equal(lens.cpu(), final)
        assert _same_bits(out, ref_out) and _same_bits(lse, ref_lse)
