"""The Python binding's host-side checks (not gpu): shapes, dtypes, option names and device
placement are rejected before any library call, so a CPU tensor never reaches the C ABI and no
silent CPU path exists; the page and entry arithmetic matches the documented layout."""
import pytest
import torch

import compressed_decode_attention_equal_b200 as skv


def test_page_layout_and_entry_bounds():
    pool = skv.NodePool(3, 128, torch.bfloat16, device="cpu")
    assert pool.page_bytes == 2 * 16 * 128 * 2 + 16 * 8 == skv.page_bytes(torch.bfloat16, 128)
    assert pool.k.shape == pool.v.shape == (3, 16, 128) and pool.ab.shape == (3, 16, 2) and pool.var is None
    dpool = skv.NodePool(2, 64, torch.float32, device="cpu", closure="diagonal")
    assert dpool.page_bytes == 3 * 16 * 64 * 4 + 16 * 8 == skv.page_bytes(torch.float32, 64, "diagonal")
    assert dpool.var.shape == (2, 16, 64)
    # views alias the page bytes: key block, then value block, then (alpha, beta), then variances
    dpool.pages.zero_()
    dpool.ab[1, 3, 1] = 2.5
    raw = dpool.pages[1].view(torch.float32)
    assert raw[(2 * 16 * 64 * 4 + 3 * 8 + 4) // 4] == 2.5
    assert skv.entries_bound(32768, 1091, 8, 48) == 1147 and skv.pages_for(32768, 1091, 8, 48) == 72
    assert skv.entries_bound(50, 10, 8, 48) == 50             # no middle: every token exact
    assert skv.entries_bound(57, 10, 8, 48) == 8 + 10 + 48    # one middle token, N segments at most
    assert skv.stream_capacity([20, 31], 8, 48) == 8 + 31 + 1 + 48


def test_option_names_are_checked():
    with pytest.raises(ValueError):
        skv.NodePool(1, 128, torch.bfloat16, device="cpu", closure="full")
    k = torch.zeros(100, 128, dtype=torch.bfloat16)
    pool = skv.NodePool(8, 128, torch.bfloat16, device="cpu")
    table = torch.zeros(1, 1, 8, dtype=torch.int32)
    with pytest.raises(ValueError):
        skv.coarsen(k, k, 1, [100], [4], 8, 48, 0, pool, table, representative="median")


@pytest.mark.parametrize("case", ["kv_mismatch", "pool_dtype", "table_dtype", "table_shape", "cpu_tensor"])
def test_coarsen_arguments_rejected_before_the_library(case):
    k = torch.zeros(100, 128, dtype=torch.bfloat16)
    v = k.clone()
    pool = skv.NodePool(8, 128, torch.bfloat16, device="cpu")
    table = torch.zeros(1, 1, 8, dtype=torch.int32)
    if case == "kv_mismatch":
        v = torch.zeros(100, 128, dtype=torch.float32)
    elif case == "pool_dtype":
        pool = skv.NodePool(8, 128, torch.float32, device="cpu")
    elif case == "table_dtype":
        table = table.long()
    elif case == "table_shape":
        table = torch.zeros(1, 8, dtype=torch.int32)
    msg = {"kv_mismatch": "same shape and dtype", "pool_dtype": "pool dtype", "table_dtype": "page_table",
           "table_shape": "page_table", "cpu_tensor": "CUDA tensor"}[case]
    with pytest.raises(ValueError, match=msg):
        skv.coarsen(k, v, 1, [100], [4], 8, 48, 0, pool, table, lens=torch.zeros(1, 1, dtype=torch.int32),
                    workspace=torch.zeros(1 << 20, dtype=torch.uint8))


@pytest.mark.parametrize("case", ["pool_dtype", "pool_d", "table_dtype", "lens_shape", "cpu_tensor"])
def test_decode_arguments_rejected_before_the_library(case):
    q = torch.zeros(1, 1, 7, 128, dtype=torch.bfloat16)
    pool = skv.NodePool(4, 128, torch.bfloat16, device="cpu")
    table = torch.zeros(1, 1, 4, dtype=torch.int32)
    lens = torch.zeros(1, 1, dtype=torch.int32)
    if case == "pool_dtype":
        pool = skv.NodePool(4, 128, torch.float32, device="cpu")
    elif case == "pool_d":
        pool = skv.NodePool(4, 64, torch.bfloat16, device="cpu")
    elif case == "table_dtype":
        table = table.long()
    elif case == "lens_shape":
        lens = torch.zeros(2, dtype=torch.int32)
    msg = {"pool_dtype": "pool dtype", "pool_d": "pool dtype", "table_dtype": "page_table", "lens_shape": "lens",
           "cpu_tensor": "CUDA tensor"}[case]
    with pytest.raises(ValueError, match=msg):
        skv.decode_attn(q, 1, pool, table, lens, out=torch.empty_like(q), lse=torch.empty(1, 1, 7),
                        workspace=torch.zeros(1 << 20, dtype=torch.uint8))


def test_unsupported_dtype_is_a_type_error():
    with pytest.raises(TypeError):
        skv.page_bytes(torch.float16, 128)
