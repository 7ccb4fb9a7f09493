"""The C-ABI library loads, exports every symbol include/skv.h declares, and rejects bad
arguments on the host before touching the GPU (not gpu: no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from compressed_decode_attention_equal_b200 import build, _lib
    build.build()
    return _lib.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "skv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(skv_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    from compressed_decode_attention_equal_b200 import _lib
    assert sorted(_lib.EXPORTS) == _declared()


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = lib.skv_status_string(code).decode()
        assert s.startswith("SKV_")
    assert "unknown" in lib.skv_status_string(12345).decode()
    assert lib.skv_abi_version() == 203
    assert lib.skv_page_bytes(1, 128) == 2 * 16 * 128 * 2 + 128
    assert lib.skv_page_bytes(0, 64) == 2 * 16 * 64 * 4 + 128
    assert lib.skv_page_bytes(1, 96) == 0


def test_workspace_queries_are_host_arithmetic(lib):
    from compressed_decode_attention_equal_b200 import coarsen_workspace_bytes, decode_workspace_bytes
    a = coarsen_workspace_bytes(4, 128, [32768] * 32, [1091] * 32, 8, 48)
    b = coarsen_workspace_bytes(4, 128, [32768] * 33, [1091] * 33, 8, 48)
    assert 0 < a < b
    assert coarsen_workspace_bytes(4, 96, [100], [4], 8, 48) == 0         # d unsupported
    assert coarsen_workspace_bytes(4, 128, [100], [0], 8, 48) == 0        # N < 1
    assert coarsen_workspace_bytes(4, 128, [1 << 22], [4], 8, 48) == 0    # too many tokens
    assert decode_workspace_bytes(32, 1, 28, 4, 128, 72) > 0
    assert decode_workspace_bytes(32, 1, 28, 5, 128, 72) == 0             # Hq % Hkv != 0
    assert decode_workspace_bytes(32, 1, 28, 4, 80, 72) == 0              # d unsupported


def test_bad_arguments_rejected_before_any_launch(lib):
    from compressed_decode_attention_equal_b200 import _lib
    null = ctypes.c_void_p(0)
    pool = _lib.SkvNodePool(0, 0)
    st = lib.skv_decode_attn(null, 1, 1, 1, 7, 1, 128, ctypes.byref(pool), null, 4, null, null, null, null, 0, null)
    assert st == _lib.SKV_ERR_INVALID_ARG
    st = lib.skv_decode_attn(null, 1, 1, 1, 7, 2, 128, ctypes.byref(pool), null, 4, null, null, null, null, 0, null)
    assert st == _lib.SKV_ERR_UNSUPPORTED
    st = lib.skv_decode_attn(null, 7, 1, 1, 7, 1, 128, ctypes.byref(pool), null, 4, null, null, null, null, 0, null)
    assert st == _lib.SKV_ERR_UNSUPPORTED
    T = (ctypes.c_int32 * 1)(100)
    N = (ctypes.c_int32 * 1)(4)
    st = lib.skv_coarsen(null, null, 1, 1, 1, 128, T, 8, 48, N, 0, None, null, 4, null, null, null, null, 0, null)
    assert st == _lib.SKV_ERR_INVALID_ARG
    st = lib.skv_coarsen(null, null, 3, 1, 1, 128, T, 8, 48, N, 0, None, null, 4, null, null, null, null, 0, null)
    assert st == _lib.SKV_ERR_UNSUPPORTED
    Tbad = (ctypes.c_int32 * 1)(-1)
    pool2 = _lib.SkvNodePool(16, 1)
    st = lib.skv_coarsen(null, null, 1, 1, 1, 128, Tbad, 8, 48, N, 0, ctypes.byref(pool2), ctypes.c_void_p(16), 4,
                         ctypes.c_void_p(16), null, null, null, 0, null)
    assert st == _lib.SKV_ERR_INVALID_ARG
    # workspace too small is reported before any launch
    st = lib.skv_coarsen(ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 1, 1, 128, T, 8, 48, N, 0,
                         ctypes.byref(pool2), ctypes.c_void_p(16), 4, ctypes.c_void_p(16), null, null,
                         ctypes.c_void_p(256), 16, null)
    assert st == _lib.SKV_ERR_WORKSPACE
    # page capacity: 8 + 4 + 48 = 60 entries need 4 pages of 16
    st = lib.skv_coarsen(ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 1, 1, 128, T, 8, 48, N, 0,
                         ctypes.byref(pool2), ctypes.c_void_p(16), 3, ctypes.c_void_p(16), null, null,
                         ctypes.c_void_p(256), 1 << 30, null)
    assert st == _lib.SKV_ERR_INVALID_ARG


def test_wait_selftest_and_noalloc_validated_before_any_launch(lib):
    """The wait check rejects a missing, misaligned or too small workspace and a poll count above
    the kernels' 2^20 limit before launching; the no-allocation decode applies skv_decode_attn's
    argument rules (shared planning code) before touching its scratch."""
    from compressed_decode_attention_equal_b200 import _lib
    null = ctypes.c_void_p(0)
    assert lib.skv_wait_selftest(null, 4096, 10, null) == _lib.SKV_ERR_WORKSPACE
    assert lib.skv_wait_selftest(ctypes.c_void_p(512 + 16), 4096, 10, null) == _lib.SKV_ERR_WORKSPACE
    assert lib.skv_wait_selftest(ctypes.c_void_p(512), 255, 10, null) == _lib.SKV_ERR_WORKSPACE
    assert lib.skv_wait_selftest(ctypes.c_void_p(512), 4096, (1 << 20) + 1, null) == _lib.SKV_ERR_INVALID_ARG
    pool = _lib.SkvNodePool(0, 0)
    for args, want in (((1, 1, 1, 7, 1, 128), _lib.SKV_ERR_INVALID_ARG),     # null buffers
                       ((1, 1, 1, 7, 2, 128), _lib.SKV_ERR_UNSUPPORTED),     # Hq % Hkv != 0
                       ((1, 1, 1, 7, 1, 96), _lib.SKV_ERR_UNSUPPORTED),      # d
                       ((1, 0, 1, 7, 1, 128), _lib.SKV_ERR_INVALID_ARG)):    # B < 1
        st = lib.skv_decode_attn_noalloc(null, *args, ctypes.byref(pool), null, 4, null, null, null, null)
        assert st == want, (args, st)


def test_coarsen_options_validated_before_any_launch(lib):
    from compressed_decode_attention_equal_b200 import _lib
    null = ctypes.c_void_p(0)
    T = (ctypes.c_int32 * 1)(100)
    N = (ctypes.c_int32 * 1)(4)
    pool2 = _lib.SkvNodePool(16, 1)
    args = (ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 1, 1, 128, T, 8, 48, N, 0, ctypes.byref(pool2),
            ctypes.c_void_p(16), 4, ctypes.c_void_p(16), null, null, ctypes.c_void_p(256), 16)
    bad_rep = _lib.SkvCoarsenOptions(2)
    assert lib.skv_coarsen_ex(*args, ctypes.byref(bad_rep), null) == _lib.SKV_ERR_INVALID_ARG
    bad_res = _lib.SkvCoarsenOptions(1)
    bad_res.reserved[3] = 1
    assert lib.skv_coarsen_ex(*args, ctypes.byref(bad_res), null) == _lib.SKV_ERR_INVALID_ARG
    # valid options fall through to the same checks as skv_coarsen (here: workspace too small)
    ok = _lib.SkvCoarsenOptions(_lib.SKV_REP_VARIATION_WEIGHTED)
    assert lib.skv_coarsen_ex(*args, ctypes.byref(ok), null) == _lib.SKV_ERR_WORKSPACE
    assert lib.skv_coarsen_ex(*args, None, null) == _lib.SKV_ERR_WORKSPACE


def test_page_bytes_and_closure_options(lib):
    from compressed_decode_attention_equal_b200 import _lib
    # [K | V | alpha,beta] and, for the diagonal closure, [K | V | alpha,beta | var]
    assert lib.skv_page_bytes_ex(1, 128, 0) == lib.skv_page_bytes(1, 128) == 2 * 16 * 128 * 2 + 128
    assert lib.skv_page_bytes_ex(1, 128, 1) == 3 * 16 * 128 * 2 + 128
    assert lib.skv_page_bytes_ex(0, 64, 1) == 3 * 16 * 64 * 4 + 128
    assert lib.skv_page_bytes_ex(1, 128, 2) == 0 and lib.skv_page_bytes_ex(1, 96, 1) == 0
    null = ctypes.c_void_p(0)
    pool = _lib.SkvNodePool(16, 1)
    args = (ctypes.c_void_p(256), 1, 1, 1, 7, 1, 128, ctypes.byref(pool), ctypes.c_void_p(16), 4,
            ctypes.c_void_p(16), ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), 16)
    bad = _lib.SkvDecodeOptions(2)
    assert lib.skv_decode_attn_ex(*args, ctypes.byref(bad), null) == _lib.SKV_ERR_INVALID_ARG
    bad_res = _lib.SkvDecodeOptions(1)
    bad_res.reserved[0] = 3
    assert lib.skv_decode_attn_ex(*args, ctypes.byref(bad_res), null) == _lib.SKV_ERR_INVALID_ARG
    ok = _lib.SkvDecodeOptions(_lib.SKV_CLOSURE_DIAGONAL)
    assert lib.skv_decode_attn_ex(*args, ctypes.byref(ok), null) == _lib.SKV_ERR_WORKSPACE
    T = (ctypes.c_int32 * 1)(100)
    N = (ctypes.c_int32 * 1)(4)
    cargs = (ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 1, 1, 128, T, 8, 48, N, 0, ctypes.byref(pool),
             ctypes.c_void_p(16), 4, ctypes.c_void_p(16), null, null, ctypes.c_void_p(256), 16)
    assert lib.skv_coarsen_ex(*cargs, ctypes.byref(_lib.SkvCoarsenOptions(0, 2)), null) == _lib.SKV_ERR_INVALID_ARG
    assert lib.skv_coarsen_ex(*cargs, ctypes.byref(_lib.SkvCoarsenOptions(1, 1)), null) == _lib.SKV_ERR_WORKSPACE


def test_stream_queries_and_validation(lib):
    from compressed_decode_attention_equal_b200 import _lib
    null = ctypes.c_void_p(0)
    N = (ctypes.c_int32 * 2)(20, 31)
    # projection block + 2 x 2 unit blocks; zero for invalid geometry
    one = lib.skv_stream_state_bytes(2, 2, 128, N, 8, 48)
    assert one > 16384 and (one - 16384) % 4 == 0 and (one - 16384) % 256 == 0
    assert lib.skv_stream_state_bytes(2, 2, 96, N, 8, 48) == 0
    assert lib.skv_stream_state_bytes(2, 2, 128, N, 8, 0) == 0           # needs a recent window
    big = (ctypes.c_int32 * 2)(9000, 1)
    assert lib.skv_stream_state_bytes(2, 2, 128, big, 8, 48) == 0        # above the node capacity
    T = (ctypes.c_int32 * 2)(56, 900)                                     # sequence 0 has no middle
    pool = _lib.SkvNodePool(16, 1)
    st = lib.skv_stream_init(ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 2, 2, 128, T, 8, 48, N, 0,
                             ctypes.byref(pool), ctypes.c_void_p(16), 80, ctypes.c_void_p(16), ctypes.c_void_p(256),
                             1 << 20, ctypes.c_void_p(256), one, null)
    assert st == _lib.SKV_ERR_UNSUPPORTED
    # append: a state smaller than the query, a workspace without the flag header, too few pages
    args = (ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 2, 2, 128, N, 8, 48, ctypes.byref(pool),
            ctypes.c_void_p(16))
    assert lib.skv_stream_append(*args, 80, ctypes.c_void_p(16), ctypes.c_void_p(256), one - 256,
                                 ctypes.c_void_p(256), 256, null) == _lib.SKV_ERR_WORKSPACE
    assert lib.skv_stream_append(*args, 80, ctypes.c_void_p(16), ctypes.c_void_p(256), one,
                                 ctypes.c_void_p(256), 16, null) == _lib.SKV_ERR_WORKSPACE
    assert lib.skv_stream_append(*args, 4, ctypes.c_void_p(16), ctypes.c_void_p(256), one,
                                 ctypes.c_void_p(256), 256, null) == _lib.SKV_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path):
    from compressed_decode_attention_equal_b200 import _lib
    saved = _lib._lib
    try:
        _lib._lib = None
        with pytest.raises(OSError):
            _lib.load(str(tmp_path / "missing.so"))
    finally:
        _lib._lib = saved


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_header_compiles_as_c_and_cpp_and_links(lib, tmp_path, compiler, std):
    """A translation unit that includes include/skv.h and takes the address of every declared entry
    point compiles warning-free as C99 and as C++17 (the extern "C" guards) and links against
    libskv.so; the program only counts the entry points (no CUDA call)."""
    import shutil
    import subprocess
    cc = shutil.which(compiler)
    if cc is None:
        pytest.skip(f"{compiler} not installed")
    names = _declared()
    body = ['#include "skv.h"', "#include <stdio.h>", "", "typedef void (*entry_fn)(void);", "",
            "int main(void) {", "    const entry_fn entries[] = {"]
    body += [f"        (entry_fn)&{n}," for n in names]
    body += ["    };", '    printf("%d\\n", (int)(sizeof entries / sizeof entries[0]));', "    return 0;", "}", ""]
    src = tmp_path / ("main.c" if compiler == "gcc" else "main.cpp")
    src.write_text("\n".join(body))
    libdir = os.path.dirname(lib._name)
    exe = tmp_path / "prog"
    subprocess.run([cc, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lskv", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    assert int(out) == len(names)
