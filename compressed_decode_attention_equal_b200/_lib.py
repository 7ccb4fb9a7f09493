"""ctypes declarations of libskv's C ABI (include/skv.h)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libskv.so")

SKV_OK = 0
SKV_ERR_INVALID_ARG, SKV_ERR_UNSUPPORTED, SKV_ERR_CUDA, SKV_ERR_OVERFLOW = -1, -2, -3, -4
SKV_ERR_TIMEOUT, SKV_ERR_WORKSPACE, SKV_ERR_DEVICE = -5, -6, -7
SKV_F32, SKV_BF16 = 0, 1
PAGE_NODES = 16
PROJ_DIM = 16
MAX_SEQS = 512
NOALLOC_SCRATCH_BYTES = 4 << 20

FLAG_OVERFLOW, FLAG_BAD_PAGE, FLAG_BAD_LENS, FLAG_TIMEOUT = 1, 2, 4, 8


class SkvNodePool(ctypes.Structure):
    _fields_ = [("pages", ctypes.c_void_p), ("num_pages", ctypes.c_int64)]


SKV_REP_MEAN, SKV_REP_VARIATION_WEIGHTED = 0, 1
SKV_CLOSURE_SCALAR, SKV_CLOSURE_DIAGONAL = 0, 1
SKV_PROJECTION_FIXED_FP32, SKV_PROJECTION_TENSOR_BF16 = 0, 1


class SkvCoarsenOptions(ctypes.Structure):
    _fields_ = [("representative", ctypes.c_int32), ("closure", ctypes.c_int32), ("center_keys", ctypes.c_int32),
                ("projection", ctypes.c_int32), ("reserved", ctypes.c_int32 * 4)]


class SkvDecodeOptions(ctypes.Structure):
    _fields_ = [("closure", ctypes.c_int32), ("reserved", ctypes.c_int32 * 7)]


class SkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


# The header declares every symbol below; tests check that the library exports all of them.
EXPORTS = ("skv_status_string", "skv_abi_version", "skv_page_bytes", "skv_page_bytes_ex", "skv_projection_matrix",
           "skv_coarsen_workspace_bytes",
           "skv_coarsen", "skv_coarsen_ex", "skv_decode_workspace_bytes", "skv_decode_attn", "skv_decode_attn_ex", "skv_decode_attn_noalloc",
           "skv_stream_state_bytes", "skv_stream_init", "skv_stream_append",
           "skv_workspace_error", "skv_wait_selftest")

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libskv.so. Raises OSError if the library has not been built: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libskv.so not found at {path}; build it with "
                      f"`python -m compressed_decode_attention_equal_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    pi32 = ctypes.POINTER(ctypes.c_int32)
    lib.skv_status_string.argtypes = [i32]
    lib.skv_status_string.restype = ctypes.c_char_p
    lib.skv_abi_version.argtypes = []
    lib.skv_abi_version.restype = i32
    lib.skv_page_bytes.argtypes = [i32, i32]
    lib.skv_page_bytes.restype = sz
    lib.skv_page_bytes_ex.argtypes = [i32, i32, i32]
    lib.skv_page_bytes_ex.restype = sz
    lib.skv_projection_matrix.argtypes = [u64, i32, ctypes.POINTER(ctypes.c_float)]
    lib.skv_projection_matrix.restype = i32
    lib.skv_coarsen_workspace_bytes.argtypes = [i32, i32, i32, pi32, pi32, i32, i32]
    lib.skv_coarsen_workspace_bytes.restype = sz
    lib.skv_coarsen.argtypes = [vp, vp, i32, i32, i32, i32, pi32, i32, i32, pi32, u64,
                                ctypes.POINTER(SkvNodePool), vp, i32, vp, vp, vp, vp, sz, vp]
    lib.skv_coarsen.restype = i32
    lib.skv_coarsen_ex.argtypes = [vp, vp, i32, i32, i32, i32, pi32, i32, i32, pi32, u64,
                                   ctypes.POINTER(SkvNodePool), vp, i32, vp, vp, vp, vp, sz,
                                   ctypes.POINTER(SkvCoarsenOptions), vp]
    lib.skv_coarsen_ex.restype = i32
    lib.skv_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.skv_decode_workspace_bytes.restype = sz
    lib.skv_decode_attn.argtypes = [vp, i32, i32, i32, i32, i32, i32, ctypes.POINTER(SkvNodePool), vp, i32,
                                    vp, vp, vp, vp, sz, vp]
    lib.skv_decode_attn.restype = i32
    lib.skv_decode_attn_ex.argtypes = [vp, i32, i32, i32, i32, i32, i32, ctypes.POINTER(SkvNodePool), vp, i32,
                                       vp, vp, vp, vp, sz, ctypes.POINTER(SkvDecodeOptions), vp]
    lib.skv_decode_attn_ex.restype = i32
    lib.skv_stream_state_bytes.argtypes = [i32, i32, i32, pi32, i32, i32]
    lib.skv_stream_state_bytes.restype = sz
    lib.skv_stream_init.argtypes = [vp, vp, i32, i32, i32, i32, pi32, i32, i32, pi32, u64,
                                    ctypes.POINTER(SkvNodePool), vp, i32, vp, vp, sz, vp, sz, vp]
    lib.skv_stream_init.restype = i32
    lib.skv_stream_append.argtypes = [vp, vp, i32, i32, i32, i32, pi32, i32, i32,
                                      ctypes.POINTER(SkvNodePool), vp, i32, vp, vp, sz, vp, sz, vp]
    lib.skv_stream_append.restype = i32
    lib.skv_decode_attn_noalloc.argtypes = [vp, i32, i32, i32, i32, i32, i32, ctypes.POINTER(SkvNodePool), vp,
                                            i32, vp, vp, vp, vp]
    lib.skv_decode_attn_noalloc.restype = i32
    lib.skv_workspace_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.skv_workspace_error.restype = i32
    lib.skv_wait_selftest.argtypes = [vp, sz, ctypes.c_uint32, vp]
    lib.skv_wait_selftest.restype = i32
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().skv_status_string(status).decode()


def check(status: int, what: str):
    if status != SKV_OK:
        raise SkvError(status, what)
