"""Equal-variation KV-cache coarsening and compressed decode attention for B200.

A thin binding over libskv's C ABI (include/skv.h): torch tensors are checked
and passed as raw device pointers with the current CUDA stream. Every step of
both operations runs in libskv's sm_100a kernels; there is no CPU or PyTorch
fallback, and a missing library raises at the first call.

  coarsen(...)      "Equal-Variation KV Cache" (synthcore idea 664) segmentation
                    of each (sequence, KV head) history into macro-nodes with
                    "SPICY-KV" node statistics (mass, mean key/value, variance)
  decode_attn(...)  "SPICY-KV" section 2 decode logit
                    q.k/sqrt(d) + ln m + |q|^2 sigma^2/(2d) with online softmax
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import PAGE_NODES, SkvError

__all__ = ["NodePool", "coarsen", "decode_attn", "coarsen_workspace_bytes", "decode_workspace_bytes",
           "workspace_error", "projection_matrix", "entries_bound", "pages_for", "page_bytes", "read_entries",
           "SkvError", "PAGE_NODES", "library_path"]


def library_path() -> str:
    return _lib.LIB_PATH


def _code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return _lib.SKV_BF16
    if dtype == torch.float32:
        return _lib.SKV_F32
    raise TypeError(f"unsupported dtype {dtype}; use torch.bfloat16 or torch.float32")


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dev(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _i32(xs):
    return (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])


def entries_bound(T: int, N: int, n_sink: int, n_recent: int) -> int:
    """Upper bound on the entries one unit produces: sinks + N segments (if any middle) + recents."""
    s = min(n_sink, T)
    r = min(n_recent, T - s)
    return s + (N if T - s - r > 0 else 0) + r


def pages_for(T: int, N: int, n_sink: int, n_recent: int) -> int:
    return -(-entries_bound(T, N, n_sink, n_recent) // PAGE_NODES)


CLOSURES = {"scalar": _lib.SKV_CLOSURE_SCALAR, "diagonal": _lib.SKV_CLOSURE_DIAGONAL}


class NodePool:
    """Paged macro-node storage: one uint8 tensor `pages` [num_pages, page_bytes]; page p holds 16
    entries of one unit as [keys 16 x d | values 16 x d | {alpha, beta} 16 x 2 fp32] (alpha = ln m,
    beta = sigma^2 / (2d)), followed for closure="diagonal" by [per-dimension key variances 16 x d].
    `k`, `v`, `ab` (and `var`) are strided views of those blocks. Within the vector blocks, 16-byte
    chunk c of slot n is stored at chunk c ^ (n & 7). coarsen() and decode_attn() use the pool's
    closure."""

    def __init__(self, num_pages: int, d: int, dtype: torch.dtype, device="cuda", closure: str = "scalar"):
        if closure not in CLOSURES:
            raise ValueError(f"closure must be one of {sorted(CLOSURES)}")
        self.num_pages, self.d, self.dtype, self.closure = int(num_pages), int(d), dtype, closure
        elem = torch.tensor([], dtype=dtype).element_size()
        self.vec_bytes = PAGE_NODES * d * elem
        self.page_bytes = (3 if closure == "diagonal" else 2) * self.vec_bytes + PAGE_NODES * 8
        P = self.num_pages
        self.pages = torch.empty(P, self.page_bytes, dtype=torch.uint8, device=device)
        vb = self.vec_bytes
        self.k = self.pages[:, :vb].view(dtype).view(P, PAGE_NODES, d)
        self.v = self.pages[:, vb:2 * vb].view(dtype).view(P, PAGE_NODES, d)
        self.ab = self.pages[:, 2 * vb:2 * vb + PAGE_NODES * 8].view(torch.float32).view(P, PAGE_NODES, 2)
        self.var = (self.pages[:, 2 * vb + PAGE_NODES * 8:].view(dtype).view(P, PAGE_NODES, d)
                    if closure == "diagonal" else None)

    def struct(self) -> _lib.SkvNodePool:
        return _lib.SkvNodePool(self.pages.data_ptr(), self.num_pages)

    def nbytes(self) -> int:
        return self.pages.numel()


def projection_matrix(seed: int, d: int) -> torch.Tensor:
    """The 16 x 2d projection skv_coarsen draws from `seed` (computed on the host)."""
    out = torch.empty(16, 2 * d, dtype=torch.float32)
    _lib.check(_lib.load().skv_projection_matrix(ctypes.c_uint64(seed), d,
                                                  ctypes.cast(out.data_ptr(), ctypes.POINTER(ctypes.c_float))),
               "skv_projection_matrix")
    return out


def coarsen_workspace_bytes(Hkv: int, d: int, T_list, N_list, n_sink: int, n_recent: int) -> int:
    B = len(T_list)
    return int(_lib.load().skv_coarsen_workspace_bytes(B, Hkv, d, _i32(T_list), _i32(N_list), n_sink, n_recent))


def coarsen(k: torch.Tensor, v: torch.Tensor, Hkv: int, T_list, N_list, n_sink: int, n_recent: int,
            proj_seed: int, pool: NodePool, page_table: torch.Tensor, lens: torch.Tensor | None = None,
            boundaries: torch.Tensor | None = None, cumvar: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, stream=None, representative: str = "mean",
            center_keys: bool = False, projection: str = "fixed") -> torch.Tensor:
    """Coarsen B sequences (k, v: [sum_b Hkv*T_b, d], sequence b a contiguous [Hkv, T_b, d] block)
    into `pool` through `page_table` [B, Hkv, max_pages] int32. Returns lens [B, Hkv] int32.
    representative: "mean" (skv_coarsen) or "variation" (skv_coarsen_ex with the
    variation-weighted segment key and value). center_keys: skv_coarsen_ex's common-mode mean
    removal (every key of a unit enters with the unit's mean key subtracted). projection: "fixed"
    (the fixed fp32 recipe) or "tensor" (skv_coarsen_ex's tensor-core bf16 projection)."""
    reps = {"mean": _lib.SKV_REP_MEAN, "variation": _lib.SKV_REP_VARIATION_WEIGHTED}
    projs = {"fixed": _lib.SKV_PROJECTION_FIXED_FP32, "tensor": _lib.SKV_PROJECTION_TENSOR_BF16}
    if representative not in reps:
        raise ValueError(f"representative must be one of {sorted(reps)}")
    if projection not in projs:
        raise ValueError(f"projection must be one of {sorted(projs)}")
    B = len(T_list)
    d = k.shape[-1]
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k and v must have the same shape and dtype")
    if pool.dtype != k.dtype or pool.d != d:
        raise ValueError("pool dtype / d must match k")
    if page_table.dtype != torch.int32 or page_table.dim() != 3 or tuple(page_table.shape[:2]) != (B, Hkv):
        raise ValueError("page_table must be int32 [B, Hkv, max_pages]")
    dev = k.device
    if lens is None:
        lens = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    ws_bytes = coarsen_workspace_bytes(Hkv, d, T_list, N_list, n_sink, n_recent)
    if ws_bytes == 0:
        raise SkvError(_lib.SKV_ERR_INVALID_ARG, "skv_coarsen_workspace_bytes")
    if workspace is None:
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    ps = pool.struct()
    null = ctypes.c_void_p(0)
    args = (_dev(k, "k") if k.numel() else null, _dev(v, "v") if v.numel() else null, _code(k.dtype), B, Hkv, d,
            _i32(T_list), n_sink, n_recent, _i32(N_list), ctypes.c_uint64(proj_seed), ctypes.byref(ps),
            _dev(page_table, "page_table"), page_table.shape[2], _dev(lens, "lens"),
            _dev(boundaries, "boundaries") if boundaries is not None else null,
            _dev(cumvar, "cumvar") if cumvar is not None else null,
            _dev(workspace, "workspace"), workspace.numel())
    if representative == "mean" and pool.closure == "scalar" and not center_keys and projection == "fixed":
        st = _lib.load().skv_coarsen(*args, ctypes.c_void_p(_stream_handle(stream)))
        _lib.check(st, "skv_coarsen")
    else:
        opts = _lib.SkvCoarsenOptions(reps[representative], CLOSURES[pool.closure], 1 if center_keys else 0,
                                      projs[projection])
        st = _lib.load().skv_coarsen_ex(*args, ctypes.byref(opts), ctypes.c_void_p(_stream_handle(stream)))
        _lib.check(st, "skv_coarsen_ex")
    return lens


def stream_state_bytes(Hkv: int, d: int, N_list, n_sink: int, n_recent: int) -> int:
    return int(_lib.load().skv_stream_state_bytes(len(N_list), Hkv, d, _i32(N_list), n_sink, n_recent))


def stream_capacity(N_list, n_sink: int, n_recent: int) -> int:
    """Entries a streamed unit may hold at once (its page-table row must cover them)."""
    return n_sink + max(int(n) for n in N_list) + 1 + n_recent


def stream_init(k: torch.Tensor, v: torch.Tensor, Hkv: int, T_list, N_list, n_sink: int, n_recent: int,
                proj_seed: int, pool: NodePool, page_table: torch.Tensor, lens: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, state: torch.Tensor | None = None, stream=None):
    """Coarsen the prompts (as coarsen()) and build the streaming state. Returns (lens, state, workspace);
    pass all three to stream_append."""
    B = len(T_list)
    d = k.shape[-1]
    if pool.closure != "scalar":
        raise ValueError("streaming coarsening keeps scalar-closure pools")
    dev = k.device
    if lens is None:
        lens = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    ws_bytes = coarsen_workspace_bytes(Hkv, d, T_list, N_list, n_sink, n_recent)
    if workspace is None:
        workspace = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    st_bytes = stream_state_bytes(Hkv, d, N_list, n_sink, n_recent)
    if st_bytes == 0:
        raise SkvError(_lib.SKV_ERR_INVALID_ARG, "skv_stream_state_bytes")
    if state is None:
        state = torch.zeros(st_bytes, dtype=torch.uint8, device=dev)
    ps = pool.struct()
    st = _lib.load().skv_stream_init(
        _dev(k, "k"), _dev(v, "v"), _code(k.dtype), B, Hkv, d, _i32(T_list), n_sink, n_recent, _i32(N_list),
        ctypes.c_uint64(proj_seed), ctypes.byref(ps), _dev(page_table, "page_table"), page_table.shape[2],
        _dev(lens, "lens"), _dev(workspace, "workspace"), workspace.numel(), _dev(state, "state"), state.numel(),
        ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "skv_stream_init")
    return lens, state, workspace


def stream_append(k_new: torch.Tensor, v_new: torch.Tensor, N_list, n_sink: int, n_recent: int,
                  pool: NodePool, page_table: torch.Tensor, lens: torch.Tensor, state: torch.Tensor,
                  workspace: torch.Tensor, stream=None):
    """Append one token per unit (k_new, v_new: [B, Hkv, d]) to streamed caches."""
    B, Hkv, d = k_new.shape
    ps = pool.struct()
    st = _lib.load().skv_stream_append(
        _dev(k_new, "k_new"), _dev(v_new, "v_new"), _code(k_new.dtype), B, Hkv, d, _i32(N_list), n_sink, n_recent,
        ctypes.byref(ps), _dev(page_table, "page_table"), page_table.shape[2],
        _dev(lens, "lens"), _dev(state, "state"), state.numel(), _dev(workspace, "workspace"), workspace.numel(),
        ctypes.c_void_p(_stream_handle(stream)))
    _lib.check(st, "skv_stream_append")


def decode_workspace_bytes(B: int, R: int, Hq: int, Hkv: int, d: int, max_pages: int) -> int:
    return int(_lib.load().skv_decode_workspace_bytes(B, R, Hq, Hkv, d, max_pages))


def decode_attn(q: torch.Tensor, Hkv: int, pool: NodePool, page_table: torch.Tensor, lens: torch.Tensor,
                out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None):
    """q [B, R, Hq, d] against the compressed cache. Returns (out [B, R, Hq, d], lse [B, R, Hq] fp32)."""
    B, R, Hq, d = q.shape
    if pool.dtype != q.dtype or pool.d != d:
        raise ValueError("pool dtype / d must match q")
    if page_table.dtype != torch.int32 or page_table.dim() != 3 or tuple(page_table.shape[:2]) != (B, Hkv):
        raise ValueError("page_table must be int32 [B, Hkv, max_pages]")
    if lens.dtype != torch.int32 or tuple(lens.shape) != (B, Hkv):
        raise ValueError("lens must be int32 [B, Hkv]")
    max_pages = page_table.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, R, Hq, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.zeros(decode_workspace_bytes(B, R, Hq, Hkv, d, max_pages), dtype=torch.uint8,
                                device=q.device)
    ps = pool.struct()
    args = (_dev(q, "q"), _code(q.dtype), B, R, Hq, Hkv, d, ctypes.byref(ps), _dev(page_table, "page_table"),
            max_pages, _dev(lens, "lens"), _dev(out, "out"), _dev(lse, "lse"), _dev(workspace, "workspace"),
            workspace.numel())
    if pool.closure == "scalar":
        st = _lib.load().skv_decode_attn(*args, ctypes.c_void_p(_stream_handle(stream)))
        _lib.check(st, "skv_decode_attn")
    else:
        opts = _lib.SkvDecodeOptions(CLOSURES[pool.closure])
        st = _lib.load().skv_decode_attn_ex(*args, ctypes.byref(opts), ctypes.c_void_p(_stream_handle(stream)))
        _lib.check(st, "skv_decode_attn_ex")
    return out, lse


def workspace_error(workspace: torch.Tensor, stream=None):
    """Synchronise and read-and-clear the device error flags of a workspace: (status, flags)."""
    flags = ctypes.c_uint32(0)
    st = _lib.load().skv_workspace_error(_dev(workspace, "workspace"), ctypes.c_void_p(_stream_handle(stream)),
                                         ctypes.byref(flags))
    return st, flags.value


def page_bytes(dtype: torch.dtype, d: int, closure: str = "scalar") -> int:
    return int(_lib.load().skv_page_bytes_ex(_code(dtype), d, CLOSURES[closure]))


def _entry_rows(pool: NodePool, page_table: torch.Tensor, b: int, h: int, E: int):
    n_pages = -(-E // PAGE_NODES)
    pages = page_table[b, h, :n_pages].long()
    slots = torch.arange(PAGE_NODES, device=pages.device)
    pg = pages[:, None].expand(n_pages, PAGE_NODES).reshape(-1)[:E]
    sl = slots[None, :].expand(n_pages, PAGE_NODES).reshape(-1)[:E]
    return pg, sl


def read_variances(pool: NodePool, page_table: torch.Tensor, lens: torch.Tensor, b: int, h: int):
    """Per-dimension key variances [E, d] of unit (b, h) in entry order (a diagonal pool)."""
    if pool.var is None:
        raise ValueError("the pool holds no per-dimension variances (closure='scalar')")
    E = int(lens[b, h])
    d = pool.d
    if E == 0:
        return pool.var.new_zeros(0, d)
    pg, sl = _entry_rows(pool, page_table, b, h, E)
    epc = 16 // pool.var.element_size()
    ch = d // epc
    phys = torch.arange(ch, device=pg.device)[None, :] ^ (sl[:, None] & 7)
    return pool.var.view(pool.num_pages, PAGE_NODES, ch, epc)[pg[:, None], sl[:, None], phys].reshape(E, d)


def read_entries(pool: NodePool, page_table: torch.Tensor, lens: torch.Tensor, b: int, h: int):
    """Entries of unit (b, h) in entry order, un-swizzled: (kt [E, d], vt [E, d], alpha [E], beta [E]).
    A layout view for inspection (indexing only)."""
    E = int(lens[b, h])
    d = pool.d
    if E == 0:
        z = pool.k.new_zeros(0, d)
        return z, z.clone(), pool.ab.new_zeros(0), pool.ab.new_zeros(0)
    pg, sl = _entry_rows(pool, page_table, b, h, E)
    epc = 16 // pool.k.element_size()
    ch = d // epc
    phys = torch.arange(ch, device=pg.device)[None, :] ^ (sl[:, None] & 7)
    k4 = pool.k.view(pool.num_pages, PAGE_NODES, ch, epc)
    v4 = pool.v.view(pool.num_pages, PAGE_NODES, ch, epc)
    kt = k4[pg[:, None], sl[:, None], phys].reshape(E, d)
    vt = v4[pg[:, None], sl[:, None], phys].reshape(E, d)
    ab = pool.ab[pg, sl]
    return kt, vt, ab[:, 0], ab[:, 1]
