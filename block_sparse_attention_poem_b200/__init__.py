"""Python binding of libpoem (include/poem.h): POEM output-relative block-sparse
attention prefill on B200 (sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libpoem.so``; PyTorch supplies device memory and the current stream.  The
library is loaded from this package directory and there is no fallback: if it
is missing or fails to load, importing the binding raises.

Functions carry the C names:
    poem_workspace_size(shape) -> (score_bytes, select_bytes, fwd_bytes)
    poem_score(q, k, v, I_hat, m_hat, ws, block=128, n_sample=16, scale=0.0)
    poem_select(I_hat, m_hat, tau, row_ptr, col_idx, ws, shape..., order=None)
    poem_select_mass_only(m_hat, ref_row_ptr, row_ptr, col_idx, ws, ...)
    poem_select_ranked_budget(shape, score, ref_row_ptr, row_ptr, col_idx, ws, ...)
    poem_select_per_head(shape, I_hat, m_hat, tau_per_head, row_ptr, col_idx, ws, ...)
    poem_select_practical_per_head(shape, m_pool, d_pool, w, gamma_per_head, rho, ...)
    bsa_fwd(q, k, v, row_ptr, col_idx, o, ws, lse=None, order=None, block=128)
    poem_check(ws) -> raises on a device-side error
    poem_pooled_workspace_size(shape) -> bytes
    poem_score_pooled(q, k, v, m_pool, d_pool, ws, ...)
    poem_select_practical(shape, m_pool, d_pool, w, gamma, rho, row_ptr, col_idx, ws, order=None)
``prefill_layer`` chains the three exact calls for one attention layer and
``prefill_layer_practical`` the practical (pooled-estimate) selector's.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# POEM_LIBRARY_VARIANT=checks selects the debug build (device bounds checks,
# libpoem_checks.so from build.py's "checks" variant); there is no other choice and
# no fallback: a missing library fails the import.
_VARIANT = os.environ.get("POEM_LIBRARY_VARIANT", "release")
if _VARIANT not in ("release", "checks"):
    raise ImportError(f"POEM_LIBRARY_VARIANT must be 'release' or 'checks', not {_VARIANT!r}")
LIB_PATH = os.path.join(_HERE, "libpoem.so" if _VARIANT == "release" else "libpoem_checks.so")

POEM_OK = 0
STATUS = {
    0: "POEM_OK", 1: "POEM_ERR_INVALID_ARG", 2: "POEM_ERR_UNSUPPORTED", 3: "POEM_ERR_CUDA",
    4: "POEM_ERR_TIMEOUT", 5: "POEM_ERR_CAPACITY", 6: "POEM_ERR_WORKSPACE", 7: "POEM_ERR_BAD_LIST",
    8: "POEM_ERR_BOUNDS",
}

EXPORTED = (
    "poem_workspace_size", "poem_score", "poem_select", "poem_select_mass_only", "bsa_fwd",
    "poem_check", "poem_set_wait_limit_ns", "poem_status_string", "poem_last_error", "poem_select_noalloc",
    "poem_pooled_workspace_size", "poem_score_pooled", "poem_select_practical", "poem_select_ranked_budget",
    "poem_select_per_head", "poem_select_practical_per_head", "bsa_fwd_grouped",
)


class PoemError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class Shape(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32), ("n_sample", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("q_offset", ctypes.c_int32),
        ("q_stride_tok", ctypes.c_int64), ("q_stride_head", ctypes.c_int64),
        ("kv_stride_tok", ctypes.c_int64), ("kv_stride_head", ctypes.c_int64),
        ("o_stride_tok", ctypes.c_int64), ("o_stride_head", ctypes.c_int64),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run block_sparse_attention_poem_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sp, i64, sz = ctypes.c_void_p, ctypes.POINTER(Shape), ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    lib.poem_workspace_size.argtypes = [sp, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.poem_workspace_size.restype = st
    lib.poem_score.argtypes = [sp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.poem_score.restype = st
    lib.poem_select.argtypes = [sp, vp, vp, ctypes.c_float, vp, vp, i64, vp, vp, sz, vp]
    lib.poem_select.restype = st
    lib.poem_select_mass_only.argtypes = [sp, vp, vp, vp, vp, i64, vp, vp, sz, vp]
    lib.poem_select_mass_only.restype = st
    lib.poem_select_per_head.argtypes = [sp, vp, vp, vp, vp, vp, i64, vp, vp, sz, vp]
    lib.poem_select_per_head.restype = st
    lib.poem_select_practical_per_head.argtypes = [sp, vp, vp, ctypes.c_double, vp, ctypes.c_double, vp, vp, i64,
                                                   vp, vp, sz, vp]
    lib.poem_select_practical_per_head.restype = st
    lib.poem_select_ranked_budget.argtypes = [sp, vp, vp, vp, vp, i64, vp, vp, sz, vp]
    lib.poem_select_ranked_budget.restype = st
    lib.poem_select_noalloc.argtypes = [sp, vp, vp, ctypes.c_float, vp, vp, i64, vp, vp]
    lib.poem_select_noalloc.restype = st
    lib.poem_pooled_workspace_size.argtypes = [sp, ctypes.POINTER(sz)]
    lib.poem_pooled_workspace_size.restype = st
    lib.poem_score_pooled.argtypes = [sp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.poem_score_pooled.restype = st
    dbl = ctypes.c_double
    lib.poem_select_practical.argtypes = [sp, vp, vp, dbl, dbl, dbl, vp, vp, i64, vp, vp, sz, vp]
    lib.poem_select_practical.restype = st
    lib.bsa_fwd.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.bsa_fwd.restype = st
    lib.bsa_fwd_grouped.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.bsa_fwd_grouped.restype = st
    lib.poem_check.argtypes = [vp, vp]
    lib.poem_check.restype = st
    lib.poem_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.poem_set_wait_limit_ns.restype = None
    lib.poem_status_string.argtypes = [st]
    lib.poem_status_string.restype = ctypes.c_char_p
    lib.poem_last_error.argtypes = []
    lib.poem_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def _raise(status: int, where: str):
    if status != POEM_OK:
        raise PoemError(status, where, _lib.poem_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_shape(q: torch.Tensor, k: torch.Tensor, block: int = 128, n_sample: int = 16, scale: float = 0.0,
               o: torch.Tensor | None = None) -> Shape:
    """Shape of a layer from q [Nq, Hq, d] and k/v [Nk, Hkv, d] (any strides with a
    contiguous head dimension); o defaults to q's strides.  Nk > Nq is a chunked
    prefill: the queries are the last Nq of the Nk tokens (q_offset = Nk - Nq)."""
    n, hq, d = q.shape
    nk, hkv = k.shape[0], k.shape[1]
    if q.stride(2) != 1 or k.stride(2) != 1:
        raise ValueError("the head dimension must be contiguous")
    if nk < n:
        raise ValueError("k/v must hold at least as many tokens as q")
    o_st = (o.stride(0), o.stride(1)) if o is not None else (q.stride(0), q.stride(1))
    return Shape(n, hq, hkv, d, block, n_sample, float(scale), nk - n, q.stride(0), q.stride(1), k.stride(0),
                 k.stride(1), o_st[0], o_st[1])


def poem_workspace_size(shape: Shape):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _raise(_lib.poem_workspace_size(ctypes.byref(shape), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "poem_workspace_size")
    return a.value, b.value, c.value


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace buffer (the error word must start clear)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def n_score_entries(n_q_heads: int, n_tiles: int, q_tile0: int = 0) -> int:
    """Entries of the per-(head, query tile, visible block) arrays: row (h, i) holds
    q_tile0 + i + 1 entries at h*E + i*q_tile0 + i*(i+1)/2."""
    return n_q_heads * (n_tiles * q_tile0 + n_tiles * (n_tiles + 1) // 2)


def score_row_offset(n_tiles: int, q_tile0: int, h: int, i: int) -> int:
    """Offset of row (head h, query tile i) in the per-(head, tile, block) arrays."""
    return h * (n_tiles * q_tile0 + n_tiles * (n_tiles + 1) // 2) + i * q_tile0 + i * (i + 1) // 2


def _check_bf16(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError("q, k, v, o must be CUDA bfloat16 tensors")


def _dims(shape: Shape):
    """(rows, entries) of a shape: rows = n_q_heads * T, entries of the per-(head,
    tile, block) arrays."""
    if shape.block <= 0 or shape.n_tokens <= 0 or shape.n_q_heads <= 0:
        return 0, 0  # an invalid shape: the library rejects it
    T = shape.n_tokens // shape.block
    t0 = max(shape.q_offset, 0) // shape.block
    return shape.n_q_heads * T, n_score_entries(shape.n_q_heads, T, t0)


def _need(t, dtype, min_numel: int, name: str, optional: bool = False):
    """A device buffer handed to the library: CUDA, contiguous, the right dtype and
    large enough for what the call writes or reads."""
    if t is None:
        if optional:
            return
        raise TypeError(f"{name} is required")
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous CUDA {dtype} tensor (got {t.dtype}, cuda={t.is_cuda})")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements; this shape needs {min_numel}")


def _check_kv(k, v):
    """The ABI describes K and V with one shape and one stride pair."""
    if k.shape != v.shape or k.stride() != v.stride():
        raise ValueError(f"k and v must have the same shape and strides (k {tuple(k.shape)} {k.stride()}, "
                         f"v {tuple(v.shape)} {v.stride()})")


def poem_score(q, k, v, I_hat, m_hat, ws, shape: Shape | None = None, stream=None, **shape_kw):
    _check_bf16(q, k, v)
    _check_kv(k, v)
    shape = shape or make_shape(q, k, **shape_kw)
    rows, ne = _dims(shape)
    _need(I_hat, torch.float32, ne, "I_hat")
    _need(m_hat, torch.float32, ne, "m_hat")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_score(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(I_hat), _ptr(m_hat), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream)), "poem_score")


def poem_select(shape: Shape, I_hat, m_hat, tau: float, row_ptr, col_idx, ws, order=None, stream=None):
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(I_hat, torch.float32, ne, "I_hat")
    _need(m_hat, torch.float32, ne, "m_hat")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_select(ctypes.byref(shape), _ptr(I_hat), _ptr(m_hat), ctypes.c_float(tau), _ptr(row_ptr),
                            _ptr(col_idx), col_idx.numel(), _ptr(order), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(stream)), "poem_select")


def poem_select_per_head(shape: Shape, I_hat, m_hat, tau_per_head, row_ptr, col_idx, ws, order=None, stream=None):
    """poem_select with a device tensor of one tau per query head (float32, [n_q_heads])."""
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(I_hat, torch.float32, ne, "I_hat")
    _need(m_hat, torch.float32, ne, "m_hat")
    _need(tau_per_head, torch.float32, shape.n_q_heads, "tau_per_head")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_select_per_head(ctypes.byref(shape), _ptr(I_hat), _ptr(m_hat), _ptr(tau_per_head),
                                     _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(order), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "poem_select_per_head")


def poem_select_practical_per_head(shape: Shape, m_pool, d_pool, w: float, gamma_per_head, rho: float, row_ptr,
                                   col_idx, ws, order=None, stream=None):
    """poem_select_practical with a device tensor of one gamma per query head."""
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(m_pool, torch.float32, ne, "m_pool")
    _need(d_pool, torch.float32, ne, "d_pool")
    _need(gamma_per_head, torch.float32, shape.n_q_heads, "gamma_per_head")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_select_practical_per_head(ctypes.byref(shape), _ptr(m_pool), _ptr(d_pool), ctypes.c_double(w),
                                               _ptr(gamma_per_head), ctypes.c_double(rho), _ptr(row_ptr),
                                               _ptr(col_idx), col_idx.numel(), _ptr(order), _ptr(ws),
                                               ws.numel() * ws.element_size(), _stream(stream)),
           "poem_select_practical_per_head")


def poem_select_mass_only(shape: Shape, m_hat, ref_row_ptr, row_ptr, col_idx, ws, order=None, stream=None):
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(m_hat, torch.float32, ne, "m_hat")
    _need(ref_row_ptr, torch.int32, rows + 1, "ref_row_ptr")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_select_mass_only(ctypes.byref(shape), _ptr(m_hat), _ptr(ref_row_ptr), _ptr(row_ptr),
                                      _ptr(col_idx), col_idx.numel(), _ptr(order), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)), "poem_select_mass_only")


def poem_select_ranked_budget(shape: Shape, score, ref_row_ptr, row_ptr, col_idx, ws, order=None, stream=None):
    """Mandatory blocks + the top candidates by `score` at the per-row budget of ref_row_ptr."""
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(score, torch.float32, ne, "score")
    _need(ref_row_ptr, torch.int32, rows + 1, "ref_row_ptr")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_select_ranked_budget(ctypes.byref(shape), _ptr(score), _ptr(ref_row_ptr), _ptr(row_ptr),
                                          _ptr(col_idx), col_idx.numel(), _ptr(order), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)),
           "poem_select_ranked_budget")


def poem_select_noalloc(shape: Shape, I_hat, m_hat, tau: float, row_ptr, col_idx, order=None, stream=None):
    """poem_select without a workspace, for callers that cannot allocate device
    memory: the scratch is a fixed 8 MiB array inside the library (shared by all
    calls -- do not overlap calls on the GPU).  Check row_ptr[-1] against
    col_idx.numel() afterwards; there is no error word to poll."""
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(I_hat, torch.float32, ne, "I_hat")
    _need(m_hat, torch.float32, ne, "m_hat")
    _raise(_lib.poem_select_noalloc(ctypes.byref(shape), _ptr(I_hat), _ptr(m_hat), ctypes.c_float(tau),
                                    _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(order), _stream(stream)),
           "poem_select_noalloc")


def poem_pooled_workspace_size(shape: Shape) -> int:
    a = ctypes.c_size_t()
    _raise(_lib.poem_pooled_workspace_size(ctypes.byref(shape), ctypes.byref(a)), "poem_pooled_workspace_size")
    return a.value


def poem_score_pooled(q, k, v, m_pool, d_pool, ws, shape: Shape | None = None, stream=None, **shape_kw):
    """Pooled estimates m~ and d~ (packed lower-triangular fp32) for the practical selector."""
    _check_bf16(q, k, v)
    _check_kv(k, v)
    shape = shape or make_shape(q, k, **shape_kw)
    rows, ne = _dims(shape)
    _need(m_pool, torch.float32, ne, "m_pool")
    _need(d_pool, torch.float32, ne, "d_pool")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_score_pooled(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(m_pool), _ptr(d_pool),
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "poem_score_pooled")


def poem_select_practical(shape: Shape, m_pool, d_pool, w: float, gamma: float, rho: float, row_ptr, col_idx, ws,
                          order=None, stream=None):
    """Two-stage practical selection (mass shortlist, log m~ + w log d~ rerank, pooled-mass threshold gamma)."""
    rows, ne = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")
    _need(order, torch.int32, rows, "order", optional=True)
    _need(m_pool, torch.float32, ne, "m_pool")
    _need(d_pool, torch.float32, ne, "d_pool")
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.poem_select_practical(ctypes.byref(shape), _ptr(m_pool), _ptr(d_pool), ctypes.c_double(w),
                                      ctypes.c_double(gamma), ctypes.c_double(rho), _ptr(row_ptr), _ptr(col_idx),
                                      col_idx.numel(), _ptr(order), _ptr(ws), ws.numel() * ws.element_size(),
                                      _stream(stream)), "poem_select_practical")


def bsa_fwd(q, k, v, row_ptr, col_idx, o, ws, lse=None, order=None, shape: Shape | None = None, stream=None,
            **shape_kw):
    _check_bf16(q, k, v, o)
    _check_kv(k, v)
    if o.shape != q.shape:
        raise ValueError("o must have q's shape")
    shape = shape or make_shape(q, k, o=o, **shape_kw)
    rows, _ = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")  # must hold row_ptr[-1] entries (not checked: on the device)
    _need(order, torch.int32, rows, "order", optional=True)
    _need(lse, torch.float32, shape.n_q_heads * shape.n_tokens, "lse", optional=True)
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.bsa_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(col_idx), _ptr(order),
                        _ptr(o), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "bsa_fwd")


def bsa_fwd_grouped(q, k, v, row_ptr, col_idx, o, ws, lse=None, shape: Shape | None = None, stream=None,
                    **shape_kw):
    """bsa_fwd's outputs, with two query heads of a KV group sharing K/V tiles."""
    _check_bf16(q, k, v, o)
    _check_kv(k, v)
    if o.shape != q.shape:
        raise ValueError("o must have q's shape")
    shape = shape or make_shape(q, k, o=o, **shape_kw)
    rows, _ = _dims(shape)
    _need(row_ptr, torch.int32, rows + 1, "row_ptr")
    _need(col_idx, torch.int32, 0, "col_idx")  # must hold row_ptr[-1] entries (not checked: on the device)
    _need(lse, torch.float32, shape.n_q_heads * shape.n_tokens, "lse", optional=True)
    _need(ws, torch.uint8, 0, "ws")
    _raise(_lib.bsa_fwd_grouped(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(col_idx),
                                _ptr(o), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "bsa_fwd_grouped")


def poem_check(ws, stream=None):
    """Synchronise and raise PoemError if a kernel recorded a device-side error."""
    _raise(_lib.poem_check(_stream(stream), _ptr(ws)), "poem_check")


def poem_check_status(ws, stream=None) -> int:
    return int(_lib.poem_check(_stream(stream), _ptr(ws)))


def poem_set_wait_limit_ns(ns: int):
    _lib.poem_set_wait_limit_ns(int(ns))


def poem_status_string(status: int) -> str:
    return _lib.poem_status_string(int(status)).decode()


def poem_last_error() -> str:
    return _lib.poem_last_error().decode(errors="replace")


@dataclass
class Layer:
    """Device buffers of one prefill layer (reused across calls)."""
    shape: Shape
    I_hat: torch.Tensor
    m_hat: torch.Tensor
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    order: torch.Tensor
    o: torch.Tensor
    lse: torch.Tensor | None
    ws_score: torch.Tensor
    ws_select: torch.Tensor
    ws_fwd: torch.Tensor
    # practical selector only: pooled estimates and the pooling workspace
    m_pool: torch.Tensor | None = None
    d_pool: torch.Tensor | None = None
    ws_pooled: torch.Tensor | None = None


def alloc_layer(q, k, block: int = 128, n_sample: int = 16, with_lse: bool = False, practical: bool = False) -> Layer:
    # O is allocated contiguous and the shape takes O's own strides (q may be a padded view)
    o = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    shape = make_shape(q, k, block=block, n_sample=n_sample, o=o)
    n, hq, d = q.shape
    T = n // block
    s_b, sel_b, f_b = poem_workspace_size(shape)
    dev = q.device
    ne = n_score_entries(hq, T, shape.q_offset // block)
    extra = {}
    if practical:
        extra = dict(m_pool=torch.empty(ne, dtype=torch.float32, device=dev),
                     d_pool=torch.empty(ne, dtype=torch.float32, device=dev),
                     ws_pooled=alloc_workspace(poem_pooled_workspace_size(shape), dev))
    return Layer(**extra,
        shape=shape,
        I_hat=torch.empty(ne, dtype=torch.float32, device=dev),
        m_hat=torch.empty(ne, dtype=torch.float32, device=dev),
        row_ptr=torch.empty(hq * T + 1, dtype=torch.int32, device=dev),
        col_idx=torch.empty(ne, dtype=torch.int32, device=dev),
        order=torch.empty(hq * T, dtype=torch.int32, device=dev),
        o=o,
        lse=torch.empty(hq, n, dtype=torch.float32, device=dev) if with_lse else None,
        ws_score=alloc_workspace(s_b, dev),
        ws_select=alloc_workspace(sel_b, dev),
        ws_fwd=alloc_workspace(f_b, dev),
    )


def prefill_layer(q, k, v, tau: float, layer: Layer | None = None, block: int = 128, stream=None) -> Layer:
    """Score, select and attend for one layer; returns the buffers (o in layer.o)."""
    layer = layer or alloc_layer(q, k, block=block)
    poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape, stream=stream)
    poem_select(layer.shape, layer.I_hat, layer.m_hat, tau, layer.row_ptr, layer.col_idx, layer.ws_select,
                order=layer.order, stream=stream)
    bsa_fwd(q, k, v, layer.row_ptr, layer.col_idx, layer.o, layer.ws_fwd, lse=layer.lse, order=layer.order,
            shape=layer.shape, stream=stream)
    return layer


def prefill_layer_practical(q, k, v, w: float, gamma: float, rho: float, layer: Layer | None = None,
                            block: int = 128, stream=None) -> Layer:
    """Pooled scoring, practical selection and attention for one layer (o in layer.o)."""
    layer = layer or alloc_layer(q, k, block=block, practical=True)
    poem_score_pooled(q, k, v, layer.m_pool, layer.d_pool, layer.ws_pooled, shape=layer.shape, stream=stream)
    poem_select_practical(layer.shape, layer.m_pool, layer.d_pool, w, gamma, rho, layer.row_ptr, layer.col_idx,
                          layer.ws_select, order=layer.order, stream=stream)
    bsa_fwd(q, k, v, layer.row_ptr, layer.col_idx, layer.o, layer.ws_fwd, lse=layer.lse, order=layer.order,
            shape=layer.shape, stream=stream)
    return layer
