"""fp64 CPU oracle for POEM-style output-relative block-sparse attention prefill.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it and shares no code with it; the product path fails loudly when
its own extension is missing instead of falling back to anything here.

The arithmetic lives in ``poem_oracle.c`` (plain C, fp64, OpenMP over
independent (head, tile) units).  This module only marshals numpy arrays.
Every function cites the passage of the method description it follows:

* "Attention deletion error" (reading note on POEM, Wu et al.), Section 4.1:
  block mass m_b, weighted block mean v_b, dense output o, renormalised sparse
  output o~, the deletion-error identity (Equation 3) and the per-block proxy
  I_b = m_b ||v_b - o|| with the triangle bound (Equation 4).
* What the note leaves open is fixed as the CUDA library fixes it: 16 strided sampled
  queries per tile, max-aggregation, mandatory blocks {0, i-1, i} and the
  stopping rule  S_m < 1 and S_I <= tau (1 - S_m)  over the discarded suffix.
* "Block-Filtered Long-Context Attention", Appendix "Block ordering": equal
  scores rank the smaller block id first; lists are traversed in ascending id.
* Practical POEM (the note's paragraph on Equation (6) and Appendix B):
  estimated (mean-pooled) block masses and deviations, a mass shortlist, a
  rerank by log mass + w log deviation, and a pooled-mass retention threshold.
  The estimators and parameters are not printed; the reading is documented
  next to the C functions.

Inputs are [n_tokens, n_heads, head_dim] arrays: float64, or uint16 arrays
holding bf16 bit patterns (widened exactly to fp64 inside the C code).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "poem_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile ``poem_oracle.c`` into ``liboracle.so`` next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


class _Shape(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block", ctypes.c_int),
        ("n_sample", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("in_kind", ctypes.c_int),
        ("q_offset", ctypes.c_int),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        sp = ctypes.POINTER(_Shape)
        vp = ctypes.c_void_p
        lib.oracle_dense_row.argtypes = [sp, vp, vp, vp, ctypes.c_int, ctypes.c_int, dp]
        lib.oracle_dense_row.restype = ctypes.c_double
        lib.oracle_block_stats.argtypes = [sp, vp, vp, vp, ctypes.c_int, ctypes.c_int, dp, dp, dp, dp]
        lib.oracle_block_stats.restype = None
        lib.oracle_score_units.argtypes = [sp, vp, vp, vp, ctypes.c_int, ip, ip, dp, dp]
        lib.oracle_score_units.restype = None
        lib.oracle_select_row.argtypes = [ctypes.c_int, dp, dp, ctypes.c_double, ip, ip]
        lib.oracle_select_row.restype = ctypes.c_int
        lib.oracle_select_mass_only_row.argtypes = [ctypes.c_int, dp, ctypes.c_int, ip]
        lib.oracle_select_mass_only_row.restype = ctypes.c_int
        lib.oracle_select_rows.argtypes = [ctypes.c_int, ctypes.c_int, ip, ip, dp, dp, ctypes.c_double, ip, ip, ip]
        lib.oracle_select_rows.restype = None
        lib.oracle_masked_row.argtypes = [sp, vp, vp, vp, ctypes.c_int, ctypes.c_int, ip, ctypes.c_int, dp]
        lib.oracle_masked_row.restype = ctypes.c_double
        lib.oracle_masked_units.argtypes = [sp, vp, vp, vp, ctypes.c_int, ip, ip, ip, ip, dp, dp]
        lib.oracle_masked_units.restype = None
        lib.oracle_dense_units.argtypes = [sp, vp, vp, vp, ctypes.c_int, ip, ip, dp, dp]
        lib.oracle_dense_units.restype = None
        lib.oracle_pooled_units.argtypes = [sp, vp, vp, vp, ctypes.c_int, ip, ip, dp, dp]
        lib.oracle_pooled_units.restype = None
        lib.oracle_select_practical_row.argtypes = [ctypes.c_int, dp, dp, ctypes.c_double, ctypes.c_double,
                                                    ctypes.c_double, ip, ip]
        lib.oracle_select_practical_row.restype = ctypes.c_int
        lib.oracle_select_practical_rows.argtypes = [ctypes.c_int, ctypes.c_int, ip, ip, dp, dp, ctypes.c_double,
                                                     ctypes.c_double, ctypes.c_double, ip, ip, ip]
        lib.oracle_select_practical_rows.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS or the affinity set)."""
    return int(_load().oracle_num_threads())


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


@dataclass
class Problem:
    """Q, K, V of one attention layer, as seen by the oracle.

    k, v: [n_tokens, n_kv_heads, head_dim]; q: [n_tokens - q_offset, n_q_heads,
    head_dim], the queries at positions q_offset .. n_tokens-1 (q_offset =
    len(k) - len(q), 0 for a whole prefill, a multiple of block otherwise: a
    chunked prefill).  Tiles and token positions are global; only tiles >=
    q_offset / block hold queries.  Either all float64 or all uint16 (bf16 bit
    patterns).  ``scale`` defaults to 1/sqrt(head_dim).
    """

    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    block: int
    n_sample: int = 16
    scale: float | None = None

    def __post_init__(self):
        kinds = {a.dtype for a in (self.q, self.k, self.v)}
        if kinds == {np.dtype(np.float64)}:
            self._kind = 0
        elif kinds == {np.dtype(np.uint16)}:
            self._kind = 1
        else:
            raise TypeError(f"q/k/v must all be float64 or all uint16 (bf16 bits), got {kinds}")
        self.q = np.ascontiguousarray(self.q)
        self.k = np.ascontiguousarray(self.k)
        self.v = np.ascontiguousarray(self.v)
        nq, hq, d = self.q.shape
        n, hkv, dk = self.k.shape
        if self.v.shape != self.k.shape or nq > n or dk != d:
            raise ValueError("shape mismatch between q, k and v")
        if (n - nq) % self.block:
            raise ValueError("q_offset = len(k) - len(q) must be a multiple of block")
        if hq % hkv:
            raise ValueError("n_q_heads must be a multiple of n_kv_heads")
        if n % self.block:
            raise ValueError("n_tokens must be a multiple of block")
        if self.block % self.n_sample:
            raise ValueError("n_sample must divide block")
        if self.scale is None:
            self.scale = 1.0 / np.sqrt(d)
        self._shape = _Shape(n, hq, hkv, d, self.block, self.n_sample, float(self.scale), self._kind, n - nq)

    @property
    def n_tokens(self):
        return self.k.shape[0]

    @property
    def q_offset(self):
        return self.k.shape[0] - self.q.shape[0]

    @property
    def q_tile0(self):
        return self.q_offset // self.block

    @property
    def n_q_heads(self):
        return self.q.shape[1]

    @property
    def head_dim(self):
        return self.q.shape[2]

    @property
    def n_tiles(self):
        return self.n_tokens // self.block

    def _ptrs(self):
        return (ctypes.byref(self._shape), self.q.ctypes.data, self.k.ctypes.data, self.v.ctypes.data)

    # -- Section 4.1: dense output o and log-sum-exp of one query row ----------
    def dense_row(self, h: int, t: int):
        o = np.zeros(self.head_dim)
        lse = _load().oracle_dense_row(*self._ptrs(), h, t, _dp(o))
        return o, lse

    # -- Section 4.1 and Eq. 4: m_b, v_b, I_b of one query row ----------------
    def block_stats(self, h: int, t: int):
        nb = t // self.block + 1
        m = np.zeros(nb)
        vb = np.zeros((nb, self.head_dim))
        I = np.zeros(nb)
        o = np.zeros(self.head_dim)
        _load().oracle_block_stats(*self._ptrs(), h, t, _dp(m), _dp(vb), _dp(I), _dp(o))
        return m, vb, I, o

    # -- Aggregated scores over the sampled queries of (h, i) units -----------
    def score_units(self, units, Ihat=None, mhat=None):
        """Fill the packed lower-triangular Ihat/mhat arrays for the listed
        (h, i) units.  Returns (Ihat, mhat), each of length n_q_heads*T(T+1)/2."""
        T = self.n_tiles
        total = self.n_q_heads * T * (T + 1) // 2
        if Ihat is None:
            Ihat = np.zeros(total)
        if mhat is None:
            mhat = np.zeros(total)
        uh = np.ascontiguousarray([u[0] for u in units], dtype=np.int32)
        ui = np.ascontiguousarray([u[1] for u in units], dtype=np.int32)
        _load().oracle_score_units(*self._ptrs(), len(units), _ip(uh), _ip(ui), _dp(Ihat), _dp(mhat))
        return Ihat, mhat

    def score_all(self):
        units = [(h, i) for h in range(self.n_q_heads) for i in range(self.n_tiles)]
        return self.score_units(units)

    # -- Section 4.1: renormalised output over a kept block set ---------------
    def masked_row(self, h: int, t: int, blocks):
        b = np.ascontiguousarray(blocks, dtype=np.int32)
        o = np.zeros(self.head_dim)
        lse = _load().oracle_masked_row(*self._ptrs(), h, t, _ip(b), len(b), _dp(o))
        return o, lse

    def masked_units(self, units, row_ptr, col_idx):
        """All B rows of each listed (h, i) unit under the CSR block lists
        (row r = h*T + i).  Returns O [n_units, B, d] and lse [n_units, B]."""
        B, d = self.block, self.head_dim
        uh = np.ascontiguousarray([u[0] for u in units], dtype=np.int32)
        ui = np.ascontiguousarray([u[1] for u in units], dtype=np.int32)
        rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
        ci = np.ascontiguousarray(col_idx, dtype=np.int32)
        O = np.zeros((len(units), B, d))
        lse = np.zeros((len(units), B))
        _load().oracle_masked_units(*self._ptrs(), len(units), _ip(uh), _ip(ui), _ip(rp), _ip(ci), _dp(O), _dp(lse))
        return O, lse

    # -- practical scoring: pooled masses and deviations (reading of Eq. 6) ----
    def pooled_units(self, units, m_pool=None, d_pool=None):
        """Pooled block masses m~ and deviations d~ = ||v~_b - o~|| for the listed
        (h, i) units, packed lower-triangular like score_units."""
        T = self.n_tiles
        total = self.n_q_heads * T * (T + 1) // 2
        if m_pool is None:
            m_pool = np.zeros(total)
        if d_pool is None:
            d_pool = np.zeros(total)
        uh = np.ascontiguousarray([u[0] for u in units], dtype=np.int32)
        ui = np.ascontiguousarray([u[1] for u in units], dtype=np.int32)
        _load().oracle_pooled_units(*self._ptrs(), len(units), _ip(uh), _ip(ui), _dp(m_pool), _dp(d_pool))
        return m_pool, d_pool

    def pooled_all(self):
        return self.pooled_units([(h, i) for h in range(self.n_q_heads) for i in range(self.n_tiles)])

    def dense_units(self, units):
        B, d = self.block, self.head_dim
        uh = np.ascontiguousarray([u[0] for u in units], dtype=np.int32)
        ui = np.ascontiguousarray([u[1] for u in units], dtype=np.int32)
        O = np.zeros((len(units), B, d))
        lse = np.zeros((len(units), B))
        _load().oracle_dense_units(*self._ptrs(), len(units), _ip(uh), _ip(ui), _dp(O), _dp(lse))
        return O, lse


def tri_offset(n_tiles: int, h: int, i: int) -> int:
    """Offset of row (h, i) in the packed lower-triangular score layout."""
    return h * (n_tiles * (n_tiles + 1) // 2) + i * (i + 1) // 2


def select_row(i: int, Ihat_row, mhat_row, tau: float):
    """Threshold selection of query tile i (Eq. 4 stopping rule).

    Returns (kept block ids ascending, k = number of candidates kept)."""
    Ih = np.ascontiguousarray(Ihat_row, dtype=np.float64)
    mh = np.ascontiguousarray(mhat_row, dtype=np.float64)
    assert Ih.shape[0] >= i + 1 and mh.shape[0] >= i + 1
    out = np.zeros(i + 1, dtype=np.int32)
    kc = np.zeros(1, dtype=np.int32)
    n = _load().oracle_select_row(i, _dp(Ih), _dp(mh), float(tau), _ip(out), _ip(kc))
    return out[:n].copy(), int(kc[0])


def select_mass_only_row(i: int, mhat_row, k_free: int):
    """Mass-only baseline: mandatory blocks plus the k_free largest-mass candidates."""
    mh = np.ascontiguousarray(mhat_row, dtype=np.float64)
    out = np.zeros(i + 1, dtype=np.int32)
    n = _load().oracle_select_mass_only_row(i, _dp(mh), int(k_free), _ip(out))
    return out[:n].copy()


def select_practical_row(i: int, m_pool_row, d_pool_row, w: float, gamma: float, rho: float):
    """Practical selection of tile i: stage-1 mass shortlist (fraction rho), stage-2
    rerank by log m~ + w log d~, keep until the pooled mass reaches gamma.
    Returns (kept ids ascending, prefix length kept from the reranked shortlist)."""
    m = np.ascontiguousarray(m_pool_row, dtype=np.float64)
    dv = np.ascontiguousarray(d_pool_row, dtype=np.float64)
    out = np.zeros(i + 1, dtype=np.int32)
    kc = np.zeros(1, dtype=np.int32)
    n = _load().oracle_select_practical_row(i, _dp(m), _dp(dv), float(w), float(gamma), float(rho), _ip(out),
                                            _ip(kc))
    return out[:n].copy(), int(kc[0])


def select_practical_all(n_q_heads: int, n_tiles: int, m_pool, d_pool, w: float, gamma: float, rho: float):
    rows = [(h, i) for h in range(n_q_heads) for i in range(n_tiles)]
    rh = np.ascontiguousarray([r[0] for r in rows], dtype=np.int32)
    ri = np.ascontiguousarray([r[1] for r in rows], dtype=np.int32)
    m = np.ascontiguousarray(m_pool, dtype=np.float64)
    dv = np.ascontiguousarray(d_pool, dtype=np.float64)
    lists = np.zeros((len(rows), n_tiles), dtype=np.int32)
    counts = np.zeros(len(rows), dtype=np.int32)
    kcut = np.zeros(len(rows), dtype=np.int32)
    _load().oracle_select_practical_rows(n_tiles, len(rows), _ip(rh), _ip(ri), _dp(m), _dp(dv), float(w),
                                         float(gamma), float(rho), _ip(lists), _ip(counts), _ip(kcut))
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate([lists[r, : counts[r]] for r in range(len(rows))])
    return row_ptr, col_idx.astype(np.int32), kcut


def select_all(n_q_heads: int, n_tiles: int, Ihat, mhat, tau: float, rows=None):
    """Selection for every (h, i) row (or the listed rows).  Returns a CSR
    (row_ptr, col_idx) over the listed rows in order, and the k of each row."""
    if rows is None:
        rows = [(h, i) for h in range(n_q_heads) for i in range(n_tiles)]
    rh = np.ascontiguousarray([r[0] for r in rows], dtype=np.int32)
    ri = np.ascontiguousarray([r[1] for r in rows], dtype=np.int32)
    Ih = np.ascontiguousarray(Ihat, dtype=np.float64)
    mh = np.ascontiguousarray(mhat, dtype=np.float64)
    lists = np.zeros((len(rows), n_tiles), dtype=np.int32)
    counts = np.zeros(len(rows), dtype=np.int32)
    kcut = np.zeros(len(rows), dtype=np.int32)
    _load().oracle_select_rows(n_tiles, len(rows), _ip(rh), _ip(ri), _dp(Ih), _dp(mh), float(tau),
                               _ip(lists), _ip(counts), _ip(kcut))
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate([lists[r, : counts[r]] for r in range(len(rows))]) if rows else np.zeros(0, np.int32)
    return row_ptr, col_idx.astype(np.int32), kcut
