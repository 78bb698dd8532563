"""CPU oracle for the DSA hot path (indexer -> top-k -> sparse GQA attention).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package; the product
path never does.  It shares no code with the CUDA path: the arithmetic lives
in ``dsa_oracle.c`` (plain loops, fp64, pthreads over query rows).

Definitions followed (Kwai Keye-VL-2.0 technical-report summary, section 1
and section 8; formula readings listed in the C file's header):

* ``index_topk``   - Lightning-Indexer scores and top-k by (score desc,
                     index asc), ascending output, -1 padding.
* ``index_scores`` - the dense causal indexer score rows.
* ``sparse_attn``  - softmax attention over the selected rows, per query head,
                     with the KV group g = h // (Hq // Hkv).
* ``dense_causal_attn`` - plain causal attention, written separately, used as
                     a pin (k >= t + 1 must reduce to it).
* ``decode``       - one new token per sequence over a packed cache.
* ``kl.indexer_kl`` - the indexer's dense warm-up loss (KL from the head-mean
                     full attention to the indexer's softmax) and its
                     gradients, in numpy float64 (``oracle/kl.py``).

Parity is pinned for every function here (see tests/test_oracle_pins.py);
the pages' own measured figures (cost ratios, dedup counts) depend on the
real model's data and stay unpinned.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from .build import build as _build, LIB_PATH

_lib = None


def lib() -> ctypes.CDLL:
    """The compiled oracle.  ORACLE_LIB_PATH, if set, names another build of
    dsa_oracle.c to load instead (the mutation test uses it to run the pins
    against a copy with a planted mistake)."""
    global _lib
    if _lib is None:
        path = os.environ.get("ORACLE_LIB_PATH")
        if not path:
            _build()
            path = LIB_PATH
        L = ctypes.CDLL(path)
        vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_e4m3.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3.restype = dbl
        L.oracle_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_bf16.restype = dbl
        L.oracle_index_topk.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, i64, vp, i32]
        L.oracle_index_topk.restype = i32
        L.oracle_index_scores.argtypes = [vp, vp, vp, i64, i32, i32, vp, i64, vp, i32]
        L.oracle_index_scores.restype = i32
        L.oracle_sparse_attn.argtypes = [vp, vp, vp, i64, vp, i32, i32, i32, i32, i32, dbl, vp,
                                         i64, vp, i32]
        L.oracle_sparse_attn.restype = i32
        L.oracle_attn_weights.argtypes = [vp, vp, i64, vp, i32, i32, i32, i32, dbl, i64, i32, vp]
        L.oracle_attn_weights.restype = i64
        L.oracle_dense_causal_attn.argtypes = [vp, vp, vp, i64, i32, i32, i32, dbl, vp, i64, vp,
                                               i32]
        L.oracle_dense_causal_attn.restype = i32
        L.oracle_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, dbl,
                                    vp, i64, vp, vp, i32]
        L.oracle_decode.restype = i32
        _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def _rows(rows, n) -> np.ndarray:
    if rows is None:
        return np.arange(n, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def _check(rc: int) -> None:
    if rc != 0:
        raise MemoryError("oracle: scratch allocation failed")


def e4m3_value(byte: int) -> float:
    return lib().oracle_e4m3(int(byte))


def bf16_value(bits: int) -> float:
    return lib().oracle_bf16(int(bits))


def index_topk(q_I, k_I, w, k: int, rows: Optional[Sequence[int]] = None,
               nthreads: int = 0) -> np.ndarray:
    """Selected keys per query row: int32 [len(rows)][k], ascending, -1 padded.

    q_I: uint8 e4m3 [L][H_I][d_I]; k_I: uint8 e4m3 [L][d_I]; w: float32 [L][H_I]."""
    q_I, k_I, w = _c(q_I, np.uint8), _c(k_I, np.uint8), _c(w, np.float32)
    L, H, d = q_I.shape
    r = _rows(rows, L)
    assert r.size == 0 or (r.min() >= 0 and r.max() < L)
    out = np.empty((r.size, k), np.int32)
    _check(lib().oracle_index_topk(q_I.ctypes.data, k_I.ctypes.data, w.ctypes.data, L, H, d, k,
                                   r.ctypes.data, r.size, out.ctypes.data, nthreads))
    return out


def index_scores(q_I, k_I, w, rows=None, nthreads: int = 0) -> np.ndarray:
    """Dense causal indexer scores: float64 [len(rows)][L], -inf above the diagonal."""
    q_I, k_I, w = _c(q_I, np.uint8), _c(k_I, np.uint8), _c(w, np.float32)
    L, H, d = q_I.shape
    r = _rows(rows, L)
    out = np.empty((r.size, L), np.float64)
    _check(lib().oracle_index_scores(q_I.ctypes.data, k_I.ctypes.data, w.ctypes.data, L, H, d,
                                     r.ctypes.data, r.size, out.ctypes.data, nthreads))
    return out


def sparse_attn(Q, K, V, idx, scale: float, rows=None, nthreads: int = 0,
                idx_by_row: bool = False) -> np.ndarray:
    """fp64 [len(rows)][Hq][d].  Q [*][Hq][d], K/V [n][Hkv][d] as bf16 bits
    (uint16); idx int32 [rows of Q][k], or [len(rows)][k] with idx_by_row."""
    Q, K, V = _c(Q, np.uint16), _c(K, np.uint16), _c(V, np.uint16)
    idx = _c(idx, np.int32)
    Lq, Hq, d = Q.shape
    n, Hkv, _ = K.shape
    k = idx.shape[1]
    r = _rows(rows, Lq)
    out = np.empty((r.size, Hq, d), np.float64)
    if idx_by_row:
        assert idx.shape[0] == r.size
    _check(lib().oracle_sparse_attn(Q.ctypes.data, K.ctypes.data, V.ctypes.data, n,
                                    idx.ctypes.data, int(idx_by_row), k, Hq, Hkv, d, float(scale),
                                    r.ctypes.data, r.size, out.ctypes.data, nthreads))
    return out


def attn_weights(Q, K, idx, scale: float, t: int, h: int) -> np.ndarray:
    """Softmax weight of each entry of idx[t] for query head h (0 for invalid)."""
    Q, K, idx = _c(Q, np.uint16), _c(K, np.uint16), _c(idx, np.int32)
    Lq, Hq, d = Q.shape
    n, Hkv, _ = K.shape
    k = idx.shape[1]
    p = np.empty(k, np.float64)
    lib().oracle_attn_weights(Q.ctypes.data, K.ctypes.data, n, idx.ctypes.data, k, Hq, Hkv, d,
                              float(scale), int(t), int(h), p.ctypes.data)
    return p


def dense_causal_attn(Q, K, V, scale: float, rows=None, nthreads: int = 0) -> np.ndarray:
    Q, K, V = _c(Q, np.uint16), _c(K, np.uint16), _c(V, np.uint16)
    L, Hq, d = Q.shape
    _, Hkv, _ = K.shape
    r = _rows(rows, L)
    out = np.empty((r.size, Hq, d), np.float64)
    _check(lib().oracle_dense_causal_attn(Q.ctypes.data, K.ctypes.data, V.ctypes.data, L, Hq,
                                          Hkv, d, float(scale), r.ctypes.data, r.size,
                                          out.ctypes.data, nthreads))
    return out


def decode(q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, k: int, scale: float,
           seqs=None, nthreads: int = 0):
    """(idx int32 [nseq][k] sequence-local ascending, O fp64 [nseq][Hq][d])."""
    q_I, w, Q = _c(q_I, np.uint8), _c(w, np.float32), _c(Q, np.uint16)
    kI_cache, K_cache, V_cache = (_c(kI_cache, np.uint8), _c(K_cache, np.uint16),
                                  _c(V_cache, np.uint16))
    cache_off = _c(cache_off, np.int64)
    B, H, dI = q_I.shape
    _, Hq, d = Q.shape
    Hkv = K_cache.shape[1]
    s = _rows(seqs, B)
    idx = np.empty((s.size, k), np.int32)
    out = np.empty((s.size, Hq, d), np.float64)
    _check(lib().oracle_decode(q_I.ctypes.data, w.ctypes.data, Q.ctypes.data,
                               kI_cache.ctypes.data, K_cache.ctypes.data, V_cache.ctypes.data,
                               cache_off.ctypes.data, H, dI, Hq, Hkv, d, k, float(scale),
                               s.ctypes.data, s.size, idx.ctypes.data, out.ctypes.data, nthreads))
    return idx, out
