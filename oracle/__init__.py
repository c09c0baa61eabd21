"""fp64 CPU oracle for varlen grouped-query attention (packed THD, decode and
short-query regime, tail-aligned causal mask).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``varlen_gqa_split_b200``) and neither imports the other.

The arithmetic lives in ``oracle.c`` (plain fp64 loops; the definition it
writes out is stated at the top of that file).  This module compiles it with
gcc on first use and marshals numpy arrays into it.  Inputs are bf16 bit
patterns as ``numpy.uint16`` arrays; outputs are ``float64``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None

_c_int = ctypes.c_int
_c_i64 = ctypes.c_int64
_c_dbl = ctypes.c_double
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``_liboracle.so`` (gcc, OpenMP). Returns the path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # VGQA_ORACLE_LIB points the pins at a deliberately broken build of
        # oracle.c (the mutation check in tests/); unset in every other use.
        path = os.environ.get("VGQA_ORACLE_LIB") or build()
        lib = ctypes.CDLL(path)
        lib.oracle_attention.restype = _c_int
        lib.oracle_attention.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_dbl, _c_int,
                                         _p, _p, _p, _p, _p, _p, _p]
        lib.oracle_attention_rows.restype = _c_int
        lib.oracle_attention_rows.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_dbl,
                                              _c_int, _p, _p, _p, _p, _p, _c_i64, _p,
                                              _p, _p]
        lib.oracle_row_weights.restype = _c_i64
        lib.oracle_row_weights.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_dbl,
                                           _c_int, _p, _p, _p, _p, _p, _c_i64, _c_i64,
                                           _c_int, _p, _p, _p]
        lib.oracle_partial.restype = None
        lib.oracle_partial.argtypes = [_c_int, _c_dbl, _p, _p, _p, _c_i64, _c_i64,
                                       _c_i64, _p, _p, _p]
        lib.oracle_merge.restype = None
        lib.oracle_merge.argtypes = [_c_int, _c_int, _p, _p, _p, _p, _p]
        lib.oracle_num_threads.restype = _c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
        return lib


def _u16(a, name):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"{name}: expected bf16 bit patterns as uint16, got {a.dtype}")
    return a


def _i32(a, name):
    a = np.ascontiguousarray(a)
    if a.dtype != np.int32:
        raise TypeError(f"{name}: expected int32, got {a.dtype}")
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_scale(D: int) -> float:
    """Softmax scale 1/sqrt(D) used by every workload of the method."""
    return 1.0 / math.sqrt(D)


def num_threads() -> int:
    """OpenMP threads the oracle uses (the CPU-baseline core count)."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's later OpenMP regions (for a single-thread
    baseline).  Sets the OpenMP runtime the oracle library is linked with."""
    _load()
    ctypes.CDLL("libgomp.so.1").omp_set_num_threads(ctypes.c_int(int(n)))


def attention(q, k, v, cu_q, cu_k, *, B, Hq, Hkv, D, scale=None, causal=True,
              out=None, lse=None):
    """Whole-batch attention.

    q: [T_q, Hq, D] uint16 (bf16 bits); k, v: [T_kv, Hkv, D] uint16;
    cu_q, cu_k: int32 with at least B+1 entries (extra entries ignored).
    out / lse: optional float64 buffers [T_q, Hq, D] / [T_q, Hq] whose rows
    outside cu_q are left as given (default NaN).  Returns (out, lse).
    """
    lib = _load()
    q, k, v = _u16(q, "q"), _u16(k, "k"), _u16(v, "v")
    cu_q, cu_k = _i32(cu_q, "cu_q"), _i32(cu_k, "cu_k")
    if cu_q.size < B + 1 or cu_k.size < B + 1:
        raise ValueError("cu_seqlens need at least B+1 entries")
    T_q = q.shape[0]
    if out is None:
        out = np.full((T_q, Hq, D), np.nan, dtype=np.float64)
    if lse is None:
        lse = np.full((T_q, Hq), np.nan, dtype=np.float64)
    assert out.dtype == np.float64 and out.flags.c_contiguous
    assert lse.dtype == np.float64 and lse.flags.c_contiguous
    s = default_scale(D) if scale is None else float(scale)
    rc = lib.oracle_attention(B, Hq, Hkv, D, s, int(bool(causal)), _ptr(q), _ptr(k),
                              _ptr(v), _ptr(cu_q), _ptr(cu_k), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attention rejected its input (code {rc})")
    return out, lse


def attention_rows(q, k, v, cu_q, cu_k, rows, *, B, Hq, Hkv, D, scale=None,
                   causal=True):
    """Selected rows.  rows: int array [n, 3] of (b, qi, h).

    Returns (out [n, D] float64, lse [n] float64)."""
    lib = _load()
    q, k, v = _u16(q, "q"), _u16(k, "k"), _u16(v, "v")
    cu_q, cu_k = _i32(cu_q, "cu_q"), _i32(cu_k, "cu_k")
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    out = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    s = default_scale(D) if scale is None else float(scale)
    rc = lib.oracle_attention_rows(B, Hq, Hkv, D, s, int(bool(causal)), _ptr(q), _ptr(k),
                                   _ptr(v), _ptr(cu_q), _ptr(cu_k), n, _ptr(rows),
                                   _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attention_rows rejected its input (code {rc})")
    return out, lse


def row_weights(q, k, v, cu_q, cu_k, b, qi, h, *, B, Hq, Hkv, D, scale=None,
                causal=True):
    """Softmax weights p_j of one row, plus its out and lse: (p[n], out[D], lse)."""
    lib = _load()
    q, k, v = _u16(q, "q"), _u16(k, "k"), _u16(v, "v")
    cu_q, cu_k = _i32(cu_q, "cu_q"), _i32(cu_k, "cu_k")
    Lk = int(cu_k[b + 1] - cu_k[b])
    p = np.zeros((max(Lk, 1),), dtype=np.float64)
    out = np.empty((D,), dtype=np.float64)
    lse = np.empty((1,), dtype=np.float64)
    s = default_scale(D) if scale is None else float(scale)
    n = lib.oracle_row_weights(B, Hq, Hkv, D, s, int(bool(causal)), _ptr(q), _ptr(k),
                               _ptr(v), _ptr(cu_q), _ptr(cu_k), int(b), int(qi), int(h),
                               _ptr(p), _ptr(out), _ptr(lse))
    if n < 0:
        raise ValueError(f"oracle_row_weights rejected its input (code {n})")
    return p[:n].copy(), out, float(lse[0])


def partial(qrow, krows, vrows, j0, j1, *, scale):
    """(o, m, l) of one query row over keys [j0, j1).

    qrow: [D] uint16; krows, vrows: [N, D] uint16 (one KV head's rows)."""
    lib = _load()
    qrow, krows, vrows = _u16(qrow, "qrow"), _u16(krows, "krows"), _u16(vrows, "vrows")
    D = qrow.shape[-1]
    o = np.empty((D,), dtype=np.float64)
    m = np.empty((1,), dtype=np.float64)
    l = np.empty((1,), dtype=np.float64)
    lib.oracle_partial(D, float(scale), _ptr(qrow), _ptr(krows), _ptr(vrows), D,
                       int(j0), int(j1), _ptr(o), _ptr(m), _ptr(l))
    return o, float(m[0]), float(l[0])


def merge(o, m, l):
    """Log-sum-exp merge of S partial states: o [S, D], m [S], l [S] -> (out, lse)."""
    lib = _load()
    o = np.ascontiguousarray(o, dtype=np.float64)
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    S, D = o.shape
    out = np.empty((D,), dtype=np.float64)
    lse = np.empty((1,), dtype=np.float64)
    lib.oracle_merge(D, S, _ptr(o), _ptr(m), _ptr(l), _ptr(out), _ptr(lse))
    return out, float(lse[0])


def gather_pages(cache, block_table, page_size, cu_k, *, B):
    """Packed [sum Lk_b, Hkv, D] keys (or values) of a paged cache, in key
    order: key j of sequence b is slot j % page_size of page
    block_table[b, j // page_size] (the paged cache of the split kernel's
    interface, magik.net "Wiring Split-K Dispatch into a Custom CUDA Attention
    Kernel", section "The Message: A Read That Reveals the Architecture").
    Returns (packed, cu) with cu the prefix sums of the lengths cu_k gives."""
    cache = _u16(cache, "cache")
    bt = np.asarray(block_table)
    cu_k = _i32(cu_k, "cu_k")
    lens = np.diff(cu_k[: B + 1].astype(np.int64))
    parts = []
    for b in range(B):
        j = np.arange(int(lens[b]))
        pages = bt[b, j // page_size].astype(np.int64)
        if pages.size and (pages.min() < 0 or pages.max() >= cache.shape[0]):
            raise ValueError(f"block table row {b} names a page outside the cache")
        parts.append(cache[pages, j % page_size])
    packed = np.concatenate(parts) if parts else cache[:0, 0]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return np.ascontiguousarray(packed), cu


def attention_paged(q, k_cache, v_cache, block_table, page_size, cu_q, cu_k, *, B, Hq, Hkv, D, scale=None,
                    causal=True):
    """attention() with K and V read from a paged cache ([num_pages,
    page_size, Hkv, D] uint16 each); only the lengths are taken from cu_k."""
    k, cu = gather_pages(k_cache, block_table, page_size, cu_k, B=B)
    v, _ = gather_pages(v_cache, block_table, page_size, cu_k, B=B)
    return attention(q, k, v, cu_q, cu, B=B, Hq=Hq, Hkv=Hkv, D=D, scale=scale, causal=causal)


def merge_lse(outs, lses):
    """Combine results over disjoint key ranges given as normalised pairs:
    outs [n, ..., D] float64, lses [n, ...] (natural log, -inf for a part
    with no key).  Per row M = max_r lse_r, w_r = exp(lse_r - M),
    out = sum_r w_r out_r / sum_r w_r, lse = M + ln sum_r w_r; a row with no
    key anywhere gives out = 0, lse = -inf (the log-sum-exp merge of split
    partials, AstrAI commit log for csrc/kernels/gqa_decode_attn.cu, split-KV
    commit, on normalised parts)."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    M = lses.max(axis=0)
    finite = np.isfinite(M)
    Mref = np.where(finite, M, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - Mref[None]), 0.0)
    L = w.sum(axis=0)
    out = np.where(finite[..., None], (w[..., None] * np.nan_to_num(outs)).sum(axis=0) /
                   np.where(L > 0, L, 1.0)[..., None], 0.0)
    lse = np.where(finite, Mref + np.log(np.where(L > 0, L, 1.0)), -np.inf)
    return out, lse
