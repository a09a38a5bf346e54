"""CPU oracle for 3D Block Sparse Attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and its
Python binding) never calls it, and it never calls the product path.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP), which restates
the method from the pages:

* "LongCat-Video Technical Report" (paper summary page), section
  "Block Sparse Attention (BSA)" -- 3D block partitioning, pooled block
  similarity S_pool = Q_pool K_pool^T / sqrt(d), top-r key blocks per query
  block, softmax(QK^T/sqrt(d)) V with non-selected positions at -inf;
  section "Block Attention with KV-Cache for Efficient Multi-Task Inference" --
  condition tokens attend only to condition tokens.
* "LongCat-Video Technical Report #" (detail page), section
  "3D Block Sparse Attention" -- chunk shape [4,4,8], Top-K / CDF modes.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against hand-derived fixtures (``tests/golden/``), library routines (numpy
sorting, reshaping and matmul), brute force on tiny inputs, closed forms and
invariants. Beyond those pins, full-size outputs are "parity unpinned" except
through the invariants, which the tests also check on sampled rows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CHUNK = (4, 4, 8)
CN = 128

c_i64p = ctypes.POINTER(ctypes.c_int64)

# selection modes: top-k, CDF threshold, and their combination (chunks kept by both)
MODES = {"topk": 0, "cdf": 1, "topk_cdf": 2}


def build(force: bool = False) -> str:
    """Compile liboracle.so (gcc, -O2, OpenMP). Portable flags: no -march."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-D_GNU_SOURCE", "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_token_of.restype = i64
            lib.oracle_token_of.argtypes = [i32, i32, i32, i64, i32]
            lib.oracle_num_chunks.restype = i64
            lib.oracle_num_chunks.argtypes = [i32, i32, i32]
            lib.oracle_num_chunks_shape.restype = i64
            lib.oracle_num_chunks_shape.argtypes = [i32] * 6
            lib.oracle_token_of_shape.restype = i64
            lib.oracle_token_of_shape.argtypes = [i32] * 6 + [i64, i32]
            lib.oracle_pool_shape.restype = i32
            lib.oracle_pool_shape.argtypes = [vp] + [i32] * 9 + [vp]
            lib.oracle_select_shape.restype = i64
            lib.oracle_select_shape.argtypes = [vp] + [i32] * 10 + [dbl, dbl, i32, vp, vp, i64]
            lib.oracle_select_qk.restype = i64
            lib.oracle_select_qk.argtypes = [vp] + [i32] * 13 + [dbl, dbl, i32, vp, vp, i64]
            lib.oracle_attend_qk.restype = i32
            lib.oracle_attend_qk.argtypes = [vp, vp, vp] + [i32] * 11 + [dbl, vp, vp, vp, i64,
                                                                        vp, vp]
            lib.oracle_attend_shape.restype = i32
            lib.oracle_attend_shape.argtypes = [vp, vp, vp] + [i32] * 8 + [dbl, vp, vp, vp, i64,
                                                                           vp, vp]
            lib.oracle_attend_bwd_qk.restype = i32
            lib.oracle_attend_bwd_qk.argtypes = [vp] * 4 + [i32] * 11 + [dbl, vp, vp, vp, i64,
                                                                       vp, vp, vp]
            lib.oracle_attend_bwd_shape.restype = i32
            lib.oracle_attend_bwd_shape.argtypes = [vp] * 4 + [i32] * 8 + [dbl, vp, vp, vp, i64,
                                                                          vp, vp, vp]
            lib.oracle_attend_bwd_part_shape.restype = i32
            lib.oracle_attend_bwd_part_shape.argtypes = [vp] * 6 + [i32] * 8 + [dbl, vp, vp, vp,
                                                                               i64, vp, vp, vp]
            lib.oracle_rearrange.restype = i32
            lib.oracle_rearrange.argtypes = [vp, i32, i32, i32, i32, i32, vp]
            lib.oracle_pool.restype = i32
            lib.oracle_pool.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp]
            lib.oracle_scores.restype = i32
            lib.oracle_scores.argtypes = [vp, vp, i32, i32, i32, i32, dbl, i32, vp]
            lib.oracle_select.restype = i64
            lib.oracle_select.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, dbl, dbl, i32,
                                          vp, vp, i64]
            lib.oracle_attend.restype = i32
            lib.oracle_attend.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, dbl, vp, vp, vp,
                                          i64, vp, vp]
            lib.oracle_dense.restype = i32
            lib.oracle_dense.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, dbl, i32, vp, i64,
                                         vp, vp]
            lib.oracle_attend_bwd.restype = i32
            lib.oracle_attend_bwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, dbl, vp, vp,
                                              vp, i64, vp, vp, vp]
            lib.oracle_lse_merge.restype = i32
            lib.oracle_lse_merge.argtypes = [vp, vp, vp, vp, i64, i32]
            lib.oracle_num_threads.restype = i32
            lib.oracle_num_threads.argtypes = []
            _lib = lib
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "inputs are bf16 bit patterns (uint16)"
    return a


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"{what} failed ({rc})")
    return rc


def num_threads() -> int:
    return _load().oracle_num_threads()


def token_of(T, H, W, c, l) -> int:
    """Token index of local slot l of chunk c, -1 past the grid edge."""
    return _load().oracle_token_of(T, H, W, c, l)


def num_chunks(T, H, W, chunk=CHUNK) -> int:
    """Chunks of the grid: ceil(T/ct) * ceil(H/ch) * ceil(W/cw) (default (4,4,8))."""
    return _load().oracle_num_chunks_shape(T, H, W, *chunk)


def rearrange(x, T, H, W):
    """THW order [B, heads, N, d] -> chunk-major [B, heads, Nc, 128, d] (bf16 bits)."""
    x = _u16(x)
    B, Hh, N, d = x.shape
    out = np.empty((B, Hh, num_chunks(T, H, W), CN, d), dtype=np.uint16)
    _check(_load().oracle_rearrange(x.ctypes.data, B * Hh, T, H, W, d, out.ctypes.data),
           "oracle_rearrange")
    return out


def pool(x, T, H, W, fp32=False, chunk=CHUNK):
    """Chunk means [B, heads, Nc, d] (float64; float-valued when fp32) over chunks of
    shape `chunk` (default the (4,4,8) query chunk)."""
    x = _u16(x)
    B, Hh, N, d = x.shape
    out = np.empty((B, Hh, num_chunks(T, H, W, chunk), d), dtype=np.float64)
    _check(_load().oracle_pool_shape(x.ctypes.data, B * Hh, T, H, W, *chunk, d, int(fp32),
                                     out.ctypes.data), "oracle_pool")
    return out


def scores(qp, kp, scale, fp32=False):
    """Pooled scores [B, heads, Nq, Nk] = qp kp^T * scale."""
    qp = np.ascontiguousarray(qp, dtype=np.float64)
    kp = np.ascontiguousarray(kp, dtype=np.float64)
    B, Hh, Nq, d = qp.shape
    Nk = kp.shape[2]
    out = np.empty((B, Hh, Nq, Nk), dtype=np.float64)
    _check(_load().oracle_scores(qp.ctypes.data, kp.ctypes.data, B * Hh, Nq, Nk, d, float(scale),
                                 int(fp32), out.ctypes.data), "oracle_scores")
    return out


def select(S, T, H, W, mode="topk", topk=0, cdf_p=0.9, cap_frac=0.25, t_cond=0, fp32=False,
           kchunk=CHUNK, qchunk=CHUNK):
    """CSR (row_ptr int32 [rows+1], col_idx int32 [nnz]) of the selected key chunks
    (of shape `kchunk`) per query chunk (of shape `qchunk`); S is [B, heads, Nq, Nk]."""
    S = np.ascontiguousarray(S, dtype=np.float64)
    B, Hh, Nq, Nk = S.shape
    rows = B * Hh * Nq
    row_ptr = np.zeros(rows + 1, dtype=np.int32)
    col_cap = rows * Nk
    col_idx = np.empty(max(col_cap, 1), dtype=np.int32)
    nnz = _check(_load().oracle_select_qk(S.ctypes.data, B * Hh, T, H, W, *qchunk, *kchunk,
                                          int(t_cond), MODES[mode], int(topk), float(cdf_p),
                                          float(cap_frac), int(fp32), row_ptr.ctypes.data,
                                          col_idx.ctypes.data, col_cap), "oracle_select")
    return row_ptr, col_idx[:nnz].copy()


def plan(q, k, T, H, W, scale, mode="topk", topk=0, cdf_p=0.9, cap_frac=0.25, t_cond=0,
         fp32=False, kchunk=CHUNK, qchunk=CHUNK):
    """pool -> scores -> select; returns (row_ptr, col_idx, S)."""
    S = scores(pool(q, T, H, W, fp32, qchunk), pool(k, T, H, W, fp32, kchunk), scale, fp32)
    rp, ci = select(S, T, H, W, mode, topk, cdf_p, cap_frac, t_cond, fp32, kchunk, qchunk)
    return rp, ci, S


def attend(q, k, v, T, H, W, scale, row_ptr, col_idx, rows, want_lse=True, kchunk=CHUNK,
           qchunk=CHUNK):
    """Sparse attention for the listed CSR rows: out [n, slots, d] f64, lse [n, slots],
    slots = the query chunk's token count (128 for (4,4,8))."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hh, N, d = q.shape
    qn = qchunk[0] * qchunk[1] * qchunk[2]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if ci.size == 0:
        ci = np.zeros(1, dtype=np.int32)
    out = np.empty((rows.size, qn, d), dtype=np.float64)
    lse = np.empty((rows.size, qn), dtype=np.float64) if want_lse else None
    _check(_load().oracle_attend_qk(q.ctypes.data, k.ctypes.data, v.ctypes.data, B * Hh, T, H,
                                    W, *qchunk, *kchunk, d, float(scale), rp.ctypes.data,
                                    ci.ctypes.data, rows.ctypes.data, rows.size,
                                    out.ctypes.data,
                                    lse.ctypes.data if lse is not None else None),
           "oracle_attend")
    return out, lse


def _f64(a):
    """bf16 bit patterns (uint16) widened exactly, or float arrays as float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32), dtype=np.float64)
    return np.ascontiguousarray(a, dtype=np.float64)


def attend_bwd(q, k, v, dout, T, H, W, scale, row_ptr, col_idx, rows, kchunk=CHUNK,
               qchunk=CHUNK):
    """Gradients of ``attend`` for upstream gradient ``dout`` (same shape as q).

    Inputs: bf16 bit patterns (uint16) or float arrays [B, heads, N, d].
    Returns dq_rows [n, slots, d] for the listed CSR rows (slots = the query
    chunk's token count) and dk, dv [B, heads, N, d] holding the contributions
    of those rows (complete for every key chunk whose selecting rows are all
    listed). float64 throughout.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hh, N, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if ci.size == 0:
        ci = np.zeros(1, dtype=np.int32)
    qn = qchunk[0] * qchunk[1] * qchunk[2]
    dq = np.empty((rows.size, qn, d), dtype=np.float64)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    _check(_load().oracle_attend_bwd_qk(q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                        dout.ctypes.data, B * Hh, T, H, W, *qchunk, *kchunk, d,
                                        float(scale), rp.ctypes.data, ci.ctypes.data,
                                        rows.ctypes.data, rows.size, dq.ctypes.data,
                                        dk.ctypes.data, dv.ctypes.data), "oracle_attend_bwd")
    return dq, dk, dv


def attend_bwd_part(q, k, v, dout, out, lse, T, H, W, scale, row_ptr, col_idx, rows,
                    kchunk=CHUNK):
    """Gradient contributions of the keys of one partition (the chunks the CSR
    lists), given the full attention's output ``out`` and natural-log ``lse``
    ([B, heads, N]) for the queries. q, dout, out: the query grid; k, v: the
    key grid (same T, H, W). Returns dq_rows [n, 128, d] and dk, dv
    [B, heads, N, d] like ``attend_bwd``; the sums over a partition of the keys
    equal ``attend_bwd``. float64 throughout."""
    q, k, v, dout, out = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(out)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    B, Hh, N, d = q.shape
    assert lse.shape == (B, Hh, N) and out.shape == q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if ci.size == 0:
        ci = np.zeros(1, dtype=np.int32)
    dq = np.empty((rows.size, CN, d), dtype=np.float64)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    _check(_load().oracle_attend_bwd_part_shape(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, out.ctypes.data,
        lse.ctypes.data, B * Hh, T, H, W, *kchunk, d, float(scale), rp.ctypes.data,
        ci.ctypes.data, rows.ctypes.data, rows.size, dq.ctypes.data, dk.ctypes.data,
        dv.ctypes.data), "oracle_attend_bwd_part")
    return dq, dk, dv


def lse_merge(o1, l1, o2, l2):
    """Merge two partial attention results over disjoint key sets by their
    log-sum-exps: returns (o, l) float64, o [..., d], l [...]."""
    o = np.array(o1, dtype=np.float64, copy=True)
    l = np.array(l1, dtype=np.float64, copy=True)
    o2 = np.ascontiguousarray(o2, dtype=np.float64)
    l2 = np.ascontiguousarray(l2, dtype=np.float64)
    d = o.shape[-1]
    _check(_load().oracle_lse_merge(o.ctypes.data, l.ctypes.data, o2.ctypes.data, l2.ctypes.data,
                                    l.size, d), "oracle_lse_merge")
    return o, l


def dense(q, k, v, T, H, W, scale, qtok, t_cond=0, want_lse=True):
    """Dense (optionally block-causal) attention for global query ids bh*N + token."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hh, N, d = q.shape
    qtok = np.ascontiguousarray(qtok, dtype=np.int64)
    out = np.empty((qtok.size, d), dtype=np.float64)
    lse = np.empty(qtok.size, dtype=np.float64) if want_lse else None
    _check(_load().oracle_dense(q.ctypes.data, k.ctypes.data, v.ctypes.data, B * Hh, T, H, W, d,
                                float(scale), int(t_cond), qtok.ctypes.data, qtok.size,
                                out.ctypes.data, lse.ctypes.data if lse is not None else None),
           "oracle_dense")
    return out, lse


def chunk_tokens(T, H, W, c, chunk=CHUNK):
    """Token indices (THW order) of the local slots of chunk c of shape `chunk`
    (default (4,4,8): 128 slots), -1 for a slot past the grid edge."""
    n = chunk[0] * chunk[1] * chunk[2]
    return np.array([_load().oracle_token_of_shape(T, H, W, *chunk, c, l) for l in range(n)],
                    dtype=np.int64)
