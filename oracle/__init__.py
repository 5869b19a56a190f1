"""ctypes front end of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
CPU-baseline leg and reference arm use it; the CUDA library never imports it,
and it imports nothing from the CUDA side.  Inputs are widened exactly from bf16 to float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

TAG_FULL, TAG_CAUSAL, TAG_MASKED = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.oracle_max_threads.restype = ctypes.c_int
        L.oracle_tile_list.restype = i64
        L.oracle_tile_list.argtypes = [P, i32, i64, i32, i32, i32, ctypes.c_int, P, i64]
        L.oracle_tile_list_bounds.restype = i64
        L.oracle_tile_list_bounds.argtypes = [P, i32, i64, P, i32, i32, i32, ctypes.c_int, P, i64]
        L.oracle_balanced_bounds.restype = ctypes.c_int
        L.oracle_balanced_bounds.argtypes = [P, i32, i64, i32, i32, P]
        L.oracle_attn_fwd.restype = ctypes.c_int
        L.oracle_attn_fwd.argtypes = [P, P, P, i64, i32, i32, i32, P, i32, dbl, i64, i64, P, P, ctypes.c_int]
        L.oracle_merge.restype = ctypes.c_int
        L.oracle_merge.argtypes = [i32, P, P, i64, i32, i32, P, P]
        L.oracle_attn_fwd_rows.restype = ctypes.c_int
        L.oracle_attn_fwd_rows.argtypes = [P, P, P, i64, i32, i32, i32, P, i32, dbl, P, i64, P, i32, P, P,
                                           ctypes.c_int]
        L.oracle_attn_bwd.restype = ctypes.c_int
        L.oracle_attn_bwd.argtypes = [P, P, P, P, i64, i32, i32, i32, P, i32, dbl, P, P, P, ctypes.c_int]
        L.oracle_attn_bwd_sampled.restype = ctypes.c_int
        L.oracle_attn_bwd_sampled.argtypes = [P, P, P, P, i64, i32, i32, i32, P, i32, dbl, i32, P, i64, P, i64,
                                              P, P, P, ctypes.c_int]
        _lib = L
    return _lib


def _f64(t) -> np.ndarray:
    """Exact widening of a (bf16/fp32/fp64) torch tensor or array to contiguous float64."""
    if hasattr(t, "detach"):
        import torch
        t = t.detach().to("cpu")
        if t.dtype == torch.bfloat16:
            t = t.float()
        return np.ascontiguousarray(t.numpy().astype(np.float64))
    return np.ascontiguousarray(np.asarray(t, dtype=np.float64))


def _cu(cu) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(cu, dtype=np.int32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {rc})")
    return rc


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def tile_list(cu_seqlens, n: int, nchunks: int, bm: int = 128, bn: int = 128, exhaustive: bool = False,
              bounds=None) -> np.ndarray:
    """Canonical non-empty tile list, int32 [items, 5] = (q_tile, kv_tile, q_chunk, kv_chunk, tag).

    Chunks: nchunks equal parts, or the explicit token bounds ``bounds`` (nchunks + 1 entries)."""
    cu = _cu(cu_seqlens)
    if bounds is None:
        def call(out, cap):
            return lib().oracle_tile_list(_ptr(cu), len(cu) - 1, n, nchunks, bm, bn, int(exhaustive), out, cap)
    else:
        b = np.ascontiguousarray(np.asarray(bounds, dtype=np.int64))
        if len(b) != nchunks + 1:
            raise ValueError("bounds needs nchunks + 1 entries")

        def call(out, cap):
            return lib().oracle_tile_list_bounds(_ptr(cu), len(cu) - 1, n, _ptr(b), nchunks, bm, bn,
                                                 int(exhaustive), out, cap)
    cnt = _check(call(None, 0), "tile_list")
    out = np.zeros((max(cnt, 1), 5), dtype=np.int32)
    cnt2 = call(_ptr(out), cnt)
    assert cnt2 == cnt
    return out[:cnt]


def balanced_bounds(cu_seqlens, n: int, nchunks: int, block: int = 128) -> np.ndarray:
    """Balanced contiguous chunk bounds (int64, nchunks + 1 token offsets): see oracle_balanced_bounds."""
    cu = _cu(cu_seqlens)
    out = np.zeros(nchunks + 1, dtype=np.int64)
    _check(lib().oracle_balanced_bounds(_ptr(cu), len(cu) - 1, n, nchunks, block, _ptr(out)), "balanced_bounds")
    return out


def attn_fwd(q, k, v, cu_seqlens, scale: float, kv_range=None, nthreads: int = 0):
    """fp64 attention. Returns (O [N,hq,d], LSE [hq,N]); kv_range=(lo,hi) restricts the keys."""
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    n, hq, d = qd.shape
    hkv = kd.shape[1]
    cu = _cu(cu_seqlens)
    lo, hi = (0, n) if kv_range is None else kv_range
    o = np.zeros((n, hq, d))
    lse = np.zeros((hq, n))
    _check(lib().oracle_attn_fwd(_ptr(qd), _ptr(kd), _ptr(vd), n, hq, hkv, d, _ptr(cu), len(cu) - 1, scale, lo, hi,
                                 _ptr(o), _ptr(lse), nthreads), "attn_fwd")
    return o, lse


def merge(o_parts, lse_parts):
    """Exact LSE merge of partials: o_parts [P,N,hq,d], lse_parts [P,hq,N]."""
    op = np.ascontiguousarray(np.asarray(o_parts, dtype=np.float64))
    lp = np.ascontiguousarray(np.asarray(lse_parts, dtype=np.float64))
    nparts, n, hq, d = op.shape
    o = np.zeros((n, hq, d))
    lse = np.zeros((hq, n))
    _check(lib().oracle_merge(nparts, _ptr(op), _ptr(lp), n, hq, d, _ptr(o), _ptr(lse)), "merge")
    return o, lse


def attn_fwd_chunked(q, k, v, cu_seqlens, scale: float, nchunks: int, nthreads: int = 0, bounds=None):
    """Partials per kv chunk (each over all query rows), then the exact merge.  Chunks: nchunks equal
    parts, or the explicit token bounds ``bounds``.

    Returns (O, LSE, o_parts, lse_parts)."""
    n = q.shape[0]
    if bounds is None:
        if nchunks < 1 or (nchunks > 1 and n % nchunks):
            raise ValueError("N must split into equal chunks")
        c = n // nchunks if nchunks > 1 else n
        bounds = [b * c for b in range(nchunks)] + [n]
    bounds = [int(x) for x in bounds]
    if len(bounds) != nchunks + 1 or bounds[0] != 0 or bounds[-1] != n:
        raise ValueError("bounds must run from 0 to N in nchunks parts")
    parts = [attn_fwd(q, k, v, cu_seqlens, scale, (bounds[b], bounds[b + 1]), nthreads) for b in range(nchunks)]
    op = np.stack([p[0] for p in parts])
    lp = np.stack([p[1] for p in parts])
    o, lse = merge(op, lp)
    return o, lse, op, lp


def attn_fwd_rows(q, k, v, cu_seqlens, scale: float, rows, heads, nthreads: int = 0):
    """fp64 forward for sampled rows x heads: (O [nrows,nheads,d], LSE [nrows,nheads])."""
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    n, hq, d = qd.shape
    hkv = kd.shape[1]
    cu = _cu(cu_seqlens)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    h = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    o = np.zeros((len(r), len(h), d))
    lse = np.zeros((len(r), len(h)))
    _check(lib().oracle_attn_fwd_rows(_ptr(qd), _ptr(kd), _ptr(vd), n, hq, hkv, d, _ptr(cu), len(cu) - 1, scale,
                                      _ptr(r), len(r), _ptr(h), len(h), _ptr(o), _ptr(lse), nthreads),
           "attn_fwd_rows")
    return o, lse


def attn_bwd(q, k, v, do, cu_seqlens, scale: float, nthreads: int = 0):
    """fp64 gradients (dQ, dK, dV) of <dO, attention(Q,K,V)>."""
    qd, kd, vd, dod = _f64(q), _f64(k), _f64(v), _f64(do)
    n, hq, d = qd.shape
    hkv = kd.shape[1]
    cu = _cu(cu_seqlens)
    dq = np.zeros_like(qd)
    dk = np.zeros_like(kd)
    dv = np.zeros_like(vd)
    _check(lib().oracle_attn_bwd(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(dod), n, hq, hkv, d, _ptr(cu), len(cu) - 1,
                                 scale, _ptr(dq), _ptr(dk), _ptr(dv), nthreads), "attn_bwd")
    return dq, dk, dv


def attn_bwd_sampled(q, k, v, do, cu_seqlens, scale: float, g: int, q_rows, kv_rows, nthreads: int = 0,
                     arrays=None):
    """fp64 gradients on a sample for kv head g: dq [nq,G,d], dk [nk,d], dv [nk,d].

    ``arrays`` may pass pre-widened float64 (q, k, v, do) to avoid repeating the conversion."""
    qd, kd, vd, dod = arrays if arrays is not None else (_f64(q), _f64(k), _f64(v), _f64(do))
    n, hq, d = qd.shape
    hkv = kd.shape[1]
    G = hq // hkv
    cu = _cu(cu_seqlens)
    qr = np.ascontiguousarray(np.asarray(q_rows, dtype=np.int64))
    kr = np.ascontiguousarray(np.asarray(kv_rows, dtype=np.int64))
    dq = np.zeros((len(qr), G, d))
    dk = np.zeros((len(kr), d))
    dv = np.zeros((len(kr), d))
    _check(lib().oracle_attn_bwd_sampled(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(dod), n, hq, hkv, d, _ptr(cu),
                                         len(cu) - 1, scale, g, _ptr(qr), len(qr), _ptr(kr), len(kr), _ptr(dq),
                                         _ptr(dk), _ptr(dv), nthreads), "attn_bwd_sampled")
    return dq, dk, dv


def widen(*ts):
    """Exact float64 copies of tensors (for repeated sampled calls)."""
    return tuple(_f64(t) for t in ts)


def unmasked_pairs(cu_seqlens) -> int:
    """Number of (i, j) pairs with j <= i inside one document: sum L(L+1)/2."""
    lens = np.diff(np.asarray(cu_seqlens, dtype=np.int64))
    return int(np.sum(lens * (lens + 1) // 2))
