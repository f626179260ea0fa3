"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``exact_io_aware_sm_b200``) never imports it, and the two share no code.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over
independent rows).  This module builds it with gcc and marshals numpy arrays.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against facts the source pages fix (worked online-softmax examples,
invariants, a library routine on small shapes, brute force).  No function is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

MASK_NONE, MASK_CAUSAL, MASK_BLOCK = 0, 1, 2
BF16, F32, F64 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into oracle/liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.ora_attn_rows.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, P, P, I, P, P]
        L.ora_attn_fwd.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, P, P, P]
        L.ora_attn_bwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, D, I, P, P, P, P]
        L.ora_decode.argtypes = [P, P, P, I, P, I, I, I, I, I, D, P, P]
        L.ora_online_softmax.argtypes = [P, P, I, P, P, P, P, P]
        L.ora_merge_partials.argtypes = [P, P, I, I, P, P]
        L.ora_frame_allowed.argtypes = [I, I, I]
        L.ora_frame_block_map.argtypes = [I, I, P]
        L.ora_classify.argtypes = [I, P, I, I, I, I, P]
        L.ora_count_allowed.argtypes = [I, P, I, I]
        L.ora_count_allowed.restype = ctypes.c_longlong
        L.ora_check_schedule.argtypes = [I, P, I, I, P, I, P, I]
        L.ora_allowed.argtypes = [I, P, I, I, I, I]
        L.ora_key_stats.argtypes = [P, I, I, I, I, I, P, P]
        L.ora_attn_bwd_dq_rows.argtypes = [P, P, P, P, I, I, I, I, I, I, I, D, I, P, P, I, P]
        L.ora_attn_fwd_bound.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, P, P, P, D, P, P, P]
        L.ora_threads.argtypes = [I]
        L.ora_threads.restype = I
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16  # bf16 bit patterns
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.float64:
        return F64
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def _bm(block_map):
    return None if block_map is None else np.ascontiguousarray(block_map, dtype=np.uint8)


def attn_fwd(q, k, v, scale, mask_kind=MASK_NONE, block_map=None):
    """Full prefill attention.  q [B,Nq,Hq,d], k/v [B,Nkv,Hkv,d] (uint16 bf16
    bits, float32 or float64).  Returns (O [B,Nq,Hq,d] f64, LSE [B,Hq,Nq] f64)."""
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    B, Nq, Hq, d = q.shape
    Nkv, Hkv = k.shape[1], k.shape[2]
    dt = _dtype_code(q)
    assert _dtype_code(k) == dt and _dtype_code(v) == dt
    o = np.zeros((B, Nq, Hq, d), np.float64)
    lse = np.zeros((B, Hq, Nq), np.float64)
    bm = _bm(block_map)
    rc = lib().ora_attn_fwd(_ptr(q), _ptr(k), _ptr(v), dt, B, Hq, Hkv, Nq, Nkv, d, float(scale),
                            mask_kind, _ptr(bm), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("ora_attn_fwd rejected its arguments")
    return o, lse


def attn_bwd(q, k, v, dout, scale, mask_kind=MASK_NONE, block_map=None):
    """Gradients (dQ, dK, dV) in fp64 for the upstream gradient dout of O.
    q, dout [B,Nq,Hq,d]; k, v [B,Nkv,Hkv,d] (one dtype: bf16 bits, fp32, fp64)."""
    q, k, v, dout = (np.ascontiguousarray(x) for x in (q, k, v, dout))
    B, Nq, Hq, d = q.shape
    Nkv, Hkv = k.shape[1], k.shape[2]
    dt = _dtype_code(q)
    assert all(_dtype_code(x) == dt for x in (k, v, dout))
    dq = np.zeros((B, Nq, Hq, d), np.float64)
    dk = np.zeros((B, Nkv, Hkv, d), np.float64)
    dv = np.zeros((B, Nkv, Hkv, d), np.float64)
    bm = _bm(block_map)
    rc = lib().ora_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), dt, B, Hq, Hkv, Nq, Nkv, d, float(scale),
                            mask_kind, _ptr(bm), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError("ora_attn_bwd rejected its arguments")
    return dq, dk, dv


def attn_rows(q, k, v, scale, rows, mask_kind=MASK_NONE, block_map=None):
    """Selected rows: rows is an int array [n,3] of (b, hq, i).
    Returns (O [n,d] f64, LSE [n] f64)."""
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    B, Nq, Hq, d = q.shape
    Nkv, Hkv = k.shape[1], k.shape[2]
    dt = _dtype_code(q)
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    o = np.zeros((rows.shape[0], d), np.float64)
    lse = np.zeros(rows.shape[0], np.float64)
    bm = _bm(block_map)
    rc = lib().ora_attn_rows(_ptr(q), _ptr(k), _ptr(v), dt, B, Hq, Hkv, Nq, Nkv, d, float(scale),
                             mask_kind, _ptr(bm), _ptr(rows), rows.shape[0], _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("ora_attn_rows rejected its arguments")
    return o, lse


def decode(q, k_cache, v_cache, seqlens, scale):
    """q [B,Hq,d]; caches [B,Lmax,Hkv,d]; seqlens [B] (host).  Returns
    (O [B,Hq,d] f64, LSE [B,Hq] f64)."""
    q, kc, vc = (np.ascontiguousarray(x) for x in (q, k_cache, v_cache))
    B, Hq, d = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    rc = lib().ora_decode(_ptr(q), _ptr(kc), _ptr(vc), _dtype_code(q), _ptr(sl), B, Hq, Hkv, Lmax, d,
                          float(scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("ora_decode rejected its arguments")
    return o, lse


def online_softmax(x, bounds):
    """Block-wise softmax statistics: returns dict of arrays m_blk, l_blk,
    m_run, l_run, resc (one entry per block)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    bounds = np.ascontiguousarray(bounds, dtype=np.int32)
    nb = len(bounds) - 1
    outs = {n: np.zeros(nb, np.float64) for n in ("m_blk", "l_blk", "m_run", "l_run", "resc")}
    rc = lib().ora_online_softmax(_ptr(x), _ptr(bounds), nb, _ptr(outs["m_blk"]), _ptr(outs["l_blk"]),
                                  _ptr(outs["m_run"]), _ptr(outs["l_run"]), _ptr(outs["resc"]))
    if rc != 0:
        raise ValueError("bad bounds")
    return outs


def merge_partials(o_parts, lse_parts):
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, d = o_parts.shape
    o = np.zeros(d, np.float64)
    lse = np.zeros(1, np.float64)
    lib().ora_merge_partials(_ptr(o_parts), _ptr(lse_parts), n, d, _ptr(o), _ptr(lse))
    return o, float(lse[0])


def frame_block_map(n_frames, frame_len):
    N = n_frames * frame_len
    nb = (N + 15) // 16
    out = np.zeros((nb, nb), np.uint8)
    if lib().ora_frame_block_map(n_frames, frame_len, _ptr(out)) != 0:
        raise ValueError("frame blocks are not uniform at 16x16")
    return out


def frame_allowed(frame_len, i, j):
    return bool(lib().ora_frame_allowed(frame_len, i, j))


def allowed(mask_kind, block_map, Nq, Nkv, i, j):
    bm = _bm(block_map)
    return bool(lib().ora_allowed(mask_kind, _ptr(bm), Nq, Nkv, i, j))


def classify(mask_kind, block_map, Nq, Nkv, tq, tk):
    out = np.zeros(((Nq + tq - 1) // tq, (Nkv + tk - 1) // tk), np.uint8)
    bm = _bm(block_map)
    if lib().ora_classify(mask_kind, _ptr(bm), Nq, Nkv, tq, tk, _ptr(out)) != 0:
        raise ValueError("ora_classify rejected its arguments")
    return out


def count_allowed(mask_kind, block_map, Nq, Nkv):
    bm = _bm(block_map)
    return int(lib().ora_count_allowed(mask_kind, _ptr(bm), Nq, Nkv))


def threads(n: int = 0) -> int:
    """Set the oracle's OpenMP thread count for calls from this thread (if
    n > 0) and return the count it will use."""
    return int(lib().ora_threads(int(n)))


def check_schedule(mask_kind, block_map, Nq, Nkv, qtiles, kvtiles):
    qt = np.ascontiguousarray(qtiles, dtype=np.int32).reshape(-1, 4)
    kt = np.ascontiguousarray(kvtiles, dtype=np.int32).reshape(-1, 3)
    bm = _bm(block_map)
    return int(lib().ora_check_schedule(mask_kind, _ptr(bm), Nq, Nkv, _ptr(qt), qt.shape[0],
                                        _ptr(kt), kt.shape[0]))


def key_stats(k):
    """Per (b, KV head): mean key kbar [B,Hkv,d] and radius max_j ||k_j - kbar||
    [B,Hkv] (TPU guide, step 4: mean-centring), fp64."""
    k = np.ascontiguousarray(k)
    B, Nkv, Hkv, d = k.shape
    kbar = np.zeros((B, Hkv, d), np.float64)
    radius = np.zeros((B, Hkv), np.float64)
    if lib().ora_key_stats(_ptr(k), _dtype_code(k), B, Nkv, Hkv, d, _ptr(kbar), _ptr(radius)) != 0:
        raise ValueError("ora_key_stats rejected its arguments")
    return kbar, radius


BOUND_LIMIT2 = 100.0  # a row uses the bound when 2*M*log2(e) <= this (P >= 2^-100)


def attn_fwd_bound(q, k, v, scale, mask_kind=MASK_NONE, block_map=None, kbar=None, radius=None,
                   limit2=BOUND_LIMIT2):
    """Attention with the bound-based softmax (TPU guide, step 4) and a per-row
    fallback to the exact max.  Returns (o, lse, bound_row)."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    B, Nq, Hq, d = q.shape
    Nkv, Hkv = k.shape[1], k.shape[2]
    if kbar is None or radius is None:
        kbar, radius = key_stats(k)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    radius = np.ascontiguousarray(radius, dtype=np.float64)
    o = np.zeros((B, Nq, Hq, d), np.float64)
    lse = np.zeros((B, Hq, Nq), np.float64)
    flags = np.zeros((B, Hq, Nq), np.int32)
    bm = _bm(block_map)
    rc = lib().ora_attn_fwd_bound(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), B, Hq, Hkv, Nq, Nkv, d, float(scale),
                                  mask_kind, _ptr(bm), _ptr(kbar), _ptr(radius), float(limit2), _ptr(o), _ptr(lse),
                                  _ptr(flags))
    if rc != 0:
        raise ValueError("ora_attn_fwd_bound rejected its arguments")
    return o, lse, flags


def attn_bwd_dq_rows(q, k, v, dout, scale, rows, mask_kind=MASK_NONE, block_map=None):
    """dQ of selected query rows (b, hq, i), as attn_bwd defines it, at O(N d)
    per row: for gradient checks at sizes where the whole gradient is too
    slow.  Returns [n, d] fp64."""
    q, k, v, dout = (np.ascontiguousarray(x) for x in (q, k, v, dout))
    B, Nq, Hq, d = q.shape
    Nkv, Hkv = k.shape[1], k.shape[2]
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    out = np.zeros((rows.shape[0], d), np.float64)
    bm = _bm(block_map)
    rc = lib().ora_attn_bwd_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _dtype_code(q), B, Hq, Hkv, Nq, Nkv, d,
                                    float(scale), mask_kind, _ptr(bm), _ptr(rows), rows.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("ora_attn_bwd_dq_rows rejected its arguments")
    return out
