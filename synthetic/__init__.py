"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws numbers. It holds none of the attention arithmetic, so
both the fp64 oracle and the CUDA library can be fed from it without sharing
any of the method's code.

Generator (counter based, so any element can be regenerated on its own):

* ``splitmix64`` (Steele, Lea, Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014) applied to the counter
  ``seed * 0x9E3779B97F4A7C15 + tensor_id * 0xD1B54A32D192ED03 + pair_index``.
* The 64-bit draw is cut into two 32-bit halves, each mapped to a uniform in
  (0, 1) as ``(u32 + 0.5) / 2**32``; Box-Muller turns the pair into two
  N(0, 1) values (elements ``2 * pair_index`` and ``2 * pair_index + 1``).
* The fp64 normal is rounded to fp32 (round to nearest even), and, for bf16
  tensors, the fp32 value is rounded to bf16 (round to nearest even on the
  fp32 bit pattern).

Decode lengths are ``1024 + draw % 7169`` (uniform on [1024, 8192] up to a
modulo bias below 2e-15).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_TID_MUL = np.uint64(0xD1B54A32D192ED03)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)

# Tensor ids used by every caller, so that a (seed, tensor) pair names one stream.
TID_Q, TID_K, TID_V, TID_SEQLENS = 1, 2, 3, 4


def splitmix64(counter: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array (wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = counter + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _C1
        z = (z ^ (z >> np.uint64(27))) * _C2
        z = z ^ (z >> np.uint64(31))
    return z


def _base(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        return np.uint64(seed) * _GOLDEN + np.uint64(tensor_id) * _TID_MUL


def _normals_chunk(base: np.uint64, pair0: int, npairs: int) -> np.ndarray:
    with np.errstate(over="ignore"):
        ctr = base + np.arange(pair0, pair0 + npairs, dtype=np.uint64)
    z = splitmix64(ctr)
    u1 = ((z >> np.uint64(32)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
    u2 = ((z & np.uint64(0xFFFFFFFF)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
    r = np.sqrt(-2.0 * np.log(u1))
    t = (2.0 * np.pi) * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    nan = np.isnan(np.ascontiguousarray(x, dtype=np.float32))
    r = r.astype(np.uint16)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_POOL: ThreadPoolExecutor | None = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(16, len(os.sched_getaffinity(0)))))
    return _POOL


def normal(seed: int, tensor_id: int, n: int, dtype: str = "bf16", start: int = 0) -> np.ndarray:
    """Elements ``start .. start+n-1`` of stream (seed, tensor_id).

    Returns uint16 bf16 bit patterns for ``dtype="bf16"`` and float32 for
    ``dtype="f32"``.  ``start`` must be even.
    """
    if start % 2:
        raise ValueError("start must be even")
    base = _base(seed, tensor_id)
    npairs = (n + 1) // 2
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)
    chunk = 1 << 20
    jobs = []

    def work(p0: int, p1: int) -> None:
        vals = _normals_chunk(base, start // 2 + p0, p1 - p0).astype(np.float32)
        lo, hi = 2 * p0, min(n, 2 * p1)
        vals = vals[: hi - lo]
        out[lo:hi] = f32_to_bf16_bits(vals) if dtype == "bf16" else vals

    for p0 in range(0, npairs, chunk):
        jobs.append(_pool().submit(work, p0, min(npairs, p0 + chunk)))
    for j in jobs:
        j.result()
    return out


def tensor(seed: int, tensor_id: int, shape, dtype: str = "bf16") -> np.ndarray:
    n = int(np.prod(shape))
    return normal(seed, tensor_id, n, dtype).reshape(shape)


def seqlens(seed: int, batch: int, lo: int = 1024, hi: int = 8192) -> np.ndarray:
    """Per-sequence KV lengths, uniform integers in [lo, hi]."""
    z = splitmix64(_base(seed, TID_SEQLENS) + np.arange(batch, dtype=np.uint64))
    return (np.uint64(lo) + z % np.uint64(hi - lo + 1)).astype(np.int32)


def kv_cache(seed: int, tensor_id: int, B: int, Lmax: int, Hkv: int, d: int, lens: np.ndarray,
             fill_bits: int = 0) -> np.ndarray:
    """A [B, Lmax, Hkv, d] bf16 cache; rows below lens[b] hold stream values
    (row-major over [B, Lmax, Hkv, d] element index), rows at or above are ``fill_bits``."""
    out = np.full((B, Lmax, Hkv, d), np.uint16(fill_bits), dtype=np.uint16)
    row = Hkv * d
    for b in range(B):
        L = int(lens[b])
        start = (b * Lmax) * row
        out[b, :L] = normal(seed, tensor_id, L * row, "bf16", start=start).reshape(L, Hkv, d)
    return out
