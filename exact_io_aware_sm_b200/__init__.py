"""Python binding of libattn_b200.so (exact, IO-aware attention on B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the shared library.  PyTorch supplies device memory and streams.
There is no fallback: if the library is missing or a call fails, an
exception is raised.

Entry points mirror include/attn.h:

    attn_fwd(q, k, v, ...)            prefill, [B, N, H, d] tensors
    attn_decode(q, k_cache, v_cache, seqlens, ...)
    attn_decode_multi(q, k_cache, v_cache, seqlens, ...)
    attn_bwd(q, k, v, o, lse, dout, ...)
    key_stats(k), attn_fwd_bound(q, k, v, kbar, radius, ...)
    frame_block_map(n_frames, frame_len)
    classify(mask_kind, block_map, Nq, Nkv, tq, tk)
    plan(mask_kind, block_map, Nq, Nkv)
    sync_status(stream=None)

Above these: exact_io_aware_sm_b200.autograd.attention (the differentiable op,
attn_fwd forward and attn_bwd backward) and exact_io_aware_sm_b200.ulysses
(sequence-parallel forward, backward and differentiable op over
torch.distributed).

The C ABI takes plain pointers and cannot see buffer sizes, so every tensor
and block map is checked here (device, contiguity, dtype, shape) before a
pointer is passed: a mis-shaped output or map raises ValueError instead of
being written or read past its end.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

ATTN_OK = 0
STATUS_NAMES = {
    0: "ATTN_OK", 1: "ATTN_ERR_NULL", 2: "ATTN_ERR_SHAPE", 3: "ATTN_ERR_ALIGN",
    4: "ATTN_ERR_UNSUPPORTED", 5: "ATTN_ERR_MASK", 6: "ATTN_ERR_CUDA",
    7: "ATTN_ERR_DEVICE_TIMEOUT", 8: "ATTN_ERR_WORKSPACE", 9: "ATTN_ERR_DEVICE_ARG",
}
MASK_NONE, MASK_CAUSAL, MASK_BLOCK = 0, 1, 2
BF16, F32 = 0, 1

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, detail: str):
        self.code = code
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {detail}")


def lib() -> ctypes.CDLL:
    """Load libattn_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m exact_io_aware_sm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, I, P]
        L.attn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, P]
        L.attn_decode_multi.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P]
        L.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, P]
        L.attn_frame_block_map.argtypes = [I, I, P]
        L.attn_classify.argtypes = [I, P, I, I, I, I, P]
        L.attn_plan.argtypes = [I, P, I, I, P, I, P, I, P, P]
        L.attn_sync_status.argtypes = [P]
        L.attn_last_error_detail.argtypes = [ctypes.c_char_p, I]
        L.attn_shutdown.argtypes = []
        L.attn_debug_fault.argtypes = [I]
        L.attn_key_stats.argtypes = [P, P, P, I, I, I, I, P]
        L.attn_fwd_bound.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P, P, P]
        L.attn_version.restype = ctypes.c_char_p
        for fn in (L.attn_fwd, L.attn_decode, L.attn_decode_multi, L.attn_bwd, L.attn_frame_block_map,
                   L.attn_classify, L.attn_plan, L.attn_key_stats, L.attn_fwd_bound,
                   L.attn_sync_status, L.attn_last_error_detail, L.attn_shutdown, L.attn_debug_fault):
            fn.restype = I
        _lib = L
    return _lib


def last_error() -> str:
    buf = ctypes.create_string_buffer(512)
    lib().attn_last_error_detail(buf, 512)
    return buf.value.decode()


def _check(rc: int) -> None:
    if rc != ATTN_OK:
        raise AttnError(rc, last_error())


def _np_ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bm(block_map, Nq=None, Nkv=None):
    """The block map as a contiguous uint8 array of ceil(Nq/16) x ceil(Nkv/16)
    (the size the library reads), or None."""
    if block_map is None:
        return None
    bm = np.ascontiguousarray(block_map, dtype=np.uint8)
    if Nq is not None:
        want = ((Nq + 15) // 16, (Nkv + 15) // 16)
        if bm.shape != want:
            raise ValueError(f"block_map has shape {bm.shape}; Nq={Nq}, Nkv={Nkv} need {want}")
    return bm


def _need(t, name, shape, dtypes, device=None):
    """Check a tensor handed to the library: a contiguous CUDA tensor of one
    of the given dtypes whose shape matches `shape` (None entries match any
    size), on `device` if given, else (the call's first tensor) on the
    current CUDA device, where the library launches."""
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}; expected {' or '.join(str(d) for d in dtypes)}")
    if t.dim() != len(shape) or any(w is not None and w != n for w, n in zip(shape, t.shape)):
        want = tuple("*" if w is None else w for w in shape)
        raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {want}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; expected {device}")
    if device is None:  # the call's first tensor: the library runs on the current device
        import torch
        cur = torch.cuda.current_device()
        if t.device.index is not None and t.device.index != cur:
            raise ValueError(f"{name} is on {t.device} but the current CUDA device is {cur}; "
                             f"call inside torch.cuda.device({t.device.index})")


def attn_fwd(q, k, v, o=None, lse=None, scale=None, mask_kind=MASK_NONE, block_map=None,
             stream=None, want_lse=True):
    """Prefill attention.  q [B,Nq,Hq,d], k/v [B,Nkv,Hkv,d] CUDA tensors
    (bf16, or fp32 for the exact fp32 path).  Returns (o, lse) with o like q
    and lse fp32 [B,Hq,Nq] (None if want_lse is False and lse is None)."""
    import torch
    _need(q, "q", (None,) * 4, (torch.bfloat16, torch.float32))
    B, Nq, Hq, d = q.shape
    _need(k, "k", (B, None, None, d), (q.dtype,), q.device)
    Nkv, Hkv = k.shape[1], k.shape[2]
    _need(v, "v", k.shape, (q.dtype,), q.device)
    dt = BF16 if q.dtype == torch.bfloat16 else F32
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, (q.dtype,), q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", (B, Hq, Nq), (torch.float32,), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    bm = _bm(block_map, Nq, Nkv)
    _check(lib().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          None if lse is None else lse.data_ptr(), B, Hq, Hkv, Nq, Nkv, d,
                          float(scale), mask_kind, _np_ptr(bm), dt, _stream_ptr(stream)))
    return o, lse


def key_stats(k, kbar=None, radius=None, stream=None):
    """Key statistics for the bound-based softmax: kbar fp32 [B,Hkv,d] (mean
    key) and radius fp32 [B,Hkv] (largest centred key norm) of a bf16
    k [B,Nkv,Hkv,d] CUDA tensor."""
    import torch
    _need(k, "k", (None,) * 4, (torch.bfloat16,))
    B, Nkv, Hkv, d = k.shape
    if kbar is None:
        kbar = torch.empty((B, Hkv, d), dtype=torch.float32, device=k.device)
    if radius is None:
        radius = torch.empty((B, Hkv), dtype=torch.float32, device=k.device)
    _need(kbar, "kbar", (B, Hkv, d), (torch.float32,), k.device)
    _need(radius, "radius", (B, Hkv), (torch.float32,), k.device)
    _check(lib().attn_key_stats(k.data_ptr(), kbar.data_ptr(), radius.data_ptr(), B, Nkv, Hkv, d,
                                _stream_ptr(stream)))
    return kbar, radius


def attn_fwd_bound(q, k, v, kbar, radius, o=None, lse=None, scale=None, mask_kind=MASK_NONE, block_map=None,
                   n_fallback=None, stream=None):
    """attn_fwd (bf16) with the bound-based softmax; kbar, radius from
    key_stats(k).  n_fallback: optional int32 CUDA tensor of one element to
    which the number of rows that kept the running max is added.
    Returns (o, lse)."""
    import torch
    _need(q, "q", (None,) * 4, (torch.bfloat16,))
    B, Nq, Hq, d = q.shape
    _need(k, "k", (B, None, None, d), (torch.bfloat16,), q.device)
    Nkv, Hkv = k.shape[1], k.shape[2]
    _need(v, "v", k.shape, (torch.bfloat16,), q.device)
    _need(kbar, "kbar", (B, Hkv, d), (torch.float32,), q.device)
    _need(radius, "radius", (B, Hkv), (torch.float32,), q.device)
    if n_fallback is not None:
        _need(n_fallback, "n_fallback", (1,), (torch.int32,), q.device)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, (torch.bfloat16,), q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    _need(lse, "lse", (B, Hq, Nq), (torch.float32,), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    bm = _bm(block_map, Nq, Nkv)
    _check(lib().attn_fwd_bound(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                                Nq, Nkv, d, float(scale), mask_kind, _np_ptr(bm), kbar.data_ptr(), radius.data_ptr(),
                                None if n_fallback is None else n_fallback.data_ptr(), _stream_ptr(stream)))
    return o, lse


def _check_cache(k_cache, v_cache, seqlens, B, d, device):
    import torch
    _need(k_cache, "k_cache", (B, None, None, d),
          (torch.bfloat16,), device)
    _need(v_cache, "v_cache", k_cache.shape, (torch.bfloat16,), device)
    _need(seqlens, "seqlens", (B,), (torch.int32,), device)


def attn_decode(q, k_cache, v_cache, seqlens, o=None, lse=None, scale=None, stream=None,
                want_lse=True):
    """Single-token decode.  q [B,Hq,d] bf16; caches [B,Lmax,Hkv,d] bf16;
    seqlens int32 [B] on the device."""
    import torch
    _need(q, "q", (None,) * 3, (torch.bfloat16,))
    B, Hq, d = q.shape
    _check_cache(k_cache, v_cache, seqlens, B, d, q.device)
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, (torch.bfloat16,), q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", (B, Hq), (torch.float32,), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(lib().attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
                             o.data_ptr(), None if lse is None else lse.data_ptr(), B, Hq, Hkv, Lmax,
                             d, float(scale), _stream_ptr(stream)))
    return o, lse


def attn_decode_multi(q, k_cache, v_cache, seqlens, o=None, lse=None, scale=None, stream=None,
                      want_lse=True):
    """Decode of the Sq newest tokens per sequence.  q [B,Sq,Hq,d] bf16;
    caches [B,Lmax,Hkv,d] bf16; seqlens int32 [B] on the device (including
    the Sq new tokens).  Returns o [B,Sq,Hq,d] and lse [B,Hq,Sq]."""
    import torch
    _need(q, "q", (None,) * 4, (torch.bfloat16,))
    B, Sq, Hq, d = q.shape
    _check_cache(k_cache, v_cache, seqlens, B, d, q.device)
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, (torch.bfloat16,), q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", (B, Hq, Sq), (torch.float32,), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check(lib().attn_decode_multi(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
                                   o.data_ptr(), None if lse is None else lse.data_ptr(), B, Sq, Hq, Hkv,
                                   Lmax, d, float(scale), _stream_ptr(stream)))
    return o, lse


def attn_bwd(q, k, v, o, lse, dout, scale=None, mask_kind=MASK_NONE, block_map=None, stream=None):
    """Gradients of attn_fwd (bf16): q, o, dout [B,Nq,Hq,d]; k, v [B,Nkv,Hkv,d];
    lse [B,Hq,Nq] fp32 from the forward; the mask as for attn_fwd.
    Returns (dq, dk, dv) like q, k, v."""
    import torch
    _need(q, "q", (None,) * 4, (torch.bfloat16,))
    B, Nq, Hq, d = q.shape
    _need(k, "k", (B, None, None, d), (torch.bfloat16,), q.device)
    Nkv, Hkv = k.shape[1], k.shape[2]
    _need(v, "v", k.shape, (torch.bfloat16,), q.device)
    _need(o, "o", q.shape, (torch.bfloat16,), q.device)
    _need(dout, "dout", q.shape, (torch.bfloat16,), q.device)
    _need(lse, "lse", (B, Hq, Nq), (torch.float32,), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bm = _bm(block_map, Nq, Nkv)
    _check(lib().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nkv, d, float(scale),
                          mask_kind, _np_ptr(bm), _stream_ptr(stream)))
    return dq, dk, dv


def frame_block_map(n_frames: int, frame_len: int) -> np.ndarray:
    nb = (n_frames * frame_len + 15) // 16
    out = np.zeros((nb, nb), np.uint8)
    _check(lib().attn_frame_block_map(n_frames, frame_len, _np_ptr(out)))
    return out


def classify(mask_kind, block_map, Nq, Nkv, tq, tk) -> np.ndarray:
    out = np.zeros(((Nq + tq - 1) // tq, (Nkv + tk - 1) // tk), np.uint8)
    bm = _bm(block_map, Nq, Nkv)
    _check(lib().attn_classify(mask_kind, _np_ptr(bm), Nq, Nkv, tq, tk, _np_ptr(out)))
    return out


def plan(mask_kind, block_map, Nq, Nkv):
    """The tile schedule attn_fwd runs: (qtiles [n,4], kvtiles [m,3]) int32."""
    bm = _bm(block_map, Nq, Nkv)
    nq, nk = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().attn_plan(mask_kind, _np_ptr(bm), Nq, Nkv, None, 0, None, 0,
                           ctypes.byref(nq), ctypes.byref(nk)))
    qt = np.zeros((nq.value, 4), np.int32)
    kt = np.zeros((nk.value, 3), np.int32)
    _check(lib().attn_plan(mask_kind, _np_ptr(bm), Nq, Nkv, _np_ptr(qt), nq.value, _np_ptr(kt),
                           nk.value, ctypes.byref(nq), ctypes.byref(nk)))
    return qt, kt


def sync_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel latched a device error."""
    _check(lib().attn_sync_status(_stream_ptr(stream)))


def debug_fault(kind: int) -> None:
    """Test hook: kind 1 makes the next bf16 attn_fwd on this thread run one
    bounded wait out, so that its sync_status raises ATTN_ERR_DEVICE_TIMEOUT."""
    _check(lib().attn_debug_fault(kind))


def shutdown() -> None:
    lib().attn_shutdown()


def version() -> str:
    return lib().attn_version().decode()
