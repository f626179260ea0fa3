"""attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot let a library call cudaMalloc (a framework that owns all
device memory through its own pool, a serving process with a memory budget
fixed at start-up, or code that cannot take the device synchronisation an
allocation may cause).  attn_decode_noalloc keeps its scratch in a fixed
device array inside the library instead.  These tests call it through the C
ABI and compare it with attn_decode and with the fp64 oracle, on two calls in
a row (the second with new inputs, so stale contents of the shared array would
show), check that its own error word reports a device-side error, and that an
oversized shape is refused before any GPU work.

This file is named so that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import exact_io_aware_sm_b200 as eio
import oracle
import synthetic

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3  # the tolerances of the other parity tests


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from exact_io_aware_sm_b200 import build
    build.build()
    L = eio.lib()
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, P]
    L.attn_decode_noalloc.restype = I
    L.attn_decode_noalloc_status.argtypes = [P]
    L.attn_decode_noalloc_status.restype = I
    return L


def _status(L):
    """The no-allocation decode's own error word (read and cleared)."""
    return L.attn_decode_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _host_inputs(seed, B, Hq, Hkv, Lmax, d):
    lens = synthetic.seqlens(seed, B, 1, Lmax)
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, Hq, d))
    kc = synthetic.kv_cache(seed, synthetic.TID_K, B, Lmax, Hkv, d, lens)
    vc = synthetic.kv_cache(seed, synthetic.TID_V, B, Lmax, Hkv, d, lens)
    return q, kc, vc, lens


def _inputs(seed, B, Hq, Hkv, Lmax, d):
    q, kc, vc, lens = _host_inputs(seed, B, Hq, Hkv, Lmax, d)

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return dev(q), dev(kc), dev(vc), torch.from_numpy(lens).cuda()


def _noalloc(L, q, kc, vc, sl, o, lse, B, Hq, Hkv, Lmax, d):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.attn_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), B, Hq, Hkv, Lmax, d, 1.0 / math.sqrt(d), stream)
    assert rc == 0, eio.last_error()


@pytest.mark.parametrize("shape", [(16, 32, 8, 4096, 128), (5, 8, 1, 1000, 64)])
def test_noalloc_matches_attn_decode_on_two_calls(lib, shape):
    B, Hq, Hkv, Lmax, d = shape
    for call, seed in enumerate((901, 902)):
        q, kc, vc, sl = _inputs(seed + d, B, Hq, Hkv, Lmax, d)
        ref_o, ref_l = eio.attn_decode(q, kc, vc, sl)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _noalloc(lib, q, kc, vc, sl, o, lse, B, Hq, Hkv, Lmax, d)
        torch.cuda.synchronize()
        if call == 1:  # the array already exists: nothing new on the device
            assert torch.cuda.mem_get_info()[0] == free_before
        err = (o.float() - ref_o.float()).abs()
        assert err.max().item() <= O_MAX and err.mean().item() <= O_MEAN
        assert (lse - ref_l).abs().max().item() <= LSE_TOL
        assert _status(lib) == 0, eio.last_error()  # its own error word: nothing latched
        # and against the fp64 oracle directly, every element
        hq, hkc, hvc, hlens = _host_inputs(seed + d, B, Hq, Hkv, Lmax, d)
        ro, rl = oracle.decode(hq, hkc, hvc, hlens, 1.0 / math.sqrt(d))
        oerr = np.abs(o.float().cpu().numpy().astype(np.float64) - ro)
        assert oerr.max() <= O_MAX and oerr.mean() <= O_MEAN
        assert np.abs(lse.cpu().numpy().astype(np.float64) - rl).max() <= LSE_TOL
    eio.sync_status()


def test_noalloc_reports_device_errors_through_its_own_status(lib):
    """A seqlens entry above Lmax is found on the device: that sequence gets
    O = 0 and LSE = -inf, and the error goes to the array's own error word,
    which attn_decode_noalloc_status returns once and then clears."""
    B, Hq, Hkv, Lmax, d = 3, 8, 2, 300, 128
    q, kc, vc, _ = _inputs(903, B, Hq, Hkv, Lmax, d)
    bad = torch.tensor([7, Lmax + 5, 300], dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    _noalloc(lib, q, kc, vc, bad, o, lse, B, Hq, Hkv, Lmax, d)
    assert _status(lib) == 9  # ATTN_ERR_DEVICE_ARG
    assert "seqlens" in eio.last_error()
    assert _status(lib) == 0  # cleared
    assert torch.all(o[1].float() == 0) and torch.isneginf(lse[1]).all()
    eio.sync_status()  # the library workspace's word is untouched


def test_noalloc_rejects_oversized_shape(lib):
    B, Hq, Hkv, Lmax, d = 512, 64, 8, 65536, 128  # needs far more than the fixed array
    q, kc, vc, sl = (torch.empty(16, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    o = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    rc = lib.attn_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(), o.data_ptr(),
                                 None, B, Hq, Hkv, Lmax, d, 0.1, None)
    assert rc == 8  # ATTN_ERR_WORKSPACE, returned before any launch
    assert "scratch" in eio.last_error()
