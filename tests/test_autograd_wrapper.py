"""The differentiable op of exact_io_aware_sm_b200.autograd, with the fp64
oracle injected in place of the two library calls (so it runs on the CPU):
what the forward saves, the order and shapes of the gradients, a
non-contiguous upstream gradient and non-contiguous inputs must all come out
as torch autograd of SDPA gives them."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_sm_b200.autograd import attention
from tests.test_oracle_pins import _allowed_matrix, _sdpa_grads, _sdpa_ref, rnd

calls = []


def _ofwd(q, k, v, mask_kind, scale, block_map):
    calls.append("fwd")
    o, lse = oracle.attn_fwd(q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), scale, mask_kind,
                             block_map)
    return torch.from_numpy(o), torch.from_numpy(lse)


def _obwd(q, k, v, o, lse, dout, mask_kind, scale, block_map):
    calls.append("bwd")
    qn, kn, vn = (t.detach().numpy() for t in (q, k, v))
    # the saved o and lse are the forward's for these very inputs
    ro, rl = oracle.attn_fwd(qn, kn, vn, scale, mask_kind, block_map)
    assert np.array_equal(o.detach().numpy(), ro) and np.array_equal(lse.detach().numpy(), rl)
    assert dout.is_contiguous()
    dq, dk, dv = oracle.attn_bwd(qn, kn, vn, dout.numpy(), scale, mask_kind, block_map)
    return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)


@pytest.mark.parametrize("case", [
    (1, 2, 2, 20, 20, 8, oracle.MASK_NONE),
    (2, 4, 2, 33, 41, 16, oracle.MASK_CAUSAL),
    (1, 6, 3, 40, 40, 8, oracle.MASK_BLOCK),
])
def test_gradients_equal_torch_autograd(case):
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = sum(case)
    qn, kn, vn = rnd((B, Nq, Hq, d), seed), rnd((B, Nkv, Hkv, d), seed + 1), rnd((B, Nkv, Hkv, d), seed + 2)
    bm = None
    if kind == oracle.MASK_BLOCK:
        bm = (np.random.default_rng(seed).random(((Nq + 15) // 16, (Nkv + 15) // 16)) < 0.6).astype(np.uint8)
        bm[:, 0] = 1
    scale = 1 / math.sqrt(d)
    q, k, v = (torch.from_numpy(x).requires_grad_(True) for x in (qn, kn, vn))
    calls.clear()
    o, lse = attention(q, k, v, mask_kind=kind, block_map=bm, return_lse=True, fwd=_ofwd, bwd=_obwd)
    assert not lse.requires_grad
    # an upstream gradient that reaches the op non-contiguous
    w = torch.from_numpy(rnd((B, Hq, Nq, d), seed + 3))
    (o.transpose(1, 2) * w).sum().backward()
    assert calls == ["fwd", "bwd"]
    dout = w.transpose(1, 2).contiguous().numpy()
    allowed = _allowed_matrix(kind, bm, Nq, Nkv)
    ro, rl = _sdpa_ref(qn, kn, vn, scale, allowed)
    np.testing.assert_allclose(o.detach().numpy(), ro, atol=1e-12)
    rq, rk, rv = _sdpa_grads(qn, kn, vn, dout, scale, allowed)
    for t, ref in ((q, rq), (k, rk), (v, rv)):
        assert t.grad.shape == t.shape
        np.testing.assert_allclose(t.grad.numpy(), ref, atol=1e-11, rtol=1e-10)


def test_non_contiguous_inputs_and_default_scale():
    """Inputs that are views (here transposed back from [B,H,N,d]) are made
    contiguous for the calls; gradients arrive in the inputs' own layout;
    the default scale is 1/sqrt(d)."""
    B, H, N, d = 1, 2, 24, 8
    base = [torch.from_numpy(rnd((B, H, N, d), s)).requires_grad_(True) for s in (1, 2, 3)]
    q, k, v = (t.transpose(1, 2) for t in base)  # [B, N, H, d] views
    assert not q.is_contiguous()
    o = attention(q, k, v, mask_kind=oracle.MASK_CAUSAL, fwd=_ofwd, bwd=_obwd)
    o.sum().backward()
    qn, kn, vn = (t.detach().contiguous().numpy() for t in (q, k, v))
    allowed = _allowed_matrix(oracle.MASK_CAUSAL, None, N, N)
    rq, rk, rv = _sdpa_grads(qn, kn, vn, np.ones((B, N, H, d)), 1 / math.sqrt(d), allowed)
    for t, ref in zip(base, (rq, rk, rv)):
        np.testing.assert_allclose(t.grad.transpose(1, 2).numpy(), ref, atol=1e-11, rtol=1e-10)
