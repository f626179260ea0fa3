"""Attention as a differentiable PyTorch op: attn_fwd forward, attn_bwd backward.

The forward keeps only what "FlashAttention: memory-saving exact attention"
(section 4) says a backward needs: the output O and the row statistics (the
LSE); the backward recomputes P from Q, K and the LSE inside attn_bwd.

    o = attention(q, k, v, mask_kind=MASK_CAUSAL)       # q [B,N,Hq,d] bf16 CUDA
    o.float().sum().backward()                          # q.grad, k.grad, v.grad

The LSE is returned with return_lse=True but is not differentiable (no
gradient flows through it).  `fwd` and `bwd` replace the two library calls,
with the signatures of default_fwd / default_bwd below; tests use that to
check this wrapper's bookkeeping against the oracle on the CPU.
"""
from __future__ import annotations

import math


def default_fwd(q, k, v, mask_kind, scale, block_map):
    from . import attn_fwd
    return attn_fwd(q, k, v, scale=scale, mask_kind=mask_kind, block_map=block_map)


def default_bwd(q, k, v, o, lse, dout, mask_kind, scale, block_map):
    from . import attn_bwd
    return attn_bwd(q, k, v, o, lse, dout, scale=scale, mask_kind=mask_kind, block_map=block_map)


def _function():
    import torch

    class _Attention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, mask_kind, scale, block_map, fwd, bwd):
            o, lse = fwd(q.contiguous(), k.contiguous(), v.contiguous(), mask_kind, scale, block_map)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.mask_kind, ctx.scale, ctx.block_map, ctx.bwd = mask_kind, scale, block_map, bwd
            ctx.mark_non_differentiable(lse)
            return o, lse

        @staticmethod
        def backward(ctx, dout, _dlse):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = ctx.bwd(q.contiguous(), k.contiguous(), v.contiguous(), o, lse, dout.contiguous(),
                                 ctx.mask_kind, ctx.scale, ctx.block_map)
            return dq, dk, dv, None, None, None, None, None

    return _Attention


_FN = None


def attention(q, k, v, mask_kind=0, scale=None, block_map=None, return_lse=False, fwd=None, bwd=None):
    """softmax(q k^T * scale + mask) v for q [B,Nq,Hq,d], k, v [B,Nkv,Hkv,d],
    differentiable in q, k and v.  mask_kind and block_map as for attn_fwd;
    scale defaults to 1/sqrt(d).  Returns o (and the LSE [B,Hq,Nq] if
    return_lse)."""
    global _FN
    if _FN is None:
        _FN = _function()
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    o, lse = _FN.apply(q, k, v, mask_kind, float(scale), block_map, fwd or default_fwd, bwd or default_bwd)
    return (o, lse) if return_lse else o
