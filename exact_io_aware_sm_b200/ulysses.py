"""Ulysses sequence parallelism around the attention call.

"TPU attention optimisation guide: collective overlap and mask removal,
verified by trace", step 2: with the sequence sharded over P ranks, an
all-to-all swaps sequence shards for head shards (every rank then holds the
whole sequence for H/P of the heads), attention runs unchanged on those heads,
and a second all-to-all swaps back.  Heads are split into groups, each with
its own pair of all-to-alls, so that one group's exchange overlaps another
group's attention (the guide's head-grouped collective overlap).

The exchanges are `torch.distributed.all_to_all_single` calls (NCCL over
NVLink / NVSwitch on GPUs, gloo on CPU) issued asynchronously; the attention
is `attn_fwd` of this package unless another callable is given.  Nothing here
reads a peer's memory directly.

Layouts (per rank r of P): q [B, N/P, Hq, d], k and v [B, N/P, Hkv, d], rank r
holding sequence rows [r N/P, (r+1) N/P); the result o [B, N/P, Hq, d] and
lse [B, Hq, N/P] for the same rows.  Query head h lives on rank h // (Hq/P)
during attention, KV head g on rank g // (Hkv/P), so GQA groups stay whole
when Hkv % P == 0.
"""
from __future__ import annotations

import math


def _check(B, Nl, Hq, Hkv, P, groups):
    if Hq % P or Hkv % P:
        raise ValueError(f"Hq ({Hq}) and Hkv ({Hkv}) must be multiples of the world size ({P})")
    if (Hkv // P) % groups:
        raise ValueError(f"Hkv / P ({Hkv // P}) must be a multiple of head_groups ({groups})")
    if Hq % Hkv:
        raise ValueError(f"Hq ({Hq}) must be a multiple of Hkv ({Hkv})")


def _to_heads(x, P, g, ng):
    """[B, Nl, H, d] -> send buffer [P, B, Nl, Hg, d]: chunk i holds head
    group g of the heads rank i will own."""
    B, Nl, H, d = x.shape
    Hp = H // P
    Hg = Hp // ng
    return x.view(B, Nl, P, Hp, d)[:, :, :, g * Hg:(g + 1) * Hg, :].permute(2, 0, 1, 3, 4).contiguous()


def _from_seq(buf):
    """receive buffer [P, B, Nl, Hg, d] (chunk j = rank j's rows) -> [B, P*Nl, Hg, d]."""
    P, B, Nl, Hg, d = buf.shape
    return buf.permute(1, 0, 2, 3, 4).reshape(B, P * Nl, Hg, d)


def default_attention(q, k, v, mask_kind, scale):
    from . import attn_fwd
    return attn_fwd(q.contiguous(), k.contiguous(), v.contiguous(), scale=scale, mask_kind=mask_kind)


def ulysses_attention(q, k, v, group=None, mask_kind=0, scale=None, head_groups=1, attention=None):
    """Sequence-parallel attention over the ranks of `group` (the default
    process group if None).  Returns (o, lse) for this rank's rows.

    attention(q, k, v, mask_kind, scale) -> (o [B,N,H,d], lse [B,H,N]) runs on
    whole sequences; the default is this package's attn_fwd (bf16 CUDA
    tensors).  mask_kind is NONE or CAUSAL: the whole sequence is present on
    every rank, so a causal mask needs no change."""
    import torch
    import torch.distributed as dist

    P = dist.get_world_size(group) if dist.is_initialized() else 1
    B, Nl, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attention = attention or default_attention
    _check(B, Nl, Hq, Hkv, P, head_groups)
    if P == 1:
        return attention(q, k, v, mask_kind, scale)
    ng = head_groups
    Hqg, Hkg = Hq // P // ng, Hkv // P // ng

    # 1. post every group's input exchange (they proceed in the background)
    sends, recvs, works = [], [], []
    for g in range(ng):
        xs = [_to_heads(t, P, g, ng) for t in (q, k, v)]
        rs = [torch.empty_like(x) for x in xs]
        works.append([dist.all_to_all_single(r_, x_, group=group, async_op=True) for r_, x_ in zip(rs, xs)])
        sends.append(xs)
        recvs.append(rs)
    # 2. per group: wait for its inputs, attend, post its output exchange
    out_works, out_bufs = [], []
    for g in range(ng):
        for w in works[g]:
            w.wait()
        qg, kg, vg = (_from_seq(r_) for r_ in recvs[g])
        o_g, lse_g = attention(qg, kg, vg, mask_kind, scale)  # [B, N, Hqg, d], [B, Hqg, N]
        o_send = o_g.view(B, P, Nl, Hqg, d).permute(1, 0, 2, 3, 4).contiguous()
        l_send = lse_g.view(B, Hqg, P, Nl).permute(2, 0, 1, 3).contiguous()
        o_recv, l_recv = torch.empty_like(o_send), torch.empty_like(l_send)
        out_works.append((dist.all_to_all_single(o_recv, o_send, group=group, async_op=True),
                          dist.all_to_all_single(l_recv, l_send, group=group, async_op=True)))
        out_bufs.append((o_send, l_send, o_recv, l_recv))
    # 3. reassemble this rank's rows: chunk i of group g holds query heads
    #    i*Hq/P + g*Hqg .. of every row here
    o = torch.empty((B, Nl, P, ng, Hqg, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, P, ng, Hqg, Nl), dtype=torch.float32 if q.is_cuda else out_bufs[0][3].dtype,
                      device=q.device)
    for g in range(ng):
        for w in out_works[g]:
            w.wait()
        o_recv, l_recv = out_bufs[g][2], out_bufs[g][3]
        o[:, :, :, g] = o_recv.permute(1, 2, 0, 3, 4)
        lse[:, :, g] = l_recv.permute(1, 0, 2, 3).to(lse.dtype)
    return o.view(B, Nl, Hq, d), lse.view(B, Hq, Nl)
