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

Layouts (per rank r of P): q [B, N_r, Hq, d], k and v [B, N_r, Hkv, d], rank r
holding the contiguous sequence rows that follow those of ranks 0..r-1; the
result o [B, N_r, Hq, d] and lse [B, Hq, N_r] for the same rows.  The shards
may differ in length (N = sum of N_r): each is padded to the longest for the
exchange, the padding is dropped before attention (which sees exactly the N
rows, so masks and the LSE are those of the unsharded sequence) and restored
for the return exchange.  Query head h lives on rank h // (Hq/P) during
attention, KV head g on rank g // (Hkv/P), so GQA groups stay whole when
Hkv % P == 0.
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


def _shard_lens(Nl, P, group, device, given=None):
    """Every rank's shard length, agreed by all ranks with one small
    all-gather before any exchange.  Each rank sends its row count and the
    shard_lens it was given (if any); every rank then checks every given list
    against the gathered counts, so all ranks reach the same verdict and raise
    together (no rank goes on into an all-to-all that another one left)."""
    import torch
    import torch.distributed as dist
    row = torch.full((P + 2,), -1, dtype=torch.int64)
    row[0] = Nl
    if given is None:
        row[1] = 0
    elif len(given) != P:
        row[1] = 2  # malformed: wrong number of entries
    else:
        row[1] = 1
        row[2:] = torch.tensor([int(n) for n in given], dtype=torch.int64)
    row = row.to(device)
    allv = [torch.zeros_like(row) for _ in range(P)]
    dist.all_gather(allv, row, group=group)
    rows = [t.cpu().tolist() for t in allv]
    actual = [r[0] for r in rows]
    bad = [i for i, r in enumerate(rows) if r[1] == 2 or (r[1] == 1 and r[2:] != actual)]
    if bad:
        raise ValueError(f"shard_lens given on rank(s) {bad} do not match the ranks' rows {actual}")
    return actual


def _pad_rows(x, n):
    """[B, Nl, ...] -> [B, n, ...] with zero rows appended (x itself if Nl == n)."""
    import torch
    if x.shape[1] == n:
        return x
    pad = torch.zeros((x.shape[0], n - x.shape[1]) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    return torch.cat([x, pad], dim=1)


def ulysses_attention(q, k, v, group=None, mask_kind=0, scale=None, head_groups=1, attention=None,
                      shard_lens=None):
    """Sequence-parallel attention over the ranks of `group` (the default
    process group if None).  Returns (o, lse) for this rank's rows.

    attention(q, k, v, mask_kind, scale) -> (o [B,N,H,d], lse [B,H,N]) runs on
    whole sequences; the default is this package's attn_fwd (bf16 CUDA
    tensors).  mask_kind is NONE or CAUSAL: the whole sequence is present on
    every rank, so a causal mask needs no change.  shard_lens: every rank's
    number of rows, in rank order, if the caller knows them; the lengths are
    gathered either way, and a given list that does not match them raises
    ValueError on every rank before any exchange (shards of equal length need
    no padding)."""
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
    lens = _shard_lens(Nl, P, group, q.device, None if shard_lens is None else list(shard_lens))
    Np = max(lens)  # every shard padded to this many rows for the exchanges
    ragged = any(n != Np for n in lens)
    # rows of the padded, gathered sequence that hold real rows, in sequence order
    keep = None
    if ragged:
        keep = torch.cat([torch.arange(j * Np, j * Np + n, device=q.device) for j, n in enumerate(lens)])
        q, k, v = (_pad_rows(t, Np) for t in (q, k, v))
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
        if ragged:  # drop the padding: attention sees exactly the N rows
            qg, kg, vg = (t.index_select(1, keep).contiguous() for t in (qg, kg, vg))
        o_g, lse_g = attention(qg, kg, vg, mask_kind, scale)  # [B, N, Hqg, d], [B, Hqg, N]
        if ragged:  # back to the padded layout for the return exchange
            o_p = torch.zeros((B, P * Np, Hqg, d), dtype=o_g.dtype, device=o_g.device)
            o_p[:, keep] = o_g
            l_p = torch.zeros((B, Hqg, P * Np), dtype=lse_g.dtype, device=lse_g.device)
            l_p[:, :, keep] = lse_g
            o_g, lse_g = o_p, l_p
        o_send = o_g.view(B, P, Np, Hqg, d).permute(1, 0, 2, 3, 4).contiguous()
        l_send = lse_g.view(B, Hqg, P, Np).permute(2, 0, 1, 3).contiguous()
        o_recv, l_recv = torch.empty_like(o_send), torch.empty_like(l_send)
        out_works.append((dist.all_to_all_single(o_recv, o_send, group=group, async_op=True),
                          dist.all_to_all_single(l_recv, l_send, group=group, async_op=True)))
        out_bufs.append((o_send, l_send, o_recv, l_recv))
    # 3. reassemble this rank's rows: chunk i of group g holds query heads
    #    i*Hq/P + g*Hqg .. of every row here
    o = torch.empty((B, Np, P, ng, Hqg, d), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, P, ng, Hqg, Np), dtype=torch.float32 if q.is_cuda else out_bufs[0][3].dtype,
                      device=q.device)
    for g in range(ng):
        for w in out_works[g]:
            w.wait()
        o_recv, l_recv = out_bufs[g][2], out_bufs[g][3]
        o[:, :, :, g] = o_recv.permute(1, 2, 0, 3, 4)
        lse[:, :, g] = l_recv.permute(1, 0, 2, 3).to(lse.dtype)
    o, lse = o.view(B, Np, Hq, d), lse.view(B, Hq, Np)
    if ragged:
        o, lse = o[:, :Nl].contiguous(), lse[:, :, :Nl].contiguous()
    return o, lse


def _lse_to_heads(lse, P, g, ng):
    """[B, H, Nl] -> send buffer [P, B, Hg, Nl]: chunk i holds head group g of
    the heads rank i will own."""
    B, H, Nl = lse.shape
    Hp = H // P
    Hg = Hp // ng
    return lse.view(B, P, Hp, Nl)[:, :, g * Hg:(g + 1) * Hg, :].permute(1, 0, 2, 3).contiguous()


def _lse_from_seq(buf):
    """receive buffer [P, B, Hg, Nl] (chunk j = rank j's rows) -> [B, Hg, P*Nl]."""
    P, B, Hg, Nl = buf.shape
    return buf.permute(1, 2, 0, 3).reshape(B, Hg, P * Nl)


def default_backward(q, k, v, o, lse, dout, mask_kind, scale):
    from . import attn_bwd
    c = [t.contiguous() for t in (q, k, v, o, lse, dout)]
    return attn_bwd(*c, scale=scale, mask_kind=mask_kind)


def ulysses_attention_bwd(q, k, v, o, lse, dout, group=None, mask_kind=0, scale=None, head_groups=1,
                          backward=None, shard_lens=None):
    """Gradients of ulysses_attention for this rank's rows: q, o, dout
    [B, N_r, Hq, d], k, v [B, N_r, Hkv, d], lse [B, Hq, N_r] as the forward
    returned them.  Returns (dq, dk, dv) shaped like q, k, v.

    The same exchanges as the forward: every input goes from sequence shards
    to head shards, backward(q, k, v, o, lse, dout, mask_kind, scale) ->
    (dq, dk, dv) runs on whole sequences (default: this package's attn_bwd,
    which recomputes P from the LSE), and the gradients return to the rows'
    owners; head groups overlap one group's exchanges with another's
    backward, and uneven shards are padded as in the forward."""
    import torch
    import torch.distributed as dist

    P = dist.get_world_size(group) if dist.is_initialized() else 1
    B, Nl, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    backward = backward or default_backward
    _check(B, Nl, Hq, Hkv, P, head_groups)
    if P == 1:
        return backward(q, k, v, o, lse, dout, mask_kind, scale)
    lens = _shard_lens(Nl, P, group, q.device, None if shard_lens is None else list(shard_lens))
    Np = max(lens)
    ragged = any(n != Np for n in lens)
    keep = None
    if ragged:
        keep = torch.cat([torch.arange(j * Np, j * Np + n, device=q.device) for j, n in enumerate(lens)])
        q, k, v, o, dout = (_pad_rows(t, Np) for t in (q, k, v, o, dout))
        lse = _pad_rows(lse.transpose(1, 2), Np).transpose(1, 2).contiguous()
    ng = head_groups
    Hqg, Hkg = Hq // P // ng, Hkv // P // ng

    # 1. post every group's input exchanges
    recvs, works = [], []
    for g in range(ng):
        xs = [_to_heads(t, P, g, ng) for t in (q, k, v, o, dout)] + [_lse_to_heads(lse, P, g, ng)]
        rs = [torch.empty_like(x) for x in xs]
        works.append([dist.all_to_all_single(r_, x_, group=group, async_op=True) for r_, x_ in zip(rs, xs)])
        recvs.append((xs, rs))
    # 2. per group: wait, run the backward on whole sequences, post the return exchanges
    out = []
    for g in range(ng):
        for w in works[g]:
            w.wait()
        rs = recvs[g][1]
        qg, kg, vg, og, dog = (_from_seq(r_) for r_ in rs[:5])
        lg = _lse_from_seq(rs[5])
        if ragged:
            qg, kg, vg, og, dog = (t.index_select(1, keep).contiguous() for t in (qg, kg, vg, og, dog))
            lg = lg.index_select(2, keep).contiguous()
        dqg, dkg, dvg = backward(qg, kg, vg, og, lg, dog, mask_kind, scale)
        sends = []
        for t, H_ in ((dqg, Hqg), (dkg, Hkg), (dvg, Hkg)):
            if ragged:
                tp = torch.zeros((B, P * Np, H_, d), dtype=t.dtype, device=t.device)
                tp[:, keep] = t
                t = tp
            sends.append(t.view(B, P, Np, H_, d).permute(1, 0, 2, 3, 4).contiguous())
        rbufs = [torch.empty_like(x) for x in sends]
        ws = [dist.all_to_all_single(r_, x_, group=group, async_op=True) for r_, x_ in zip(rbufs, sends)]
        out.append((sends, rbufs, ws))
    # 3. reassemble this rank's rows
    dq = torch.empty((B, Np, P, ng, Hqg, d), dtype=q.dtype, device=q.device)
    dk = torch.empty((B, Np, P, ng, Hkg, d), dtype=k.dtype, device=k.device)
    dv = torch.empty((B, Np, P, ng, Hkg, d), dtype=v.dtype, device=v.device)
    for g in range(ng):
        sends, rbufs, ws = out[g]
        for w in ws:
            w.wait()
        for dst, r_ in zip((dq, dk, dv), rbufs):
            dst[:, :, :, g] = r_.permute(1, 2, 0, 3, 4).to(dst.dtype)
    dq, dk, dv = dq.view(B, Np, Hq, d), dk.view(B, Np, Hkv, d), dv.view(B, Np, Hkv, d)
    if ragged:
        dq, dk, dv = (t[:, :Nl].contiguous() for t in (dq, dk, dv))
    return dq, dk, dv


def ulysses_attention_autograd(q, k, v, group=None, mask_kind=0, scale=None, head_groups=1, attention=None,
                               backward=None, shard_lens=None):
    """ulysses_attention as a differentiable op: its backward is
    ulysses_attention_bwd with the O and LSE the forward returned.  Returns o
    for this rank's rows (the LSE carries no gradient and is not returned).
    attention / backward replace the whole-sequence calls as in the two
    functions above."""
    import torch

    class _Ulysses(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q_, k_, v_):
            o, lse = ulysses_attention(q_.contiguous(), k_.contiguous(), v_.contiguous(), group=group,
                                       mask_kind=mask_kind, scale=scale, head_groups=head_groups,
                                       attention=attention, shard_lens=shard_lens)
            ctx.save_for_backward(q_, k_, v_, o, lse)
            return o

        @staticmethod
        def backward(ctx, dout):
            q_, k_, v_, o, lse = ctx.saved_tensors
            return ulysses_attention_bwd(q_.contiguous(), k_.contiguous(), v_.contiguous(), o, lse, dout.contiguous(),
                                         group=group, mask_kind=mask_kind, scale=scale, head_groups=head_groups,
                                         backward=backward, shard_lens=shard_lens)

    return _Ulysses.apply(q, k, v)
