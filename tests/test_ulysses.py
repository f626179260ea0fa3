"""Ulysses sequence parallelism on CPU ranks (gloo).

Each rank holds a slice of the sequence; the module swaps sequence shards for
head shards with all-to-alls, runs attention on whole sequences for its heads
and swaps back.  With the fp64 oracle as the attention (test infrastructure
only), the result gathered over the ranks must equal the oracle on the whole,
unsharded tensors: the exchange is pure data movement, so the comparison is
exact up to the oracle's own rounding.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_attention(q, k, v, mask_kind, scale):
    import oracle
    o, lse = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), scale, mask_kind)
    return torch.from_numpy(o), torch.from_numpy(lse)


def _inputs(B, N, Hq, Hkv, d):
    rng = np.random.default_rng(77)
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    return q, k, v


def _rank_main(rank, world, port, shape, mask_kind, groups, out_q, lens=None, pass_lens=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    from exact_io_aware_sm_b200.ulysses import ulysses_attention
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, Hq, Hkv, d = shape
        q, k, v = _inputs(B, N, Hq, Hkv, d)
        lens = lens or [N // world] * world
        r0 = sum(lens[:rank])
        sl = slice(r0, r0 + lens[rank])
        tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x[:, sl])) for x in (q, k, v))
        o, lse = ulysses_attention(tq, tk, tv, mask_kind=mask_kind, scale=1 / math.sqrt(d), head_groups=groups,
                                   attention=_oracle_attention, shard_lens=lens if pass_lens else None)
        out_q.put((rank, o.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _run(world, shape, mask_kind, groups, lens=None, pass_lens=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, shape, mask_kind, groups, q, lens, pass_lens))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, o, lse = q.get(timeout=180)
        got[r] = (o, lse)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    o = np.concatenate([got[r][0] for r in range(world)], axis=1)
    lse = np.concatenate([got[r][1] for r in range(world)], axis=2)
    return o, lse


@pytest.mark.parametrize("world,shape,mask_kind,groups", [
    (2, (1, 64, 4, 2, 8), 1, 1),   # causal, GQA (2 query heads per KV head)
    (2, (2, 48, 8, 4, 16), 0, 2),  # two head groups, each with its own exchanges
    (4, (1, 64, 8, 4, 8), 1, 1),   # four ranks
])
def test_ulysses_equals_unsharded_attention(world, shape, mask_kind, groups):
    import oracle
    B, N, Hq, Hkv, d = shape
    o, lse = _run(world, shape, mask_kind, groups)
    q, k, v = _inputs(B, N, Hq, Hkv, d)
    ro, rlse = oracle.attn_fwd(q, k, v, 1 / math.sqrt(d), mask_kind)
    np.testing.assert_allclose(o, ro, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse, rlse, atol=1e-13, rtol=0)


@pytest.mark.parametrize("world,shape,mask_kind,groups,lens,pass_lens", [
    (2, (1, 61, 4, 2, 8), 1, 1, [33, 28], False),     # causal, last shard shorter, lengths gathered
    (2, (2, 40, 4, 4, 8), 0, 2, [9, 31], True),       # first shard shorter, lengths given, two groups
    (3, (1, 50, 6, 3, 8), 1, 1, [20, 1, 29], False),  # three ranks, one holding a single row
])
def test_ulysses_uneven_shards(world, shape, mask_kind, groups, lens, pass_lens):
    """Shards of different lengths: padded for the exchanges, the padding is
    never attended (keys) nor returned (rows), so the gathered result equals
    attention on the unsharded sequence."""
    import oracle
    B, N, Hq, Hkv, d = shape
    assert sum(lens) == N
    o, lse = _run(world, shape, mask_kind, groups, lens, pass_lens)
    q, k, v = _inputs(B, N, Hq, Hkv, d)
    ro, rlse = oracle.attn_fwd(q, k, v, 1 / math.sqrt(d), mask_kind)
    assert o.shape == ro.shape and lse.shape == rlse.shape
    np.testing.assert_allclose(o, ro, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse, rlse, atol=1e-13, rtol=0)


def test_layout_helpers_round_trip():
    """The send buffer of head group g for rank i holds exactly rank i's heads
    of that group; reassembling the received chunks restores the rows."""
    from exact_io_aware_sm_b200.ulysses import _from_seq, _to_heads
    B, Nl, H, d, P, ng = 2, 3, 8, 4, 2, 2
    x = torch.arange(B * Nl * H * d, dtype=torch.float64).view(B, Nl, H, d)
    for g in range(ng):
        buf = _to_heads(x, P, g, ng)
        assert buf.shape == (P, B, Nl, H // P // ng, d)
        for i in range(P):
            h0 = i * (H // P) + g * (H // P // ng)
            assert torch.equal(buf[i], x[:, :, h0:h0 + H // P // ng])
    # as if every rank sent this same buffer: rows of rank j land at j*Nl
    buf = _to_heads(x, P, 0, 1)
    whole = _from_seq(buf)
    assert whole.shape == (B, P * Nl, H // P, d)
    assert torch.equal(whole[:, Nl:2 * Nl], x[:, :, H // P:2 * (H // P)])


def test_argument_checks():
    from exact_io_aware_sm_b200.ulysses import _check
    with pytest.raises(ValueError):
        _check(1, 8, 6, 3, 4, 1)   # heads not divisible by the world size
    with pytest.raises(ValueError):
        _check(1, 8, 8, 4, 2, 4)   # Hkv/P = 2 not a multiple of 4 head groups
    _check(1, 8, 8, 4, 2, 2)


def test_single_rank_is_the_plain_call():
    from exact_io_aware_sm_b200.ulysses import ulysses_attention
    q, k, v = (torch.from_numpy(x) for x in _inputs(1, 16, 2, 1, 4))
    calls = []

    def att(q_, k_, v_, mk, sc):
        calls.append(q_.shape)
        return _oracle_attention(q_, k_, v_, mk, sc)
    o, lse = ulysses_attention(q, k, v, mask_kind=1, attention=att)
    assert calls == [q.shape]


def _oracle_backward(q, k, v, o, lse, dout, mask_kind, scale):
    """The fp64 oracle's gradients.  It recomputes P from q, k, v, so it also
    checks that the o and lse it was handed are those of the same rows and
    heads (the exchanges must move them with their q)."""
    import oracle
    ro, rl = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), scale, mask_kind)
    assert np.array_equal(o.numpy(), ro) and np.array_equal(lse.numpy(), rl), "o / lse routed to the wrong rows"
    dq, dk, dv = oracle.attn_bwd(q.numpy(), k.numpy(), v.numpy(), dout.numpy(), scale, mask_kind)
    return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)


def _bwd_rank_main(rank, world, port, shape, mask_kind, groups, out_q, lens):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import oracle
    from exact_io_aware_sm_b200.ulysses import ulysses_attention_bwd
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, Hq, Hkv, d = shape
        q, k, v = _inputs(B, N, Hq, Hkv, d)
        dout = np.random.default_rng(78).standard_normal((B, N, Hq, d))
        scale = 1 / math.sqrt(d)
        o, lse = oracle.attn_fwd(q, k, v, scale, mask_kind)
        r0 = sum(lens[:rank])
        sl = slice(r0, r0 + lens[rank])
        t = [torch.from_numpy(np.ascontiguousarray(x[:, sl])) for x in (q, k, v, o, dout)]
        tl = torch.from_numpy(np.ascontiguousarray(lse[:, :, sl]))
        dq, dk, dv = ulysses_attention_bwd(t[0], t[1], t[2], t[3], tl, t[4], mask_kind=mask_kind, scale=scale,
                                           head_groups=groups, backward=_oracle_backward)
        out_q.put((rank, dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape,mask_kind,groups,lens", [
    (2, (1, 64, 4, 2, 8), 1, 1, [32, 32]),       # causal, GQA, equal shards
    (2, (2, 40, 8, 4, 8), 0, 2, [15, 25]),       # two head groups, uneven shards
    (3, (1, 45, 6, 3, 8), 1, 1, [20, 1, 24]),    # three ranks, one holding a single row
])
def test_ulysses_backward_equals_unsharded_gradients(world, shape, mask_kind, groups, lens):
    import oracle
    B, N, Hq, Hkv, d = shape
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_rank_main, args=(r, world, port, shape, mask_kind, groups, qq, lens))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, dq, dk, dv = qq.get(timeout=180)
        got[r] = (dq, dk, dv)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    dq, dk, dv = (np.concatenate([got[r][i] for r in range(world)], axis=1) for i in range(3))
    q, k, v = _inputs(B, N, Hq, Hkv, d)
    dout = np.random.default_rng(78).standard_normal((B, N, Hq, d))
    rq, rk, rv = oracle.attn_bwd(q, k, v, dout, 1 / math.sqrt(d), mask_kind)
    for got_, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert got_.shape == ref.shape
        np.testing.assert_allclose(got_, ref, atol=1e-12, rtol=0)


def _plain_oracle_backward(q, k, v, o, lse, dout, mask_kind, scale):
    import oracle
    dq, dk, dv = oracle.attn_bwd(q.numpy(), k.numpy(), v.numpy(), dout.numpy(), scale, mask_kind)
    return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)


def _autograd_rank_main(rank, world, port, shape, mask_kind, lens, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    from exact_io_aware_sm_b200.ulysses import ulysses_attention_autograd
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, Hq, Hkv, d = shape
        q, k, v = _inputs(B, N, Hq, Hkv, d)
        w = np.random.default_rng(79).standard_normal((B, N, Hq, d))
        r0 = sum(lens[:rank])
        sl = slice(r0, r0 + lens[rank])
        tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x[:, sl])).requires_grad_(True) for x in (q, k, v))
        o = ulysses_attention_autograd(tq, tk, tv, mask_kind=mask_kind, scale=1 / math.sqrt(d),
                                       attention=_oracle_attention, backward=_plain_oracle_backward)
        (o * torch.from_numpy(np.ascontiguousarray(w[:, sl]))).sum().backward()
        out_q.put((rank, tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape,mask_kind,lens", [
    (2, (1, 48, 4, 2, 8), 1, [24, 24]),
    (3, (2, 40, 6, 3, 8), 0, [10, 17, 13]),
])
def test_ulysses_autograd_gradients(world, shape, mask_kind, lens):
    """Each rank backpropagates a loss over its own rows; the gathered input
    gradients equal those of the loss over the unsharded sequence."""
    import oracle
    B, N, Hq, Hkv, d = shape
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_autograd_rank_main, args=(r, world, port, shape, mask_kind, lens, qq))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, dq, dk, dv = qq.get(timeout=180)
        got[r] = (dq, dk, dv)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    dq, dk, dv = (np.concatenate([got[r][i] for r in range(world)], axis=1) for i in range(3))
    q, k, v = _inputs(B, N, Hq, Hkv, d)
    w = np.random.default_rng(79).standard_normal((B, N, Hq, d))
    rq, rk, rv = oracle.attn_bwd(q, k, v, w, 1 / math.sqrt(d), mask_kind)
    for got_, ref in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(got_, ref, atol=1e-12, rtol=0)


def _bad_lens_rank_main(rank, world, port, out_q, lens_per_rank, backward=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    from exact_io_aware_sm_b200.ulysses import ulysses_attention, ulysses_attention_bwd
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = torch.zeros((1, 4, 2, 8), dtype=torch.float64)  # every rank holds 4 rows
        lse = torch.zeros((1, 2, 4), dtype=torch.float64)
        try:
            if backward:
                ulysses_attention_bwd(x, x, x, x, lse, x, backward=lambda *a: None,
                                      shard_lens=lens_per_rank[rank])
            else:
                ulysses_attention(x, x, x, attention=_oracle_attention, shard_lens=lens_per_rank[rank])
            out_q.put((rank, "returned"))
        except ValueError as e:
            out_q.put((rank, "ValueError" if "shard_lens" in str(e) else str(e)))
        # The group is still usable: a collective after the refusal completes.
        t = torch.ones(1)
        dist.all_reduce(t)
        assert t.item() == world
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens_per_rank,backward", [
    ([[5, 3], [5, 3]], False),   # every rank's own entry is wrong
    ([[4, 3], [4, 3]], False),   # only rank 1's entry is wrong: rank 0 must raise too
    ([[4, 4], [4, 3]], False),   # the ranks pass different lists
    ([[4, 4], [4, 4, 0]], False),  # one rank's list has the wrong length
    ([[4, 3], [4, 3]], True),    # the same agreement in the backward
])
def test_ulysses_rejects_shard_lengths_that_do_not_match(lens_per_rank, backward):
    """shard_lens that disagree with the rows the ranks hold raise ValueError
    on every rank before any exchange starts (so nothing waits on a peer),
    even when a rank's own entry is right or the ranks pass different lists."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bad_lens_rank_main, args=(r, 2, port, q, lens_per_rank, backward))
             for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert got == {0: "ValueError", 1: "ValueError"}
