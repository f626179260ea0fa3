"""Ulysses sequence parallelism with this library's CUDA kernels, against the
fp64 oracle on the unsharded tensors.

"TPU attention optimisation guide: collective overlap and mask removal,
verified by trace", step 2: each rank holds a slice of the sequence, an
all-to-all swaps sequence shards for head shards, attention runs on whole
sequences for the rank's heads, and a second all-to-all swaps back.

Two or three ranks run as separate processes on the one GPU of this machine.
The exchanges are gloo all-to-alls over CPU tensors (bf16 as is); the
attention and its backward are the package's attn_fwd / attn_bwd on cuda:0,
each call moving its head shard to the device and its result back.  No rank's
kernel waits on another rank: every exchange happens on the host, between
kernel calls.  The gathered O, LSE, dQ, dK and dV must meet the same
tolerances as the single-call parity tests.
"""
import datetime
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synthetic

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3
GRAD_MAX_REL, GRAD_MEAN_REL = 2e-2, 1e-2

# world, (B, N, Hq, Hkv, d), mask kind, head groups, shard lengths (None: equal)
CASES = [
    (2, (1, 384, 8, 4, 128), 1, 1, None),            # causal GQA, equal shards
    (2, (2, 256, 8, 4, 64), 0, 2, None),             # no mask, two head groups with their own exchanges
    (3, (2, 301, 6, 3, 64), 1, 1, [100, 1, 200]),    # three ranks, uneven shards, one holding a single row
    (3, (1, 390, 6, 3, 128), 1, 1, [130, 130, 130]), # three ranks, Hq/P = 2 query heads per rank
]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(case_index, B, N, Hq, Hkv, d):
    seed = 4400 + case_index
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, N, Hq, d))
    k = synthetic.tensor(seed, synthetic.TID_K, (B, N, Hkv, d))
    v = synthetic.tensor(seed, synthetic.TID_V, (B, N, Hkv, d))
    dout = synthetic.tensor(seed, 9, (B, N, Hq, d))
    return q, k, v, dout


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _rank_main(rank, world, port, case_index, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import exact_io_aware_sm_b200 as eio
    from exact_io_aware_sm_b200.ulysses import (default_attention, default_backward, ulysses_attention,
                                                ulysses_attention_bwd)
    torch.cuda.set_device(0)
    eio.lib()
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        world_, (B, N, Hq, Hkv, d), mask_kind, groups, lens = CASES[case_index]
        lens = lens or [N // world] * world
        q, k, v, dout = _inputs(case_index, B, N, Hq, Hkv, d)
        r0 = sum(lens[:rank])
        sl = slice(r0, r0 + lens[rank])
        tq, tk, tv, tdo = (_bf16(x[:, sl]) for x in (q, k, v, dout))
        scale = 1 / math.sqrt(d)

        def attention(q_, k_, v_, mk, sc):
            o_, l_ = default_attention(q_.cuda(), k_.cuda(), v_.cuda(), mk, sc)
            eio.sync_status()
            return o_.cpu(), l_.cpu()

        def backward(q_, k_, v_, o_, l_, do_, mk, sc):
            g = default_backward(*(t.cuda() for t in (q_, k_, v_, o_, l_, do_)), mk, sc)
            eio.sync_status()
            return tuple(t.cpu() for t in g)

        o, lse = ulysses_attention(tq, tk, tv, mask_kind=mask_kind, scale=scale, head_groups=groups,
                                   attention=attention, shard_lens=lens)
        dq, dk, dv = ulysses_attention_bwd(tq, tk, tv, o, lse, tdo, mask_kind=mask_kind, scale=scale,
                                           head_groups=groups, backward=backward, shard_lens=lens)
        f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
        out_q.put((rank, f64(o), lse.numpy().astype(np.float64), f64(dq), f64(dk), f64(dv)))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from exact_io_aware_sm_b200 import build
    build.build()


def _check_grad(got, ref, where):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{where}: non-finite gradient"
    assert err.max() <= GRAD_MAX_REL * np.abs(ref).max() + 1e-6, f"{where}: max err {err.max():.3e}"
    assert err.mean() <= GRAD_MEAN_REL * np.abs(ref).mean() + 1e-7, f"{where}: mean err {err.mean():.3e}"


@pytest.mark.parametrize("case_index", range(len(CASES)),
                         ids=[f"P{c[0]}-N{c[1][1]}-d{c[1][4]}-mask{c[2]}-g{c[3]}" for c in CASES])
def test_ulysses_with_cuda_kernels_equals_unsharded_oracle(case_index):
    world, (B, N, Hq, Hkv, d), mask_kind, groups, lens = CASES[case_index]
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case_index, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            r, *res = out_q.get(timeout=300)
            got[r] = res
    finally:
        for p in procs:
            p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    o, dq, dk, dv = (np.concatenate([got[r][i] for r in range(world)], axis=1) for i in (0, 2, 3, 4))
    lse = np.concatenate([got[r][1] for r in range(world)], axis=2)

    q, k, v, dout = _inputs(case_index, B, N, Hq, Hkv, d)
    scale = 1 / math.sqrt(d)
    ro, rl = oracle.attn_fwd(q, k, v, scale, mask_kind)
    err = np.abs(o - ro)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN, f"O {err.max():.3e} {err.mean():.3e}"
    assert np.abs(lse - rl).max() <= LSE_TOL
    rq, rk, rv = oracle.attn_bwd(q, k, v, dout, scale, mask_kind)
    _check_grad(dq, rq, "dq")
    _check_grad(dk, rk, "dk")
    _check_grad(dv, rv, "dv")
