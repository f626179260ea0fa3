"""Seeded random shapes through every entry point, against the fp64 oracle.

The hand-picked cases in test_gpu_parity.py cover the tile boundaries and
degenerate cases one by one; these draw the sizes at random (from one fixed
seed, so every run checks the same shapes) over the whole supported range:
batch, query heads per KV head (including odd groups), ragged lengths with
Nq != Nkv in both directions, d in {64, 128}, every mask kind, block maps of
varying density with empty block rows, decode lengths of zero, and
multi-token decode.  Two sets: a quick one (sequences up to 700) and a
larger one (up to 1500).  The tolerances are those of the other parity tests.
"""
import math

import numpy as np
import pytest
import torch

import exact_io_aware_sm_b200 as eio
import oracle
import synthetic
from tests.test_gpu_parity import (check, check_grad, dev_bf16, make_inputs, oracle_decode_multi, run_decode,
                                   run_fwd)

pytestmark = pytest.mark.gpu

SEED = 20240611      # the quick set
SEED_LARGE = 777001  # the larger set


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from exact_io_aware_sm_b200 import build
    build.build()
    eio.lib()
    yield
    eio.sync_status()


def _block_map(rng, Nq, Nkv):
    p = float(rng.uniform(0.15, 0.85))
    bm = (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < p).astype(np.uint8)
    if bm.shape[0] > 2 and rng.random() < 0.5:
        bm[int(rng.integers(0, bm.shape[0]))] = 0  # a block row that sees no key
    return bm


def _fwd_cases(n, seed, nmax, groups, kinds, base):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([64, 128]))
        G = int(rng.choice(groups))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 4))
        Nq, Nkv = (int(x) for x in rng.integers(1, nmax, size=2))
        kind = str(rng.choice(kinds))
        out.append((base, i, B, G * Hkv, Hkv, Nq, Nkv, d, kind))
    return out


def _ids(cases):
    return [f"{c[0]}-{c[-1]}-b{c[2]}h{c[3]}g{c[3] // c[4]}-{c[5]}x{c[6]}-d{c[7]}" for c in cases]


def _mask(kind, rng, Nq, Nkv):
    if kind == "none":
        return eio.MASK_NONE, None
    if kind == "causal":
        return eio.MASK_CAUSAL, None
    return eio.MASK_BLOCK, _block_map(rng, Nq, Nkv)


FWD = (_fwd_cases(24, SEED, 700, [1, 2, 3, 4, 8], ["none", "causal", "block"], SEED) +
       _fwd_cases(120, SEED_LARGE, 1500, [1, 2, 3, 4, 8], ["none", "causal", "block"], SEED_LARGE))


@pytest.mark.parametrize("case", FWD, ids=_ids(FWD))
def test_fuzz_forward_bf16(case):
    base, i, B, Hq, Hkv, Nq, Nkv, d, kind = case
    rng = np.random.default_rng(base + 1000 + i)
    q, k, v = make_inputs(base + i, B, Hq, Hkv, Nq, Nkv, d)
    mk, bm = _mask(kind, rng, Nq, Nkv)
    scale = float(rng.uniform(0.5, 1.5)) / math.sqrt(d)
    o, lse = run_fwd(q, k, v, scale, mk, bm)
    ro, rl = oracle.attn_fwd(q, k, v, scale, mk, bm)
    check(o, lse, ro, rl, f"fwd {case}")


FWD32 = [(*c[:7], int(np.random.default_rng(SEED + 50 + c[1]).choice([32, 64, 128])), c[8])
         for c in _fwd_cases(6, SEED + 50, 300, [1, 2, 4], ["none", "causal", "block"], SEED)]


@pytest.mark.parametrize("case", FWD32, ids=_ids(FWD32))
def test_fuzz_forward_fp32(case):
    base, i, B, Hq, Hkv, Nq, Nkv, d, kind = case
    rng = np.random.default_rng(base + 2000 + i)
    q, k, v = make_inputs(base + 100 + i, B, Hq, Hkv, Nq, Nkv, d, "f32")
    mk, bm = _mask(kind, rng, Nq, Nkv)
    scale = 1 / math.sqrt(d)
    o, lse = run_fwd(q, k, v, scale, mk, bm)
    ro, rl = oracle.attn_fwd(q, k, v, scale, mk, bm)
    check(o, lse, ro, rl, f"fwd32 {case}")


def _decode_cases(n, seed, base):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([64, 128]))
        G = int(rng.choice([1, 2, 4, 8]))
        Sq = int(rng.choice([s for s in (1, 2, 3, 4, 8, 16) if G * s <= 16]))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 7))
        Lmax = int(rng.integers(1, 3000))
        lens = rng.integers(0, Lmax + 1, size=B).astype(np.int32)
        if rng.random() < 0.3:
            lens[int(rng.integers(0, B))] = 0
        if rng.random() < 0.3:
            lens[int(rng.integers(0, B))] = Lmax
        out.append((base, i, B, Sq, G * Hkv, Hkv, Lmax, d, tuple(int(x) for x in lens)))
    return out


DEC = _decode_cases(14, SEED + 7, SEED) + _decode_cases(50, SEED_LARGE + 1, SEED_LARGE)


@pytest.mark.parametrize("case", DEC,
                         ids=[f"{c[0]}-b{c[2]}s{c[3]}h{c[4]}g{c[4] // c[5]}-L{c[6]}-d{c[7]}" for c in DEC])
def test_fuzz_decode(case):
    base, i, B, Sq, Hq, Hkv, Lmax, d, lens = case
    lens = np.array(lens, np.int32)
    seed = base + 300 + i
    scale = 1 / math.sqrt(d)
    kc = synthetic.kv_cache(seed, synthetic.TID_K, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)  # NaN past len
    vc = synthetic.kv_cache(seed, synthetic.TID_V, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    if Sq == 1:
        q = synthetic.tensor(seed, synthetic.TID_Q, (B, Hq, d))
        o, lse = run_decode(q, kc, vc, lens, scale)
        ro, rl = oracle.decode(q, kc, vc, lens, scale)
    else:
        q = synthetic.tensor(seed, synthetic.TID_Q, (B, Sq, Hq, d))
        o, lse = eio.attn_decode_multi(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(lens).cuda(),
                                       scale=scale)
        eio.sync_status()
        ro, rl = oracle_decode_multi(q, kc, vc, lens, scale)
    check(o, lse, ro, rl, f"decode {case}")


BWD = (_fwd_cases(10, SEED + 11, 400, [1, 2, 3, 4], ["none", "causal", "block"], SEED) +
       _fwd_cases(30, SEED_LARGE + 2, 700, [1, 2, 3, 4], ["none", "causal", "block"], SEED_LARGE))


@pytest.mark.parametrize("case", BWD, ids=_ids(BWD))
def test_fuzz_backward(case):
    base, i, B, Hq, Hkv, Nq, Nkv, d, kind = case
    B = min(B, 2)
    rng = np.random.default_rng(base + 3000 + i)
    q, k, v = make_inputs(base + 400 + i, B, Hq, Hkv, Nq, Nkv, d)
    dout = synthetic.tensor(base + 400 + i, 9, (B, Nq, Hq, d))
    mk, bm = _mask(kind, rng, Nq, Nkv)
    scale = 1 / math.sqrt(d)
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(dout)
    o, lse = eio.attn_fwd(tq, tk, tv, scale=scale, mask_kind=mk, block_map=bm)
    dq, dk, dv = eio.attn_bwd(tq, tk, tv, o, lse, tdo, scale=scale, mask_kind=mk, block_map=bm)
    eio.sync_status()
    rq, rk, rv = oracle.attn_bwd(q, k, v, dout, scale, mk, bm)
    check_grad(dq, rq, f"{case} dq")
    check_grad(dk, rk, f"{case} dk")
    check_grad(dv, rv, f"{case} dv")


BOUND = (_fwd_cases(8, SEED + 13, 600, [1, 2, 4, 8], ["none", "causal", "block"], SEED) +
         _fwd_cases(25, SEED_LARGE + 3, 1000, [1, 2, 4, 8], ["none", "causal", "block"], SEED_LARGE))


@pytest.mark.parametrize("case", BOUND, ids=_ids(BOUND))
def test_fuzz_bound_forward(case):
    base, i, B, Hq, Hkv, Nq, Nkv, d, kind = case
    rng = np.random.default_rng(base + 4000 + i)
    q, k, v = make_inputs(base + 500 + i, B, Hq, Hkv, Nq, Nkv, d)
    # keys offset by a random vector, so that the centring matters
    shift = rng.standard_normal(d).astype(np.float32)
    k = synthetic.f32_to_bf16_bits(synthetic.bf16_bits_to_f32(k) + shift)
    mk, bm = _mask(kind, rng, Nq, Nkv)
    scale = 1 / math.sqrt(d)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    kbar, radius = eio.key_stats(tk)
    rk, rr = oracle.key_stats(k)
    np.testing.assert_allclose(kbar.cpu().numpy(), rk, atol=2e-5, rtol=1e-5)
    np.testing.assert_allclose(radius.cpu().numpy(), rr, rtol=1e-5)
    nfb = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = eio.attn_fwd_bound(tq, tk, tv, kbar, radius, scale=scale, mask_kind=mk, block_map=bm, n_fallback=nfb)
    eio.sync_status()
    ro, rl = oracle.attn_fwd(q, k, v, scale, mk, bm)
    check(o, lse, ro, rl, f"bound {case}")
    _, _, flags = oracle.attn_fwd_bound(q, k, v, scale, mk, bm)
    assert int(nfb.item()) == int((flags == 0).sum())
