"""GPU parity: the CUDA library against the fp64 oracle, element by element.

Tolerances (fixed by the benchmark spec for bf16 inputs, applied to the fp32
case as well): O max-abs error <= 2e-2 and mean-abs error <= 2e-3, LSE within
1e-3; rows without any allowed key must give O = 0 and LSE = -inf exactly.
Small shapes and the five workloads at full size are compared on every
element of O and the LSE (the errors seen at full size are printed at the end
of the run), plus properties that hold at any size (determinism, masked keys
carry no weight, GQA == repeated MHA).
"""
import functools
import math

import numpy as np
import pytest
import torch

import exact_io_aware_sm_b200 as eio
import oracle
import synthetic
from conftest import record_parity

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from exact_io_aware_sm_b200 import build
    build.build()
    eio.lib()
    yield
    eio.sync_status()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def check(o_gpu, lse_gpu, o_ref, lse_ref, where="", log=False):
    o = host_f64(o_gpu).reshape(o_ref.shape)
    assert np.isfinite(o).all(), f"{where}: non-finite output"
    err = np.abs(o - o_ref)
    del o
    mx, mean = float(err.max()), float(err.mean())
    del err
    lmx = 0.0
    if lse_gpu is not None:
        lg = lse_gpu.cpu().numpy().astype(np.float64).reshape(lse_ref.shape)
        ninf = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lg), ninf), f"{where}: -inf LSE rows differ"
        if (~ninf).any():
            lmx = float(np.abs(lg[~ninf] - lse_ref[~ninf]).max())
    if log:
        record_parity(where, mx, mean, lmx, o_ref.size)
    assert mx <= O_MAX, f"{where}: O max-abs {mx:.3e}"
    assert mean <= O_MEAN, f"{where}: O mean-abs {mean:.3e}"
    assert lmx <= LSE_TOL, f"{where}: LSE err {lmx:.3e}"
    return mx, mean


def make_inputs(seed, B, Hq, Hkv, Nq, Nkv, d, dtype="bf16"):
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, Nq, Hq, d), dtype)
    k = synthetic.tensor(seed, synthetic.TID_K, (B, Nkv, Hkv, d), dtype)
    v = synthetic.tensor(seed, synthetic.TID_V, (B, Nkv, Hkv, d), dtype)
    return q, k, v


def run_fwd(q, k, v, scale, kind, bm):
    if q.dtype == np.uint16:
        tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    else:
        tq, tk, tv = (torch.from_numpy(x).cuda() for x in (q, k, v))
    o, lse = eio.attn_fwd(tq, tk, tv, scale=scale, mask_kind=kind, block_map=bm)
    eio.sync_status()
    return o, lse


def random_block_map(seed, Nq, Nkv, p=0.5):
    rng = np.random.default_rng(seed)
    return (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < p).astype(np.uint8)


SMALL = [
    # B, Hq, Hkv, Nq, Nkv, d, mask
    (1, 2, 2, 256, 256, 64, "none"),
    (1, 2, 2, 256, 256, 128, "none"),
    (2, 4, 4, 300, 300, 64, "causal"),
    (1, 8, 2, 517, 517, 128, "causal"),
    (1, 4, 1, 200, 333, 128, "causal"),
    (1, 2, 2, 333, 200, 64, "causal"),
    (1, 2, 2, 1, 1, 64, "none"),
    (1, 2, 1, 1, 77, 128, "none"),
    (3, 3, 3, 17, 5, 64, "none"),
    (2, 3, 1, 130, 257, 64, "none"),
    (1, 4, 2, 400, 300, 128, "block"),
    (2, 2, 2, 250, 250, 64, "block"),
    (1, 2, 2, 240, 240, 128, "frame48"),
    (1, 2, 2, 3120, 3120, 128, "frame1040"),
    (1, 2, 2, 3120, 3120, 64, "frame1040"),
    (2, 5, 5, 300, 300, 64, "causal"),   # d=64 head pairs, odd head count
    (1, 3, 3, 517, 700, 64, "causal"),
]


def mask_args(kind, Nq, Nkv, seed):
    """(mask kind, block map for the library, block map for the oracle): a
    frame map is built by each side on its own."""
    if kind == "none":
        return eio.MASK_NONE, None, None
    if kind == "causal":
        return eio.MASK_CAUSAL, None, None
    if kind == "block":
        bm = random_block_map(seed, Nq, Nkv, 0.45)
        return eio.MASK_BLOCK, bm, bm
    L = int(kind[len("frame"):])
    return eio.MASK_BLOCK, eio.frame_block_map(Nq // L, L), oracle.frame_block_map(Nq // L, L)


@pytest.mark.parametrize("case", SMALL, ids=[f"{c[-1]}-{c[3]}x{c[4]}-d{c[5]}-g{c[1]//c[2]}" for c in SMALL])
def test_prefill_small_all_elements(case):
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = 7000 + SMALL.index(case)
    q, k, v = make_inputs(seed, B, Hq, Hkv, Nq, Nkv, d)
    mk, bm, bm_ref = mask_args(kind, Nq, Nkv, seed)
    scale = 1 / math.sqrt(d)
    o, lse = run_fwd(q, k, v, scale, mk, bm)
    ro, rl = oracle.attn_fwd(q, k, v, scale, mk, bm_ref)
    check(o, lse, ro, rl, str(case))


def test_config1_tiny_fp32():
    """B=1, H=2, N=256, d=64, fp32 inputs, no mask (all elements)."""
    q, k, v = make_inputs(1001, 1, 2, 2, 256, 256, 64, "f32")
    o, lse = run_fwd(q, k, v, 1 / 8, eio.MASK_NONE, None)
    ro, rl = oracle.attn_fwd(q, k, v, 1 / 8, eio.MASK_NONE)
    mx, mean = check(o, lse, ro, rl, "config1 attn_fwd (fp32)", log=True)
    assert mx < 1e-5  # exact fp32 arithmetic


@pytest.mark.parametrize("case", [(2, 4, 4, 100, 100, 64, 0), (1, 4, 2, 64, 200, 128, 1),
                                  (1, 2, 1, 40, 40, 32, 2)])
def test_fp32_masks(case):
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    q, k, v = make_inputs(1100 + kind, B, Hq, Hkv, Nq, Nkv, d, "f32")
    bm = random_block_map(5, Nq, Nkv) if kind == 2 else None
    o, lse = run_fwd(q, k, v, 0.2, kind, bm)
    ro, rl = oracle.attn_fwd(q, k, v, 0.2, kind, bm)
    check(o, lse, ro, rl, str(case))


# The three bf16 prefill workloads at full size: inputs from their seeds, and
# the oracle's whole O and LSE (computed once per workload and shared by the
# tests below; the long-context one is about a minute of fp64 on 16 cores).
FULL = {
    "config2": dict(B=8, Hq=12, Hkv=12, N=1024, d=64, mask="causal", seed=1002),
    "config3": dict(B=1, Hq=32, Hkv=8, N=16384, d=128, mask="causal", seed=1003),
    "config4": dict(B=1, Hq=24, Hkv=24, N=24 * 1040, d=128, mask="frame", seed=1004),
}


def full_masks(name):
    """(kind, library block map, oracle block map): each side builds the frame map itself."""
    c = FULL[name]
    if c["mask"] == "causal":
        return eio.MASK_CAUSAL, None, None
    return eio.MASK_BLOCK, eio.frame_block_map(24, 1040), oracle.frame_block_map(24, 1040)


@functools.lru_cache(maxsize=None)
def full_inputs(name):
    c = FULL[name]
    return make_inputs(c["seed"], c["B"], c["Hq"], c["Hkv"], c["N"], c["N"], c["d"])


@functools.lru_cache(maxsize=None)
def full_reference(name):
    c = FULL[name]
    q, k, v = full_inputs(name)
    kind, _, obm = full_masks(name)
    return oracle.attn_fwd(q, k, v, 1 / math.sqrt(c["d"]), kind, obm)


@pytest.mark.parametrize("name", ["config2", "config3", "config4"])
def test_prefill_full_size_every_element(name):
    """GPT-2 causal (B=8, H=12, N=1024, d=64), long-context GQA causal (Hq=32,
    Hkv=8, N=16384, d=128) and frame block-sparse (24 heads, 24 x 1040 tokens,
    d=128): every element of O and of the LSE against the oracle, with the
    max-abs and mean-abs gates evaluated over the whole output."""
    c = FULL[name]
    q, k, v = full_inputs(name)
    kind, bm, _ = full_masks(name)
    o, lse = run_fwd(q, k, v, 1 / math.sqrt(c["d"]), kind, bm)
    ro, rl = full_reference(name)
    check(o, lse, ro, rl, f"{name} attn_fwd", log=True)


# ------------------------------------------------------------------ backward
# Gradients are bf16 outputs of products whose P and dS operands are rounded to
# bf16 (relative 2^-9 each) and D = rowsum(dO * O) uses the bf16 O of the
# forward; the bound is relative to each gradient's own scale.
GRAD_MAX_REL, GRAD_MEAN_REL = 2e-2, 1e-2


def check_grad(got, ref, where):
    g = host_f64(got).reshape(ref.shape)
    assert np.isfinite(g).all(), f"{where}: non-finite gradient"
    err = np.abs(g - ref)
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= GRAD_MAX_REL * scale_max + 1e-6, f"{where}: max err {err.max():.3e} vs {scale_max:.3e}"
    assert err.mean() <= GRAD_MEAN_REL * scale_mean + 1e-7, f"{where}: mean err {err.mean():.3e} vs {scale_mean:.3e}"


BWD_CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 2, 2, 128, 128, 64, False),
    (2, 4, 2, 200, 200, 128, True),
    (1, 4, 1, 77, 130, 64, True),
    (1, 2, 1, 130, 77, 128, True),   # rows that see no key
    (1, 3, 3, 300, 300, 128, False),
    (2, 8, 2, 64, 64, 64, True),
    (1, 4, 2, 400, 333, 64, True),    # several 128-row tiles, ragged, rows that see no key
    (1, 8, 2, 520, 520, 128, True),   # GQA group of 4 over five Q and KV tiles
    (2, 2, 2, 256, 384, 64, False),
]


@pytest.mark.parametrize("case", BWD_CASES)
def test_backward_small(case):
    B, Hq, Hkv, Nq, Nkv, d, causal = case
    seed = 3100 + BWD_CASES.index(case)
    q, k, v = make_inputs(seed, B, Hq, Hkv, Nq, Nkv, d)
    dout = synthetic.tensor(seed, 9, (B, Nq, Hq, d))
    kind = eio.MASK_CAUSAL if causal else eio.MASK_NONE
    scale = 1 / math.sqrt(d)
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(dout)
    o, lse = eio.attn_fwd(tq, tk, tv, scale=scale, mask_kind=kind)
    dq, dk, dv = eio.attn_bwd(tq, tk, tv, o, lse, tdo, scale=scale, mask_kind=kind)
    eio.sync_status()
    rq, rk, rv = oracle.attn_bwd(q, k, v, dout, scale, kind)
    check_grad(dq, rq, f"{case} dq")
    check_grad(dk, rk, f"{case} dk")
    check_grad(dv, rv, f"{case} dv")


BWD_BLOCK_CASES = [
    # B, Hq, Hkv, N, d, map
    (1, 2, 2, 300, 64, "random"),
    (2, 4, 2, 250, 128, "random"),
    (1, 2, 2, 480, 64, "frames"),  # 6 frames x 80 tokens: own, previous and first frame
]


@pytest.mark.parametrize("case", BWD_BLOCK_CASES)
def test_backward_block_mask(case):
    B, Hq, Hkv, N, d, kind = case
    seed = 3500 + BWD_BLOCK_CASES.index(case)
    q, k, v = make_inputs(seed, B, Hq, Hkv, N, N, d)
    dout = synthetic.tensor(seed, 9, (B, N, Hq, d))
    if kind == "frames":
        bm = eio.frame_block_map(6, 80)
    else:
        bm = random_block_map(seed, N, N, p=0.4)
        bm[3] = 0  # a block row with no key: its gradients are zero
    scale = 1 / math.sqrt(d)
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(dout)
    o, lse = eio.attn_fwd(tq, tk, tv, scale=scale, mask_kind=eio.MASK_BLOCK, block_map=bm)
    dq, dk, dv = eio.attn_bwd(tq, tk, tv, o, lse, tdo, scale=scale, mask_kind=eio.MASK_BLOCK, block_map=bm)
    eio.sync_status()
    rq, rk, rv = oracle.attn_bwd(q, k, v, dout, scale, oracle.MASK_BLOCK, bm)
    check_grad(dq, rq, f"{case} dq")
    check_grad(dk, rk, f"{case} dk")
    check_grad(dv, rv, f"{case} dv")


def test_backward_gpt2_shape_first_batch_element():
    B, H, N, d = 8, 12, 1024, 64
    q, k, v = make_inputs(1002, B, H, H, N, N, d)
    dout = synthetic.tensor(1002, 9, (B, N, H, d))
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(dout)
    o, lse = eio.attn_fwd(tq, tk, tv, mask_kind=eio.MASK_CAUSAL)
    dq, dk, dv = eio.attn_bwd(tq, tk, tv, o, lse, tdo, mask_kind=eio.MASK_CAUSAL)
    eio.sync_status()
    rq, rk, rv = oracle.attn_bwd(q[:1], k[:1], v[:1], dout[:1], 1 / math.sqrt(d), oracle.MASK_CAUSAL)
    check_grad(dq[:1], rq, "gpt2 dq")
    check_grad(dk[:1], rk, "gpt2 dk")
    check_grad(dv[:1], rv, "gpt2 dv")


# ------------------------------------------------------------------ decode
def run_decode(q, kc, vc, lens, scale):
    o, lse = eio.attn_decode(dev_bf16(q), dev_bf16(kc), dev_bf16(vc),
                             torch.from_numpy(np.asarray(lens, np.int32)).cuda(), scale=scale)
    eio.sync_status()
    return o, lse


DECODE_SMALL = [
    # B, Hq, Hkv, Lmax, d, lens
    (4, 8, 8, 600, 128, [1, 15, 16, 17]),
    (3, 8, 4, 1100, 128, [511, 512, 513]),
    (2, 16, 2, 2000, 128, [1025, 2000]),
    (2, 8, 1, 700, 64, [700, 3]),
    (5, 4, 2, 64, 64, [64, 1, 33, 2, 63]),
    (3, 8, 2, 1037, 128, [1037, 1000, 45]),
    (2, 4, 1, 37, 64, [37, 20]),
]


@pytest.mark.parametrize("case", DECODE_SMALL)
def test_decode_small(case):
    B, Hq, Hkv, Lmax, d, lens = case
    lens = np.array(lens, np.int32)
    seed = 2100 + DECODE_SMALL.index(case)
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, Hq, d))
    kc = synthetic.kv_cache(seed, synthetic.TID_K, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)  # NaN past len
    vc = synthetic.kv_cache(seed, synthetic.TID_V, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    o, lse = run_decode(q, kc, vc, lens, 1 / math.sqrt(d))
    ro, rl = oracle.decode(q, kc, vc, lens, 1 / math.sqrt(d))
    check(o, lse, ro, rl, str(case))


def oracle_decode_multi(q, kc, vc, lens, scale):
    """Sq newest tokens per sequence = the last Sq rows of a causal prefill
    with Nq = Sq, Nkv = len (bottom-right alignment)."""
    B, Sq, Hq, d = q.shape
    o = np.zeros((B, Sq, Hq, d))
    lse = np.full((B, Hq, Sq), -np.inf)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        ob, lb = oracle.attn_fwd(q[b:b + 1], kc[b:b + 1, :L], vc[b:b + 1, :L], scale, oracle.MASK_CAUSAL, None)
        o[b], lse[b] = ob[0], lb[0]
    return o, lse


DECODE_MULTI = [
    # B, Sq, Hq, Hkv, Lmax, d, lens
    (3, 2, 8, 2, 1100, 128, [1100, 513, 1]),
    (4, 4, 4, 2, 700, 64, [700, 3, 512, 2]),
    (2, 8, 2, 2, 600, 64, [600, 5]),
    (3, 2, 2, 1, 64, 128, [64, 0, 33]),
    # two groups of 8 MMA columns: (Hq/Hkv) * Sq in 9..16
    (3, 2, 16, 2, 1100, 128, [1100, 513, 1]),   # G = 8, MTP-2
    (2, 4, 8, 2, 700, 64, [700, 3]),            # G = 4, four tokens
    (2, 16, 2, 2, 600, 128, [600, 7]),          # G = 1, sixteen tokens, a sequence shorter than Sq
    (2, 3, 8, 2, 333, 64, [333, 2]),            # G = 4, three tokens: 12 live columns of 16
]


@pytest.mark.parametrize("case", DECODE_MULTI)
def test_decode_multi_token(case):
    B, Sq, Hq, Hkv, Lmax, d, lens = case
    lens = np.array(lens, np.int32)
    seed = 2300 + DECODE_MULTI.index(case)
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, Sq, Hq, d))
    kc = synthetic.kv_cache(seed, synthetic.TID_K, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)  # NaN past len
    vc = synthetic.kv_cache(seed, synthetic.TID_V, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    o, lse = eio.attn_decode_multi(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(lens).cuda(),
                                   scale=1 / math.sqrt(d))
    eio.sync_status()
    ro, rl = oracle_decode_multi(q, kc, vc, lens, 1 / math.sqrt(d))
    check(o, lse, ro, rl, str(case))


def test_binding_rejects_mis_shaped_tensors():
    """Outputs, statistics and lengths of the wrong shape, dtype or layout
    raise ValueError before any launch (the C ABI cannot see their sizes)."""
    B, N, H, d = 1, 64, 2, 64
    q = dev_bf16(synthetic.tensor(1, 1, (B, N, H, d)))
    with pytest.raises(ValueError, match="lse"):
        eio.attn_fwd(q, q, q, lse=torch.empty(B, H, N - 1, device="cuda"))
    with pytest.raises(ValueError, match="o has dtype"):
        eio.attn_fwd(q, q, q, o=torch.empty(B, N, H, d, device="cuda"))
    with pytest.raises(ValueError, match="contiguous"):
        eio.attn_fwd(q, q.transpose(1, 2).contiguous().transpose(1, 2), q)
    with pytest.raises(ValueError, match="k has shape"):
        eio.attn_fwd(q, q[..., :32].contiguous(), q)
    with pytest.raises(ValueError, match="kbar"):
        eio.key_stats(q, kbar=torch.empty(B, H, d + 1, device="cuda"))
    kbar, radius = eio.key_stats(q)
    with pytest.raises(ValueError, match="radius"):
        eio.attn_fwd_bound(q, q, q, kbar, radius.double())
    qd = q[:, 0].contiguous()
    with pytest.raises(ValueError, match="seqlens"):
        eio.attn_decode(qd, q, q, torch.full((B,), N, dtype=torch.int64, device="cuda"))
    with pytest.raises(ValueError, match="lse"):
        eio.attn_bwd(q, q, q, q, torch.empty(B, H, N, dtype=torch.float16, device="cuda"), q)
    eio.sync_status()


def test_decode_multi_equals_single_at_sq1():
    B, Hq, Hkv, Lmax, d = 4, 8, 2, 900, 128
    lens = np.array([900, 1, 511, 512], np.int32)
    q = synthetic.tensor(2400, synthetic.TID_Q, (B, Hq, d))
    kc = dev_bf16(synthetic.kv_cache(2400, synthetic.TID_K, B, Lmax, Hkv, d, lens))
    vc = dev_bf16(synthetic.kv_cache(2400, synthetic.TID_V, B, Lmax, Hkv, d, lens))
    tl = torch.from_numpy(lens).cuda()
    o1, l1 = eio.attn_decode(dev_bf16(q), kc, vc, tl)
    o2, l2 = eio.attn_decode_multi(dev_bf16(q).reshape(B, 1, Hq, d), kc, vc, tl)
    eio.sync_status()
    assert torch.equal(o1, o2.reshape(B, Hq, d)) and torch.equal(l1, l2.reshape(B, Hq))


@pytest.mark.parametrize("Sq,Hq", [(2, 32), (2, 64)], ids=["G4-mtp2", "G8-mtp2"])
def test_decode_multi_full_size_mtp2(Sq, Hq):
    """The decode workload (64 sequences, lengths U[1024, 8192], 8 KV heads,
    d = 128) with two new tokens per sequence, every element against the
    oracle's causal prefill; with 64 query heads (G = 8) the 16 (head, token)
    pairs of a KV group fill two groups of MMA columns."""
    B, Hkv, Lmax, d = 64, 8, 8192, 128
    lens = synthetic.seqlens(2005, B)
    q = synthetic.tensor(1005, synthetic.TID_Q, (B, Sq, Hq, d))
    kc = synthetic.kv_cache(1005, synthetic.TID_K, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    vc = synthetic.kv_cache(1005, synthetic.TID_V, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    o, lse = eio.attn_decode_multi(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(lens).cuda())
    eio.sync_status()
    ro, rl = oracle_decode_multi(q, kc, vc, lens, 1 / math.sqrt(d))
    check(o, lse, ro, rl, f"attn_decode_multi Sq={Sq} Hq={Hq} full size", log=True)


def test_decode_more_sequences_than_one_launch_holds():
    # more than 2048 sequences: the split kernel runs in sequence groups
    B, Hq, Hkv, Lmax, d = 2100, 4, 2, 40, 64
    lens = (np.arange(B, dtype=np.int64) * 7919 % 41).astype(np.int32)  # 0..40, zeros included
    q = synthetic.tensor(2200, synthetic.TID_Q, (B, Hq, d))
    kc = synthetic.kv_cache(2200, synthetic.TID_K, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    vc = synthetic.kv_cache(2200, synthetic.TID_V, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    o, lse = run_decode(q, kc, vc, lens, 0.125)
    ro, rl = oracle.decode(q, kc, vc, lens, 0.125)
    check(o, lse, ro, rl, "B=2100")


def test_decode_zero_length_and_bad_length():
    B, Hq, Hkv, Lmax, d = 3, 4, 4, 64, 128
    q = synthetic.tensor(5, 1, (B, Hq, d))
    lens = np.array([0, 64, 5], np.int32)
    kc = synthetic.kv_cache(5, 2, B, Lmax, Hkv, d, lens)
    vc = synthetic.kv_cache(5, 3, B, Lmax, Hkv, d, lens)
    o, lse = run_decode(q, kc, vc, lens, 0.1)
    ro, rl = oracle.decode(q, kc, vc, lens, 0.1)
    check(o, lse, ro, rl, "zero-length")
    # a length above Lmax is latched as a device argument error; that row reads nothing
    bad = np.array([3, 65, 5], np.int32)
    o2, l2 = eio.attn_decode(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(bad).cuda(), scale=0.1)
    with pytest.raises(eio.AttnError) as ei:
        eio.sync_status()
    assert ei.value.code == 9
    assert torch.all(o2[1].float() == 0) and torch.isneginf(l2[1]).all()
    eio.sync_status()  # cleared


def test_device_timeout_is_latched_and_context_recovers():
    # The hook makes CTA 0 skip one K tile copy, so the MMA issuer's bounded
    # wait on that stage runs out; the kernel must stop by itself, latch
    # ATTN_ERR_DEVICE_TIMEOUT and leave the context usable.
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 128
    q, k, v = make_inputs(77, B, Hq, Hkv, N, N, d)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    eio.debug_fault(1)
    eio.attn_fwd(tq, tk, tv, scale=0.088, mask_kind=eio.MASK_CAUSAL)
    with pytest.raises(eio.AttnError) as ei:
        eio.sync_status()
    assert ei.value.code == 7
    eio.sync_status()  # the error word was cleared
    o, lse = run_fwd(q, k, v, 0.088, eio.MASK_CAUSAL, None)
    ro, rl = oracle.attn_fwd(q, k, v, 0.088, eio.MASK_CAUSAL, None)
    check(o, lse, ro, rl, "after time-out")


def test_config5_gqa_decode_full_size():
    B, Hq, Hkv, Lmax, d = 64, 32, 8, 8192, 128
    lens = synthetic.seqlens(2005, B)
    q = synthetic.tensor(1005, synthetic.TID_Q, (B, Hq, d))
    kc = synthetic.kv_cache(1005, synthetic.TID_K, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    vc = synthetic.kv_cache(1005, synthetic.TID_V, B, Lmax, Hkv, d, lens, fill_bits=0x7FC0)
    o, lse = run_decode(q, kc, vc, lens, 1 / math.sqrt(d))
    ro, rl = oracle.decode(q, kc, vc, lens, 1 / math.sqrt(d))
    check(o, lse, ro, rl, "config5 attn_decode", log=True)


# ------------------------------------------------------------------ properties
def test_masked_keys_carry_no_weight_bitwise():
    """Causal: keys a row must not see changed to 1e4 -> bit-identical output.
    Block map: keys in blocks no query may see set to NaN (never loaded)."""
    B, H, N, d = 1, 2, 384, 128
    q, k, v = make_inputs(31, B, H, H, N, N, d)
    o1, l1 = run_fwd(q, k, v, 0.09, eio.MASK_CAUSAL, None)
    k2, v2 = k.copy(), v.copy()
    big = synthetic.f32_to_bf16_bits(np.float32([1e4, -1e4]))
    k2[0, 200:] = big[0]
    v2[0, 200:] = big[1]
    # rows < 200 cannot see keys >= 200
    o2, l2 = run_fwd(q, k2, v2, 0.09, eio.MASK_CAUSAL, None)
    assert torch.equal(o1[:, :200], o2[:, :200]) and torch.equal(l1[:, :, :200], l2[:, :, :200])

    bm = np.ones((N // 16, N // 16), np.uint8)
    bm[:, 5:9] = 0  # key blocks 5..8 seen by nobody
    o3, l3 = run_fwd(q, k, v, 0.09, eio.MASK_BLOCK, bm)
    k3, v3 = k.copy(), v.copy()
    k3[0, 80:144] = 0x7FC0
    v3[0, 80:144] = 0x7FC0
    o4, l4 = run_fwd(q, k3, v3, 0.09, eio.MASK_BLOCK, bm)
    assert torch.equal(o3, o4) and torch.equal(l3, l4)


def test_deterministic():
    q, k, v = make_inputs(41, 2, 4, 2, 700, 700, 128)
    a = run_fwd(q, k, v, 0.1, eio.MASK_CAUSAL, None)
    b = run_fwd(q, k, v, 0.1, eio.MASK_CAUSAL, None)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_gqa_equals_repeated_mha_bitwise():
    q, k, v = make_inputs(51, 1, 8, 2, 300, 300, 64)
    o1, l1 = run_fwd(q, k, v, 0.12, eio.MASK_CAUSAL, None)
    kr, vr = np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2)
    o2, l2 = run_fwd(q, kr, vr, 0.12, eio.MASK_CAUSAL, None)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_constant_v_rows():
    B, H, N, d = 1, 2, 300, 128
    q, k, _ = make_inputs(61, B, H, H, N, N, d)
    c = synthetic.normal(62, 1, d)
    v = np.broadcast_to(c, (B, N, H, d)).copy()
    o, _ = run_fwd(q, k, v, 0.1, eio.MASK_CAUSAL, None)
    cf = synthetic.bf16_bits_to_f32(c).astype(np.float64)
    err = np.abs(host_f64(o) - cf).max()
    assert err <= 8e-3 * max(1.0, np.abs(cf).max())


# ------------------------------------------------------- bound-based softmax
BOUND_CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, kind
    (2, 4, 2, 300, 300, 64, eio.MASK_CAUSAL),
    (1, 8, 2, 257, 513, 128, eio.MASK_NONE),
    (1, 4, 4, 200, 200, 64, eio.MASK_BLOCK),
    (1, 2, 1, 130, 77, 128, eio.MASK_CAUSAL),  # rows that see no key
]


@pytest.mark.parametrize("case", BOUND_CASES)
def test_key_stats_and_bound_forward(case):
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = 3300 + BOUND_CASES.index(case)
    q, k, v = make_inputs(seed, B, Hq, Hkv, Nq, Nkv, d)
    # an offset on the keys, so that the centring matters
    kf = synthetic.bf16_bits_to_f32(k) + np.float32(0.75)
    k = synthetic.f32_to_bf16_bits(kf)
    bm = random_block_map(seed, Nq, Nkv) if kind == eio.MASK_BLOCK else None
    scale = 1 / math.sqrt(d)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    kbar, radius = eio.key_stats(tk)
    rk, rr = oracle.key_stats(k)
    np.testing.assert_allclose(kbar.cpu().numpy(), rk, atol=2e-5, rtol=1e-5)
    np.testing.assert_allclose(radius.cpu().numpy(), rr, rtol=1e-5)
    nfb = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = eio.attn_fwd_bound(tq, tk, tv, kbar, radius, scale=scale, mask_kind=kind, block_map=bm, n_fallback=nfb)
    eio.sync_status()
    ro, rlse = oracle.attn_fwd(q, k, v, scale, kind, bm)
    check(o, lse, ro, rlse, f"bound {case}")
    _, _, flags = oracle.attn_fwd_bound(q, k, v, scale, kind, bm)
    assert int(nfb.item()) == int((flags == 0).sum()) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_key_stats_repeatable_and_reset_on_every_call(d):
    """The chunk sums are added in a fixed order, so repeated calls agree bit
    for bit; the radius starts from zero on every call, so statistics of wide
    keys followed by narrow keys into the same buffers give the narrow keys'
    radius.  129 chunks: not a multiple of the mean's eight runs."""
    B, Hkv, N = 2, 3, 128 * 128 + 77
    _, k, _ = make_inputs(3500 + d, B, Hkv, Hkv, 1, N, d)
    kf = synthetic.bf16_bits_to_f32(k) + np.float32(0.5)
    k = synthetic.f32_to_bf16_bits(kf)
    wide = synthetic.f32_to_bf16_bits(kf * np.float32(8.0))
    kbar = torch.empty((B, Hkv, d), dtype=torch.float32, device="cuda")
    radius = torch.empty((B, Hkv), dtype=torch.float32, device="cuda")
    eio.key_stats(dev_bf16(wide), kbar=kbar, radius=radius)
    r_wide = radius.clone()
    tk = dev_bf16(k)
    eio.key_stats(tk, kbar=kbar, radius=radius)
    kb1, r1 = kbar.clone(), radius.clone()
    kb2, r2 = eio.key_stats(tk)
    eio.sync_status()
    assert torch.equal(kb1, kb2) and torch.equal(r1, r2)
    assert (r1 < r_wide).all()
    rk, rr = oracle.key_stats(k)
    np.testing.assert_allclose(kb1.cpu().numpy(), rk, atol=2e-5, rtol=1e-5)
    np.testing.assert_allclose(r1.cpu().numpy(), rr, rtol=1e-5)


def test_bound_forward_falls_back_on_long_queries():
    """Every fifth query 40x longer: those rows' bounds exceed the limit and
    keep the running max; the count matches the oracle's and O is exact."""
    B, Hq, Hkv, N, d = 1, 4, 2, 320, 64
    q, k, v = make_inputs(3350, B, Hq, Hkv, N, N, d)
    qf = synthetic.bf16_bits_to_f32(q)
    qf[:, ::5] *= np.float32(40.0)
    q = synthetic.f32_to_bf16_bits(qf)
    scale = 1 / math.sqrt(d)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    kbar, radius = eio.key_stats(tk)
    nfb = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = eio.attn_fwd_bound(tq, tk, tv, kbar, radius, scale=scale, mask_kind=eio.MASK_CAUSAL, n_fallback=nfb)
    eio.sync_status()
    ro, rlse, flags = oracle.attn_fwd_bound(q, k, v, scale, oracle.MASK_CAUSAL)
    # the decision is far from the limit on both sides (about 32 and 1270 log2 units)
    assert int(nfb.item()) == int((flags == 0).sum()) == B * Hq * (N // 5)
    rq = oracle.attn_fwd(q, k, v, scale, oracle.MASK_CAUSAL)
    np.testing.assert_allclose(ro, rq[0], atol=1e-10)
    # long rows have sharp softmaxes: compare with the forward tolerance
    check(o, lse, ro, rlse, "bound with fallback rows")


def test_bound_forward_matches_online_forward_gpt2_shape():
    """The similarity band between the bound-based and the online forward on
    the GPT-2 workload shape: same result up to rounding."""
    B, H, N, d = 8, 12, 1024, 64
    q, k, v = make_inputs(1002, B, H, H, N, N, d)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    o0, l0 = eio.attn_fwd(tq, tk, tv, mask_kind=eio.MASK_CAUSAL)
    kbar, radius = eio.key_stats(tk)
    nfb = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = eio.attn_fwd_bound(tq, tk, tv, kbar, radius, mask_kind=eio.MASK_CAUSAL, n_fallback=nfb)
    eio.sync_status()
    assert int(nfb.item()) == 0
    a, b = o0.float(), o1.float()
    assert (a - b).abs().max().item() <= 2e-2
    cos = torch.nn.functional.cosine_similarity(a.reshape(-1, d), b.reshape(-1, d), dim=1)
    assert cos.min().item() > 0.9999
    assert (l0 - l1).abs().max().item() <= 1e-3
    rows = np.array([[0, 0, 0], [3, 7, 511], [7, 11, 1023], [5, 2, 1]], np.int32)
    ro, rlse = oracle.attn_rows(q, k, v, 1 / math.sqrt(d), rows, oracle.MASK_CAUSAL)
    got = np.stack([host_f64(o1[b_, i, h]) for b_, h, i in rows])
    assert np.abs(got - ro).max() <= O_MAX


def test_ulysses_single_rank_uses_the_cuda_forward():
    """Without a process group (one rank) the Ulysses entry is the CUDA
    forward itself: bit-identical to attn_fwd."""
    from exact_io_aware_sm_b200.ulysses import ulysses_attention
    q, k, v = make_inputs(3400, 1, 4, 2, 200, 200, 64)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    o0, l0 = eio.attn_fwd(tq, tk, tv, mask_kind=eio.MASK_CAUSAL)
    o1, l1 = ulysses_attention(tq, tk, tv, mask_kind=eio.MASK_CAUSAL)
    eio.sync_status()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


BWD_FULL = [
    # B, Hq, Hkv, N, d, mask: the GQA causal backward shape and the frame workload at full size
    (1, 32, 8, 4096, 128, "causal"),
    (1, 24, 24, 24960, 128, "frames"),
]


@pytest.mark.parametrize("case", BWD_FULL)
def test_backward_full_size_sampled_rows_and_identities(case):
    """At full size: dQ on sampled query rows against the oracle's per-row
    dQ, and two identities over all keys that hold at any size: every row's
    probabilities sum to one, so sum_j dV_j equals the sum of dO over the
    rows and query heads of the group; every row's dS sums to zero, so
    sum_j dK_j = 0 (both per batch element, KV head and column)."""
    B, Hq, Hkv, N, d, kind = case
    seed = 3600 + BWD_FULL.index(case)
    q, k, v = make_inputs(seed, B, Hq, Hkv, N, N, d)
    dout = synthetic.tensor(seed, 9, (B, N, Hq, d))
    mk, bm = (eio.MASK_CAUSAL, None) if kind == "causal" else (eio.MASK_BLOCK, eio.frame_block_map(24, 1040))
    scale = 1 / math.sqrt(d)
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(dout)
    o, lse = eio.attn_fwd(tq, tk, tv, scale=scale, mask_kind=mk, block_map=bm)
    dq, dk, dv = eio.attn_bwd(tq, tk, tv, o, lse, tdo, scale=scale, mask_kind=mk, block_map=bm)
    eio.sync_status()
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, B, 16), rng.integers(0, Hq, 16), rng.integers(0, N, 16)], axis=1).astype(np.int32)
    rows[0] = (0, 0, 0)
    rows[1] = (B - 1, Hq - 1, N - 1)
    ref = oracle.attn_bwd_dq_rows(q, k, v, dout, scale, rows, mk, bm)
    got = np.stack([host_f64(dq[b, i, h]) for b, h, i in rows])
    check_grad(torch.from_numpy(got), ref, f"{case} dq rows")
    G = Hq // Hkv
    do64 = synthetic.bf16_bits_to_f32(dout).astype(np.float64).reshape(B, N, Hkv, G, d)
    want_dv = do64.sum(axis=(1, 3))                      # [B, Hkv, d]
    dv64, dk64 = host_f64(dv), host_f64(dk)
    err_v = np.abs(dv64.sum(axis=1) - want_dv)
    assert (err_v <= 4e-3 * np.abs(dv64).sum(axis=1) + 1e-3).all(), err_v.max()
    err_k = np.abs(dk64.sum(axis=1))
    assert (err_k <= 4e-3 * np.abs(dk64).sum(axis=1) + 1e-3).all(), err_k.max()


@pytest.mark.parametrize("name", ["config3", "config4"])
def test_bound_forward_full_size_d128(name):
    """The bound-based forward (key statistics + attn_fwd_bound) on the two
    d = 128 workloads at full size, every element of O and the LSE against
    the oracle's plain definition; no row needs the fallback on these inputs
    (the oracle's rule agrees)."""
    c = FULL[name]
    q, k, v = full_inputs(name)
    kind, bm, _ = full_masks(name)
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    kbar, radius = eio.key_stats(tk)
    nfb = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = eio.attn_fwd_bound(tq, tk, tv, kbar, radius, mask_kind=kind, block_map=bm, n_fallback=nfb)
    eio.sync_status()
    assert int(nfb.item()) == 0
    rk, rr = oracle.key_stats(k)
    np.testing.assert_allclose(kbar.cpu().numpy(), rk, atol=2e-5, rtol=1e-5)
    np.testing.assert_allclose(radius.cpu().numpy(), rr, rtol=1e-5)
    del tq, tk, tv
    ro, rl = full_reference(name)
    check(o, lse, ro, rl, f"{name} attn_fwd_bound", log=True)
