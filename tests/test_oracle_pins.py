"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: the pages'
printed worked examples, a library routine (torch SDPA / logsumexp in fp64),
exact arithmetic on tiny inputs, closed forms and invariants.  A plausible
slip in the oracle (a dropped term, a wrong sign, a transposed operand, a
wrong GQA index) fails at least one of them.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.conftest import read_golden


def rnd(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


# --------------------------------------------------------------------------
# Online softmax: the pages' worked examples
# --------------------------------------------------------------------------

def _check_golden_online(name):
    g = read_golden(name)
    tol = 0.5 * 10 ** (-int(g["decimals"])) + 1e-12
    r = oracle.online_softmax(g["x"], [int(b) for b in g["bounds"]])
    for key in ("m_blk", "l_blk", "m_run", "l_run"):
        np.testing.assert_allclose(r[key], g[key], atol=tol, rtol=0, err_msg=key)
    if "resc" in g:
        np.testing.assert_allclose(r["resc"], g["resc"], atol=tol, rtol=0)
    # the rescaled previous sum (second block merged onto the first)
    np.testing.assert_allclose(r["l_run"][0] * math.exp(r["m_run"][0] - r["m_run"][1]),
                               g["resc_times_l_prev"], atol=tol, rtol=0)
    x = np.array(g["x"])
    np.testing.assert_allclose(np.exp(x - x.max()).sum(), g["full_sum"], atol=tol, rtol=0)
    if "full_terms" in g:
        np.testing.assert_allclose(np.exp(x - g["full_max"]), g["full_terms"], atol=tol, rtol=0)


def test_online_softmax_flashattention_page_example():
    _check_golden_online("online_softmax_flashattention_sec2.txt")


def test_online_softmax_inference_page_example():
    _check_golden_online("online_softmax_inference_example.txt")


@pytest.mark.parametrize("seed", range(6))
def test_online_softmax_blockwise_equals_one_shot(seed):
    """Block-wise statistics merged over any split equal the one-shot max and
    sum (the exactness claim, Theorem 1 of the FlashAttention page, for the
    softmax normaliser)."""
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    x = rng.standard_normal(n) * rng.uniform(0.1, 30)
    cuts = np.sort(rng.choice(np.arange(1, n), size=min(n - 1, int(rng.integers(0, 12))), replace=False)) if n > 1 else []
    bounds = [0, *[int(c) for c in cuts], n]
    r = oracle.online_softmax(x, bounds)
    m = x.max()
    assert r["m_run"][-1] == m
    np.testing.assert_allclose(r["l_run"][-1], np.exp(x - m).sum(), rtol=1e-13)


# --------------------------------------------------------------------------
# Whole oracle vs a library routine (torch SDPA, math path, fp64 CPU)
# --------------------------------------------------------------------------

def _sdpa_ref(q, k, v, scale, allowed):
    """torch SDPA on [B,N,H,d] inputs with a boolean [Nq,Nkv] mask; GQA via
    torch's own enable_gqa head mapping.  LSE via torch.logsumexp."""
    Q = torch.from_numpy(q).permute(0, 2, 1, 3)
    K = torch.from_numpy(k).permute(0, 2, 1, 3)
    V = torch.from_numpy(v).permute(0, 2, 1, 3)
    M = torch.from_numpy(allowed)
    G = Q.shape[1] // K.shape[1]
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=M, scale=scale,
                                                         enable_gqa=G > 1)
    Kr = K.repeat_interleave(G, dim=1)
    logits = torch.matmul(Q, Kr.transpose(-1, -2)) * scale
    logits = logits.masked_fill(~M, float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)
    return O.permute(0, 2, 1, 3).numpy(), lse.numpy()


def _allowed_matrix(kind, bm, Nq, Nkv):
    i = np.arange(Nq)[:, None]
    j = np.arange(Nkv)[None, :]
    if kind == oracle.MASK_NONE:
        return np.ones((Nq, Nkv), bool)
    if kind == oracle.MASK_CAUSAL:
        return j <= i + (Nkv - Nq)
    return bm[i // 16, j // 16].astype(bool)


CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, kind
    (1, 2, 2, 7, 7, 4, oracle.MASK_NONE),
    (2, 4, 2, 33, 33, 16, oracle.MASK_CAUSAL),
    (1, 4, 1, 20, 45, 8, oracle.MASK_CAUSAL),
    (1, 6, 3, 64, 64, 32, oracle.MASK_BLOCK),
    (2, 2, 1, 50, 40, 8, oracle.MASK_BLOCK),
    (1, 8, 2, 17, 64, 64, oracle.MASK_NONE),
]


@pytest.mark.parametrize("case", CASES)
def test_oracle_matches_torch_sdpa(case):
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = hash(case) & 0xFFFF
    q, k, v = rnd((B, Nq, Hq, d), seed), rnd((B, Nkv, Hkv, d), seed + 1), rnd((B, Nkv, Hkv, d), seed + 2)
    bm = None
    if kind == oracle.MASK_BLOCK:
        rng = np.random.default_rng(seed)
        bm = (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < 0.6).astype(np.uint8)
        bm[:, 0] = 1  # every row keeps at least one key for SDPA's sake
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(q, k, v, scale, kind, bm)
    allowed = _allowed_matrix(kind, bm, Nq, Nkv)
    if kind == oracle.MASK_CAUSAL and Nq > Nkv:
        pytest.skip("rows without keys are pinned separately")
    ro, rlse = _sdpa_ref(q, k, v, scale, allowed)
    np.testing.assert_allclose(o, ro, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, rlse, atol=1e-12, rtol=1e-12)


def test_oracle_rows_equals_full():
    B, Hq, Hkv, Nq, Nkv, d = 2, 4, 2, 40, 40, 16
    q, k, v = rnd((B, Nq, Hq, d), 5), rnd((B, Nkv, Hkv, d), 6), rnd((B, Nkv, Hkv, d), 7)
    o, lse = oracle.attn_fwd(q, k, v, 0.25, oracle.MASK_CAUSAL)
    rows = np.array([(1, 3, 39), (0, 0, 0), (1, 2, 17), (0, 1, 5)])
    ro, rl = oracle.attn_rows(q, k, v, 0.25, rows, oracle.MASK_CAUSAL)
    for n, (b, h, i) in enumerate(rows):
        assert np.array_equal(ro[n], o[b, i, h])
        assert rl[n] == lse[b, h, i]


def test_oracle_bf16_input_reading():
    """bf16 bit patterns are read as the exact values they encode."""
    x = synthetic.normal(3, 1, 64 * 4, "bf16").reshape(1, 16, 4, 4)
    xf = synthetic.bf16_bits_to_f32(x).reshape(x.shape).astype(np.float64)
    o1, l1 = oracle.attn_fwd(x, x, x, 0.5, oracle.MASK_CAUSAL)
    o2, l2 = oracle.attn_fwd(xf, xf, xf, 0.5, oracle.MASK_CAUSAL)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # a few exact bf16 values
    bits = np.array([0x3F80, 0xC000, 0x3E00, 0x0000], np.uint16)
    np.testing.assert_array_equal(synthetic.bf16_bits_to_f32(bits), [1.0, -2.0, 0.125, 0.0])


# --------------------------------------------------------------------------
# Brute force with exact arithmetic on tiny inputs
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(4))
def test_oracle_vs_exact_decimal(seed):
    """N <= 8, d <= 4, inputs on a dyadic grid so the logits are exact; the
    softmax is then evaluated with 50-digit decimals."""
    getcontext().prec = 50
    rng = np.random.default_rng(100 + seed)
    Nq, Nkv, d = int(rng.integers(1, 9)), int(rng.integers(1, 9)), int(rng.integers(1, 5))
    q = rng.integers(-4, 5, (1, Nq, 1, d)) / 4.0
    k = rng.integers(-4, 5, (1, Nkv, 1, d)) / 4.0
    v = rng.integers(-4, 5, (1, Nkv, 1, d)) / 4.0
    scale = 0.5
    o, lse = oracle.attn_fwd(q, k, v, scale, oracle.MASK_NONE)
    for i in range(Nq):
        logits = [Decimal(float(scale * sum(q[0, i, 0, t] * k[0, j, 0, t] for t in range(d))))
                  for j in range(Nkv)]
        w = [x.exp() for x in logits]
        Z = sum(w)
        for t in range(d):
            ref = sum(w[j] * Decimal(float(v[0, j, 0, t])) for j in range(Nkv)) / Z
            assert abs(float(ref) - o[0, i, 0, t]) < 1e-14
        assert abs(float(Z.ln()) - lse[0, 0, i]) < 1e-14


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

def test_constant_v_rows_reproduce_v():
    B, H, N, d = 1, 2, 50, 8
    q, k = rnd((B, N, H, d), 1), rnd((B, N, H, d), 2)
    c = rnd((d,), 3)
    v = np.broadcast_to(c, (B, N, H, d)).copy()
    for kind in (oracle.MASK_NONE, oracle.MASK_CAUSAL):
        o, _ = oracle.attn_fwd(q, k, v, 0.3, kind)
        np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=1e-14, atol=1e-15)


def test_key_shift_invariance():
    """Softmax is unchanged by a per-row constant shift: replacing every key
    k_j by k_j - u shifts each logit of row i by -scale*q_i.u, so O is
    unchanged and LSE moves by exactly that amount (mean-centring of keys,
    TPU attention guide, step 4)."""
    B, H, N, d = 1, 3, 40, 16
    q, k, v = rnd((B, N, H, d), 11), rnd((B, N, H, d), 12), rnd((B, N, H, d), 13)
    u = rnd((d,), 14) * 3
    scale = 0.25
    o1, l1 = oracle.attn_fwd(q, k, v, scale, oracle.MASK_CAUSAL)
    o2, l2 = oracle.attn_fwd(q, k - u, v, scale, oracle.MASK_CAUSAL)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    shift = scale * np.einsum("bihd,d->bhi", q, u)
    np.testing.assert_allclose(l2, l1 - shift, rtol=1e-11, atol=1e-11)


def test_dominant_logit_selects_its_row():
    B, H, N, d = 1, 1, 30, 8
    rng = np.random.default_rng(21)
    q = rng.standard_normal((B, N, H, d)) * 0.1
    k = rng.standard_normal((B, N, H, d)) * 0.1
    v = rng.standard_normal((B, N, H, d))
    jstar = 17
    q[0, :, 0, 0] = 10.0
    k[0, jstar, 0, 0] = 10.0  # logit for jstar is ~100*scale above the rest
    scale = 0.5
    o, lse = oracle.attn_fwd(q, k, v, scale, oracle.MASK_NONE)
    for i in range(N):
        np.testing.assert_allclose(o[0, i, 0], v[0, jstar, 0], rtol=1e-12, atol=1e-12)
        logit = scale * float(q[0, i, 0] @ k[0, jstar, 0])
        np.testing.assert_allclose(lse[0, 0, i], logit, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", [oracle.MASK_CAUSAL, oracle.MASK_BLOCK])
def test_masked_keys_have_zero_weight(kind):
    """Changing K/V at masked keys to huge finite values changes nothing."""
    B, H, N, d = 1, 2, 48, 8
    q, k, v = rnd((B, N, H, d), 31), rnd((B, N, H, d), 32), rnd((B, N, H, d), 33)
    bm = None
    if kind == oracle.MASK_BLOCK:
        bm = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 0]], np.uint8)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.3, kind, bm)
    allowed = _allowed_matrix(kind, bm, N, N)
    k2, v2 = k.copy(), v.copy()
    i = 5  # poison every key row 5 cannot see
    for j in range(N):
        if not allowed[i, j]:
            k2[0, j] = 1e4
            v2[0, j] = -1e4
    r1 = oracle.attn_rows(q, k, v, 0.3, [(0, h, i) for h in range(H)], kind, bm)
    r2 = oracle.attn_rows(q, k2, v2, 0.3, [(0, h, i) for h in range(H)], kind, bm)
    assert np.array_equal(r1[0], r2[0]) and np.array_equal(r1[1], r2[1])


def test_row_without_keys():
    """A row whose every key is masked gives O = 0, LSE = -inf."""
    q, k, v = rnd((1, 20, 1, 4), 41), rnd((1, 10, 1, 4), 42), rnd((1, 10, 1, 4), 43)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, oracle.MASK_CAUSAL)  # off = -10: rows 0..9 see nothing
    assert np.all(o[0, :10] == 0) and np.all(np.isneginf(lse[0, 0, :10]))
    assert np.all(np.isfinite(lse[0, 0, 10:]))


def test_gqa_equals_mha_with_repeated_kv():
    """Contiguous groups (inference page, GQA mapping diagram): query head h
    uses KV head h // (Hq/Hkv)."""
    B, Hq, Hkv, N, d = 2, 8, 2, 24, 8
    q, k, v = rnd((B, N, Hq, d), 51), rnd((B, N, Hkv, d), 52), rnd((B, N, Hkv, d), 53)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.3, oracle.MASK_CAUSAL)
    kr, vr = np.repeat(k, Hq // Hkv, axis=2), np.repeat(v, Hq // Hkv, axis=2)
    o2, l2 = oracle.attn_fwd(q, kr, vr, 0.3, oracle.MASK_CAUSAL)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # and the mapping is not the modulo one: head 1 must differ from head 1 of a mod mapping
    kmod, vmod = np.tile(k, (1, 1, Hq // Hkv, 1)), np.tile(v, (1, 1, Hq // Hkv, 1))
    o3, _ = oracle.attn_fwd(q, kmod, vmod, 0.3, oracle.MASK_CAUSAL)
    assert not np.allclose(o1[:, :, 1], o3[:, :, 1])


def test_causal_row_zero_closed_form():
    B, H, N, d = 2, 2, 16, 8
    q, k, v = rnd((B, N, H, d), 61), rnd((B, N, H, d), 62), rnd((B, N, H, d), 63)
    scale = 0.35
    o, lse = oracle.attn_fwd(q, k, v, scale, oracle.MASK_CAUSAL)
    for b in range(B):
        for h in range(H):
            assert np.array_equal(o[b, 0, h], v[b, 0, h])
            np.testing.assert_allclose(lse[b, h, 0], scale * float(q[b, 0, h] @ k[b, 0, h]), rtol=1e-15, atol=1e-15)


def test_decode_equals_last_causal_row():
    """Decode step (inference page, section "Decode"): the newest query over
    the whole cache equals the last row of a causal prefill of that length."""
    B, Hq, Hkv, Lmax, d = 3, 4, 2, 40, 16
    lens = np.array([40, 1, 23], np.int32)
    kc, vc = rnd((B, Lmax, Hkv, d), 71), rnd((B, Lmax, Hkv, d), 72)
    qd = rnd((B, Hq, d), 73)
    o, lse = oracle.decode(qd, kc, vc, lens, 0.25)
    for b in range(B):
        L = int(lens[b])
        qp = rnd((1, L, Hq, d), 74)
        qp[0, L - 1] = qd[b]
        op, lp = oracle.attn_fwd(qp, kc[b:b + 1, :L], vc[b:b + 1, :L], 0.25, oracle.MASK_CAUSAL)
        np.testing.assert_allclose(o[b], op[0, L - 1], rtol=1e-15, atol=1e-15)
        np.testing.assert_allclose(lse[b], lp[0, :, L - 1], rtol=1e-15, atol=1e-15)


def test_decode_zero_length():
    o, lse = oracle.decode(rnd((1, 2, 4), 1), rnd((1, 8, 1, 4), 2), rnd((1, 8, 1, 4), 3), np.array([0]), 0.5)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_split_merge_equals_unsplit():
    """Partials over disjoint key sets, merged with the rescaling rule, equal
    attention over the union (the combine step of split-KV decode)."""
    B, H, N, d = 1, 1, 64, 8
    q, k, v = rnd((B, N, H, d), 81), rnd((B, N, H, d), 82), rnd((B, N, H, d), 83)
    nbr = nbc = 4
    parts = [[0], [1, 3], [2]]
    rows = [(0, 0, i) for i in (0, 9, 33, 63)]
    o_full, l_full = oracle.attn_rows(q, k, v, 0.3, rows, oracle.MASK_NONE)
    o_parts, l_parts = [], []
    for cols in parts:
        bm = np.zeros((nbr, nbc), np.uint8)
        bm[:, cols] = 1
        o_s, l_s = oracle.attn_rows(q, k, v, 0.3, rows, oracle.MASK_BLOCK, bm)
        o_parts.append(o_s)
        l_parts.append(l_s)
    for r in range(len(rows)):
        o, l = oracle.merge_partials(np.stack([p[r] for p in o_parts]), np.array([p[r] for p in l_parts]))
        np.testing.assert_allclose(o, o_full[r], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(l, l_full[r], rtol=1e-14, atol=1e-14)
    # an empty partial contributes nothing
    o, l = oracle.merge_partials(np.stack([o_full[0], np.full(d, 7.0)]), np.array([l_full[0], -np.inf]))
    np.testing.assert_allclose(o, o_full[0], rtol=1e-15)
    assert l == l_full[0]


# --------------------------------------------------------------------------
# Masks and tile classification
# --------------------------------------------------------------------------

def test_frame_block_map_and_counts():
    """24 frames x 1040 tokens, query frame f sees key frames {0, f-1, f}.
    Closed forms: 1 + 2 + 3*22 = 69 live frame pairs; at 16x16 every block is
    uniform, 65 blocks per frame side, so 69*65^2 full tiles."""
    F, L = 24, 1040
    bm = oracle.frame_block_map(F, L)
    nb = F * L // 16
    assert bm.shape == (nb, nb)
    fb = np.arange(nb) * 16 // L
    ref = (fb[None, :] == 0) | (fb[None, :] == fb[:, None]) | (fb[None, :] == fb[:, None] - 1)
    assert np.array_equal(bm.astype(bool), ref)
    cls16 = oracle.classify(oracle.MASK_BLOCK, bm, F * L, F * L, 16, 16)
    assert (cls16 == 1).sum() == 69 * 65 * 65 == 291525
    assert (cls16 == 2).sum() == 0
    assert (cls16 == 0).sum() == nb * nb - 291525 == 2142075
    assert oracle.count_allowed(oracle.MASK_BLOCK, bm, F * L, F * L) == 69 * L * L


def test_frame_classification_128():
    """At 128x128 the 1040-token frames straddle tile edges (1040 is not a
    multiple of 128), which creates partial tiles (TPU attention guide,
    step 3).  Independent count: aggregate the 16x16 block map per 8x8."""
    F, L = 24, 1040
    bm = oracle.frame_block_map(F, L)
    cls = oracle.classify(oracle.MASK_BLOCK, bm, F * L, F * L, 128, 128)
    nb = bm.shape[0]
    nt = (nb + 7) // 8
    pad = np.zeros((nt * 8, nt * 8), np.int64)
    pad[:nb, :nb] = bm
    cnt = pad.reshape(nt, 8, nt, 8).sum(axis=(1, 3))
    tot = np.zeros_like(cnt)
    valid = np.zeros((nt * 8, nt * 8), np.int64)
    valid[:nb, :nb] = 1
    tot = valid.reshape(nt, 8, nt, 8).sum(axis=(1, 3))
    ref = np.where(cnt == 0, 0, np.where(cnt == tot, 1, 2))
    assert np.array_equal(cls, ref)
    assert ((cls == 1).sum(), (cls == 2).sum(), (cls == 0).sum()) == (4205, 818, 33002)


def test_causal_classification_closed_form():
    cls = oracle.classify(oracle.MASK_CAUSAL, None, 1024, 1024, 128, 128)
    n = 8
    assert (cls == 1).sum() == n * (n - 1) // 2 == 28
    assert (cls == 2).sum() == n == 8
    assert (cls == 0).sum() == 28
    assert oracle.count_allowed(oracle.MASK_CAUSAL, None, 1024, 1024) == 1024 * 1025 // 2
    # bottom-right alignment with Nq < Nkv: the last query sees every key
    assert oracle.allowed(oracle.MASK_CAUSAL, None, 3, 10, 2, 9)
    assert not oracle.allowed(oracle.MASK_CAUSAL, None, 3, 10, 0, 8)
    assert oracle.count_allowed(oracle.MASK_CAUSAL, None, 3, 10) == 8 + 9 + 10


def test_check_schedule_detects_planted_mistakes():
    N = 64
    good_q = [(0, 32, 0, 1), (32, 32, 1, 2)]
    good_kv = [(0, 32, 1), (0, 32, 0), (32, 32, 1)]
    assert oracle.check_schedule(oracle.MASK_CAUSAL, None, N, N, good_q, good_kv) == 0
    # gap in Q rows
    assert oracle.check_schedule(oracle.MASK_CAUSAL, None, N, N, [(0, 32, 0, 1)], good_kv) == 1
    # overlapping KV tiles
    assert oracle.check_schedule(oracle.MASK_CAUSAL, None, N, N, good_q,
                                 [(0, 32, 1), (0, 32, 0), (16, 48, 1)]) == 2
    # missing coverage (diagonal tile dropped)
    assert oracle.check_schedule(oracle.MASK_CAUSAL, None, N, N, [(0, 32, 0, 1), (32, 32, 1, 1)],
                                 good_kv) == 3
    # a diagonal tile claimed full
    assert oracle.check_schedule(oracle.MASK_CAUSAL, None, N, N, good_q,
                                 [(0, 32, 0), (0, 32, 0), (32, 32, 1)]) == 4


# --------------------------------------------------------------------------
# Gradients (the backward pass): torch autograd, finite differences, invariants
# --------------------------------------------------------------------------

def _sdpa_grads(q, k, v, dout, scale, allowed):
    """dQ, dK, dV of torch SDPA (fp64, CPU, math path, torch's own GQA
    mapping) for the upstream gradient dout."""
    Q, K, V = (torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True) for x in (q, k, v))
    G = Q.shape[1] // K.shape[1]
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(allowed),
                                                         scale=scale, enable_gqa=G > 1)
    O.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    return tuple(t.grad.permute(0, 2, 1, 3).numpy() for t in (Q, K, V))


@pytest.mark.parametrize("case", CASES)
def test_oracle_gradients_match_torch_autograd(case):
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = (hash(case) & 0xFFFF) + 17
    q, k, v = rnd((B, Nq, Hq, d), seed), rnd((B, Nkv, Hkv, d), seed + 1), rnd((B, Nkv, Hkv, d), seed + 2)
    dout = rnd((B, Nq, Hq, d), seed + 3)
    bm = None
    if kind == oracle.MASK_BLOCK:
        rng = np.random.default_rng(seed)
        bm = (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < 0.6).astype(np.uint8)
        bm[:, 0] = 1
    if kind == oracle.MASK_CAUSAL and Nq > Nkv:
        pytest.skip("rows without keys are pinned separately")
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale, kind, bm)
    rq, rk, rv = _sdpa_grads(q, k, v, dout, scale, _allowed_matrix(kind, bm, Nq, Nkv))
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(got, ref, atol=1e-11, rtol=1e-10)


def test_oracle_gradients_match_finite_differences():
    # central differences of the forward oracle's loss sum(O * dout)
    B, Hq, Hkv, Nq, Nkv, d = 1, 4, 2, 6, 9, 3
    rng = np.random.default_rng(5)
    q, k, v, dout = (rng.standard_normal(s) for s in ((B, Nq, Hq, d), (B, Nkv, Hkv, d), (B, Nkv, Hkv, d),
                                                        (B, Nq, Hq, d)))
    scale, kind = 0.7, oracle.MASK_CAUSAL
    grads = oracle.attn_bwd(q, k, v, dout, scale, kind)

    def loss(q_, k_, v_):
        return float((oracle.attn_fwd(q_, k_, v_, scale, kind)[0] * dout).sum())

    h = 1e-5
    for which, x in enumerate((q, k, v)):
        for flat in rng.choice(x.size, size=6, replace=False):
            idx = np.unravel_index(flat, x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p, args_m = [q, k, v], [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grads[which][idx]) <= 1e-7 + 1e-6 * abs(fd), (which, idx, fd, grads[which][idx])


def test_oracle_gradient_invariants():
    B, Hq, Hkv, Nq, Nkv, d = 2, 6, 3, 40, 70, 16
    q, k, v, dout = rnd((B, Nq, Hq, d), 71), rnd((B, Nkv, Hkv, d), 72), rnd((B, Nkv, Hkv, d), 73), \
        rnd((B, Nq, Hq, d), 74)
    scale = 0.25
    # bottom-right causal: rows see keys up to i + 30, so keys 0..30 are seen by every row
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale, oracle.MASK_CAUSAL)
    # each row's dS sums to zero over its keys (softmax is shift invariant), so sum_j dK_j = 0
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-11)
    # with dout = 1 every row's probabilities sum to one: sum_j dV_j = rows x query heads
    _, _, dv1 = oracle.attn_bwd(q, k, v, np.ones_like(dout), scale, oracle.MASK_CAUSAL)
    np.testing.assert_allclose(dv1.sum(axis=1), Nq * (Hq // Hkv), rtol=1e-12)
    # keys that no row may see get no gradient; neither does a row that sees no key
    bm = np.ones(((Nq + 15) // 16, (Nkv + 15) // 16), np.uint8)
    bm[:, 2] = 0           # keys 32..47 masked for everyone
    bm[1, :] = 0           # rows 16..31 see nothing
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale, oracle.MASK_BLOCK, bm)
    assert not dk[:, 32:48].any() and not dv[:, 32:48].any()
    assert not dq[:, 16:32].any()
    assert dk[:, :32].any() and dq[:, :16].any()


@pytest.mark.parametrize("case", [CASES[1], CASES[3], CASES[5]])
def test_oracle_dq_rows_match_torch_autograd(case):
    """The per-row dQ (for gradient checks at full size) against torch
    autograd of SDPA on sampled rows, masks and GQA included."""
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = (hash(case) & 0xFFFF) + 29
    q, k, v = rnd((B, Nq, Hq, d), seed), rnd((B, Nkv, Hkv, d), seed + 1), rnd((B, Nkv, Hkv, d), seed + 2)
    dout = rnd((B, Nq, Hq, d), seed + 3)
    bm = None
    if kind == oracle.MASK_BLOCK:
        rng = np.random.default_rng(seed)
        bm = (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < 0.6).astype(np.uint8)
        bm[:, 0] = 1
    scale = 1.0 / math.sqrt(d)
    rq, _, _ = _sdpa_grads(q, k, v, dout, scale, _allowed_matrix(kind, bm, Nq, Nkv))
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, B, 12), rng.integers(0, Hq, 12), rng.integers(0, Nq, 12)], axis=1).astype(np.int32)
    got = oracle.attn_bwd_dq_rows(q, k, v, dout, scale, rows, kind, bm)
    ref = np.stack([rq[b, i, h] for b, h, i in rows])
    np.testing.assert_allclose(got, ref, atol=1e-11, rtol=1e-10)
