"""Pins for the oracle's bound-based softmax (TPU attention guide, step 4).

The method replaces each row's running max by an upper bound of its scores
(Cauchy-Schwarz after centring the keys on their mean) and falls back to the
exact max where the bound could drive P below the floating-point range.  It
computes the same attention as the definition; these tests pin the oracle's
key statistics to library routines, the bound to the inequality it must
satisfy, the whole result to torch SDPA in fp64, and the fallback rule to
inputs where skipping it visibly fails.
"""
import math

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _allowed_matrix, _sdpa_ref, rnd


def test_key_stats_are_the_mean_and_the_largest_centred_norm():
    k = rnd((2, 37, 3, 16), 11)
    kbar, radius = oracle.key_stats(k)
    np.testing.assert_allclose(kbar, k.mean(axis=1), rtol=0, atol=1e-13)
    centred = k - k.mean(axis=1, keepdims=True)
    np.testing.assert_allclose(radius, np.linalg.norm(centred, axis=3).max(axis=1), rtol=1e-13)


def test_key_stats_on_bf16_inputs_use_the_stored_values():
    k32 = rnd((1, 29, 2, 8), 12, np.float32)
    bits = (k32.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 values will do
    kv = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    kbar, radius = oracle.key_stats(bits)
    np.testing.assert_allclose(kbar, kv.mean(axis=1), atol=1e-13)
    np.testing.assert_allclose(radius, np.linalg.norm(kv - kv.mean(axis=1, keepdims=True), axis=3).max(axis=1),
                               rtol=1e-13)


@pytest.mark.parametrize("seed", range(4))
def test_cauchy_schwarz_bound_holds_for_every_row(seed):
    """M_i = scale ||q_i|| radius bounds every centred score of the row from
    above, and -M_i bounds it from below."""
    B, Nq, Nkv, Hq, Hkv, d = 1, 40, 53, 4, 2, 32
    q, k = rnd((B, Nq, Hq, d), 100 + seed), rnd((B, Nkv, Hkv, d), 200 + seed) + 0.7
    scale = 1 / math.sqrt(d)
    kbar, radius = oracle.key_stats(k)
    G = Hq // Hkv
    for hq in range(Hq):
        h = hq // G
        s = scale * q[0, :, hq, :] @ (k[0, :, h, :] - kbar[0, h]).T  # [Nq, Nkv]
        M = scale * np.linalg.norm(q[0, :, hq, :], axis=1) * radius[0, h]
        assert np.all(s.max(axis=1) <= M * (1 + 1e-12))
        assert np.all(s.min(axis=1) >= -M * (1 + 1e-12))


BOUND_CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, kind
    (1, 2, 2, 9, 9, 4, oracle.MASK_NONE),
    (2, 4, 2, 33, 33, 16, oracle.MASK_CAUSAL),
    (1, 6, 3, 64, 64, 32, oracle.MASK_BLOCK),
    (1, 8, 2, 17, 64, 64, oracle.MASK_NONE),
]


@pytest.mark.parametrize("case", BOUND_CASES)
@pytest.mark.parametrize("limit2", [oracle.BOUND_LIMIT2, 0.0])
def test_bound_softmax_matches_torch_sdpa(case, limit2):
    """Bound rows (default limit) and fallback rows (limit 0) both give the
    definition's O and LSE; keys are offset so that centring matters."""
    B, Hq, Hkv, Nq, Nkv, d, kind = case
    seed = hash(case) & 0xFFFF
    q, k, v = rnd((B, Nq, Hq, d), seed), rnd((B, Nkv, Hkv, d), seed + 1) + 1.5, rnd((B, Nkv, Hkv, d), seed + 2)
    bm = None
    if kind == oracle.MASK_BLOCK:
        rng = np.random.default_rng(seed)
        bm = (rng.random(((Nq + 15) // 16, (Nkv + 15) // 16)) < 0.6).astype(np.uint8)
        bm[:, 0] = 1
    scale = 1.0 / math.sqrt(d)
    o, lse, flags = oracle.attn_fwd_bound(q, k, v, scale, kind, bm, limit2=limit2)
    ro, rlse = _sdpa_ref(q, k, v, scale, _allowed_matrix(kind, bm, Nq, Nkv))
    np.testing.assert_allclose(o, ro, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, rlse, atol=1e-12, rtol=1e-12)
    if limit2 == 0.0:
        assert flags.sum() == 0
    else:
        assert flags.all()  # unit-normal inputs at these sizes are far inside the limit


def test_fallback_rule_follows_the_bound_size():
    """A row uses the bound iff 2 M log2(e) <= limit: rows with a large query
    norm fall back, the others do not."""
    B, Nq, Nkv, H, d = 1, 24, 30, 1, 16
    q, k, v = rnd((B, Nq, H, d), 7), rnd((B, Nkv, H, d), 8), rnd((B, Nkv, H, d), 9)
    q[0, ::3] *= 40.0  # every third query is 40x longer
    scale = 0.25
    kbar, radius = oracle.key_stats(k)
    M = scale * np.linalg.norm(q[0, :, 0, :], axis=1) * radius[0, 0]
    expect = (2 * M * math.log2(math.e) <= oracle.BOUND_LIMIT2).astype(np.int32)
    assert 0 < expect.sum() < Nq  # both kinds of row present
    o, lse, flags = oracle.attn_fwd_bound(q, k, v, scale)
    np.testing.assert_array_equal(flags[0, 0], expect)
    ro, rlse = _sdpa_ref(q, k, v, scale, np.ones((Nq, Nkv), bool))
    np.testing.assert_allclose(o, ro, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(lse, rlse, atol=1e-10, rtol=1e-12)


def test_without_the_fallback_large_bounds_underflow():
    """The fallback is needed: forcing the bound on rows whose bound is huge
    drives every P to 0 (l = 0), which the default rule avoids."""
    B, Nq, Nkv, H, d = 1, 4, 8, 1, 8
    q, k, v = rnd((B, Nq, H, d), 21) * 300.0, rnd((B, Nkv, H, d), 22), rnd((B, Nkv, H, d), 23)
    scale = 1.0
    with np.errstate(invalid="ignore", divide="ignore"):
        o_forced, _, flags_forced = oracle.attn_fwd_bound(q, k, v, scale, limit2=1e30)
    assert flags_forced.all()
    assert not np.isfinite(o_forced).all()
    o, lse, flags = oracle.attn_fwd_bound(q, k, v, scale)
    assert flags.sum() == 0
    ro, rlse = _sdpa_ref(q, k, v, scale, np.ones((Nq, Nkv), bool))
    np.testing.assert_allclose(o, ro, atol=1e-12, rtol=1e-10)


def test_shifting_every_key_changes_lse_only_by_the_shift():
    """Adding u to every key of a head moves kbar by u, keeps the radius and
    O, and shifts each row's LSE by scale q_i . u (mean-centring is exact)."""
    B, Nq, Nkv, Hq, Hkv, d = 1, 20, 20, 2, 1, 8
    q, k, v = rnd((B, Nq, Hq, d), 31), rnd((B, Nkv, Hkv, d), 32), rnd((B, Nkv, Hkv, d), 33)
    u = rnd((d,), 34) * 3.0
    scale = 0.3
    kb0, r0 = oracle.key_stats(k)
    kb1, r1 = oracle.key_stats(k + u)
    np.testing.assert_allclose(kb1, kb0 + u, atol=1e-12)
    np.testing.assert_allclose(r1, r0, rtol=1e-12)
    o0, l0, f0 = oracle.attn_fwd_bound(q, k, v, scale, oracle.MASK_CAUSAL)
    o1, l1, f1 = oracle.attn_fwd_bound(q, k + u, v, scale, oracle.MASK_CAUSAL)
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    shift = scale * np.einsum("bnhd,d->bhn", q, u)
    np.testing.assert_allclose(l1, l0 + shift, atol=1e-11)
    np.testing.assert_array_equal(f0, f1)


def test_identical_keys_give_the_plain_mean_of_values():
    """All keys equal: radius 0, every score equal, P = 1 on every allowed key,
    O = the mean of the allowed values (causal: a prefix mean)."""
    B, N, H, d = 1, 12, 1, 4
    q, v = rnd((B, N, H, d), 41), rnd((B, N, H, d), 42)
    k = np.broadcast_to(rnd((1, 1, 1, d), 43), (B, N, H, d)).copy()
    kbar, radius = oracle.key_stats(k)
    assert radius[0, 0] < 1e-12
    o, lse, flags = oracle.attn_fwd_bound(q, k, v, 0.5, oracle.MASK_CAUSAL)
    assert flags.all()
    prefix_mean = np.cumsum(v[0, :, 0, :], axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(o[0, :, 0, :], prefix_mean, atol=1e-13)
    s = 0.5 * q[0, :, 0, :] @ k[0, 0, 0, :]
    np.testing.assert_allclose(lse[0, 0], s + np.log(np.arange(1, N + 1)), atol=1e-12)
