"""A host model of the mbarrier protocol of the prefill kernel's main
pipeline (whole 128-key tiles), checked for deadlock and parity ambiguity
under random schedules, for both layouts:

  d = 64:  P in its own TMEM columns; the issuer puts S(j+1) on the tensor
           core as soon as the softmax has loaded S(j) (s_free), and the
           softmax writes P(j) only after PV(j-1) has completed (pv_done);
           Q double-buffered per slot; an 8-stage K/V ring.
  d = 128: P over S; the issuer puts S(j+1) right after PV(j) (one thread's
           MMAs complete in issue order, so the commit for S(j+1) also covers
           PV(j)); one Q buffer per slot; a 4-stage ring.

with and without the slot offset (slot A starts an item once slot B has
finished the exponentials of its first tile; slot B can be up to QB - 1
short items ahead of slot A's wait, so the kernel signals offset item n on
barrier n % QB).  Items are pairs as the planner makes them: equal slots,
slot A one tile shorter (causal pairs, not offset), a lone tile in slot B,
and a slot B with no key tile at all.  The half-tile pipeline of the
bound-based form has its own model (test_pipeline_model.py).
"""
import random

import pytest

from protocol_model import Bar, run


def prefill_model(items, D, stagger, rng, s_free_wait=True, b_first_bars=None):
    sep_p = D == 64
    R = 8 if D == 64 else 4
    QB = 2 if D == 64 else 1
    # slot B's offset signal: offset item n on barrier n % NB, NB = QB in the
    # kernel (a test plants one barrier at d = 64)
    NB = QB if b_first_bars is None else b_first_bars
    bars = {f"b_first{i}": Bar(4) for i in range(NB)}
    for x in (0, 1):
        for n, c in (("s_full", 1), ("p_full", 4), ("pv_done", 1), ("o_free", 4), ("s_free", 4)):
            bars[f"{n}{x}"] = Bar(c)
        for q in range(QB):
            bars[f"q_full{x}_{q}"] = Bar(1)
            bars[f"q_empty{x}_{q}"] = Bar(1)
    for i in range(R):
        bars[f"ring_full{i}"] = Bar(1)
        bars[f"ring_empty{i}"] = Bar(2)  # released by both slots' issuers
    queue = []

    def op(*commits):
        queue.append("op")
        queue.extend(commits)

    def producer():
        seq, qcnt = 0, [0, 0]
        for it in items:
            for x, n in ((0, it["nA"]), (1, it["nB"])):
                if n == 0:
                    continue
                qb, use = qcnt[x] % QB, qcnt[x] // QB
                if use > 0:
                    yield (f"q_empty{x}_{qb}", use - 1)
                bars[f"q_full{x}_{qb}"].arrive()
                qcnt[x] += 1
            for _ in range(2 * it["nB"]):
                if seq >= R:
                    yield (f"ring_empty{seq % R}", seq // R - 1)
                bars[f"ring_full{seq % R}"].arrive()
                seq += 1

    def issuer(x):
        seq = qcnt = scnt = pcnt = ocnt = 0
        for it in items:
            nX, nB = (it["nA"] if x == 0 else it["nB"]), it["nB"]
            if nX > 0:
                qb = qcnt % QB
                yield (f"q_full{x}_{qb}", qcnt // QB)
                qcnt += 1

                def issue_s(kpos):
                    nonlocal scnt
                    if sep_p and scnt > 0 and s_free_wait:
                        yield (f"s_free{x}", scnt - 1)
                    op(f"s_full{x}", f"ring_empty{kpos % R}")
                    scnt += 1

                yield (f"ring_full{seq % R}", seq // R)
                yield from issue_s(seq)
                for j in range(nX):
                    vseq, kseq = seq + 2 * j + 1, seq + 2 * j + 2
                    nxt = j + 1 < nX
                    if sep_p and nxt:
                        yield (f"ring_full{kseq % R}", kseq // R)
                        yield from issue_s(kseq)
                    yield (f"ring_full{vseq % R}", vseq // R)
                    yield (f"p_full{x}", pcnt)
                    if j == 0 and ocnt > 0:
                        yield (f"o_free{x}", ocnt - 1)
                    op(f"pv_done{x}", f"ring_empty{vseq % R}")
                    pcnt += 1
                    if not sep_p and nxt:
                        yield (f"ring_full{kseq % R}", kseq // R)
                        yield from issue_s(kseq)
                ocnt += 1
            for j in range(nX, nB):  # stages this slot does not visit
                for t in (0, 1):
                    pos = seq + 2 * j + t
                    yield (f"ring_full{pos % R}", pos // R)
                    bars[f"ring_empty{pos % R}"].arrive()
            seq += 2 * nB
            if nX > 0:
                queue.append(f"q_empty{x}_{qb}")

    def softmax(x):
        tcnt = bcnt = 0
        for it in items:
            nX = it["nA"] if x == 0 else it["nB"]
            nrows = it["rowsA"] if x == 0 else it["rowsB"]
            if nrows == 0:
                continue
            stag = stagger and it["nA"] > 0
            if stag and x == 0:
                yield (f"b_first{bcnt % NB}", bcnt // NB)
            if stag:
                bcnt += 1
            for t in range(nX):
                yield (f"s_full{x}", tcnt)
                if sep_p:
                    bars[f"s_free{x}"].arrive()  # S loaded into registers
                if stag and x == 1 and t == 0:
                    bars[f"b_first{(bcnt - 1) % NB}"].arrive()
                if sep_p and t > 0:
                    yield (f"pv_done{x}", tcnt - 1)  # P columns and O free
                bars[f"p_full{x}"].arrive()
                tcnt += 1
            if nX > 0:
                yield (f"pv_done{x}", tcnt - 1)  # the item's last PV
                bars[f"o_free{x}"].arrive()

    roles = {"producer": producer(), "issuer0": issuer(0), "issuer1": issuer(1)}
    for x in (0, 1):
        for q in range(4):
            roles[f"softmax{x}{q}"] = softmax(x)
    return roles, bars, queue


def random_items(rng, stagger):
    items = []
    for _ in range(rng.randint(1, 8)):
        nB = rng.randint(0, 10)
        kinds = [0, 2] if stagger else [0, 1, 2]
        kind = rng.choice(kinds) if nB > 0 else 2
        nA = nB if kind == 0 else (nB - 1 if kind == 1 else 0)
        items.append(dict(nA=nA, nB=nB, rowsA=128 if nA > 0 else 0, rowsB=rng.choice([16, 128])))
    return items


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("stagger", [False, True])
def test_prefill_protocol_has_no_deadlock_or_parity_ambiguity(D, stagger):
    rng = random.Random(D * 7 + stagger)
    for trial in range(250):
        roles, bars, queue = prefill_model(random_items(rng, stagger), D, stagger, random.Random(trial))
        r = run(roles, bars, queue, random.Random(trial))
        assert r == "ok", (trial, r)


def test_model_catches_s_issued_before_the_softmax_has_loaded_it():
    """The model has teeth: at d = 64 without the s_free wait (S(j+1) issued
    into the columns the softmax may still be reading), a schedule puts the
    softmax two phases behind s_full."""
    rng = random.Random(9)
    found = False
    for trial in range(300):
        items = random_items(rng, False)
        roles, bars, queue = prefill_model(items, 64, False, random.Random(trial), s_free_wait=False)
        r = run(roles, bars, queue, random.Random(trial))
        if r != "ok":
            assert "s_full" in r, r
            found = True
            break
    assert found


def test_one_offset_barrier_with_two_q_buffers_is_parity_ambiguous():
    """The model has teeth: at d = 64 (two Q buffers per slot) with one
    offset barrier, slot B can finish the first tile of the next short item
    before slot A waits for the current one."""
    rng = random.Random(4)
    found = False
    for trial in range(400):
        items = random_items(rng, True)
        roles, bars, queue = prefill_model(items, 64, True, random.Random(trial), b_first_bars=1)
        r = run(roles, bars, queue, random.Random(trial))
        if r != "ok":
            assert "b_first" in r, r
            found = True
            break
    assert found
