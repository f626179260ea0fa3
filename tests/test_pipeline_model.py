"""A host model of the mbarrier protocol of the prefill kernel's half-tile
pipeline (d = 128, bound-based softmax), checked for deadlock and for parity
ambiguity under random schedules.

The kernel's roles and barriers, as the model has them (one CTA):
  producer   Q of each slot, then K_j, V_j of every KV tile into a ring of R
             stages (ring_full / ring_empty, each stage released by both
             slots' issuers);
  issuer x   per item: S(0), S(1), then for each half-tile step s: PV(s) once
             the softmax has written P(s), then S(s + 2).  S(s) goes to buffer
             s & 1 of slot x and signals s_full[x][s & 1]; PV(s) signals
             pv_done; the item's last PV signals o_ready; the K (V) stage is
             released after the S (PV) of the tile's last half; the first PV of
             an item waits until the softmax has read the previous item's O;
  softmax x  per step: wait for S(s), write P(s), arrive on p_full[x][s & 1];
             per item: the epilogue waits for o_ready and frees O; slot A
             starts each item after slot B's first step (the stagger).
A tensor-core operation completes in issue order at a random later time, and
any role can be held back for a while (the shared engine in protocol_model.py).

An mbarrier wait names only the parity of the phase it waits for, so a waiter
must never fall two phases behind its barrier (it would then wait for a phase
that has already gone by, forever).  The model gives each wait the index of
its phase and fails if that ever happens; with one P barrier per slot instead
of one per S buffer, the softmax can finish step s + 1 before the issuer has
waited for step s, which the last test reproduces.
"""
import random

import pytest

from protocol_model import Bar, run


def simulate(items, rng, R=4, stagger=True, p_per_buffer=True, max_rounds=400000):
    bars = {}

    def bar(name, count):
        bars[name] = Bar(count)

    for x in (0, 1):
        for n, c in (("q_full", 1), ("q_empty", 1), ("s_full0", 1), ("s_full1", 1), ("p_full0", 4),
                     ("p_full1", 4), ("pv_done", 1), ("o_free", 4), ("o_ready", 1)):
            bar(f"{n}{x}", c)
    for i in range(R):
        bar(f"ring_full{i}", 1)
        bar(f"ring_empty{i}", 2)
    bar("b_first", 4)
    tensor_queue = []  # issued tensor-core operations ("op") and their commits, in issue order

    def op(*commits):
        tensor_queue.append("op")
        tensor_queue.extend(commits)

    def p_bar(x, step):
        return f"p_full{step & 1}{x}" if p_per_buffer else f"p_full0{x}"

    def p_index(step):
        return step >> 1 if p_per_buffer else step

    def producer():
        seq, qcnt = 0, [0, 0]
        for it in items:
            for x, n in ((0, it["nA"]), (1, it["nB"])):
                if n == 0:
                    continue
                if qcnt[x] > 0:
                    yield (f"q_empty{x}", qcnt[x] - 1)
                bars[f"q_full{x}"].arrive()
                qcnt[x] += 1
            for _ in range(2 * it["nB"]):
                if seq >= R:
                    yield (f"ring_empty{seq % R}", seq // R - 1)
                bars[f"ring_full{seq % R}"].arrive()
                seq += 1

    def issuer(x):
        seq = qcnt = scnt = pcnt = ocnt = 0
        for it in items:
            nX, nB, kv = (it["nA"] if x == 0 else it["nB"]), it["nB"], it["kv"]
            if nX > 0:
                yield (f"q_full{x}", qcnt)
                qcnt += 1
                steps = [(j, h) for j in range(nX) for h in range(2 if kv[j] > 64 else 1)]
                last_half = {(j, h): h == (1 if kv[j] > 64 else 0) for j, h in steps}
                s_next = 0

                def issue_s():
                    nonlocal s_next, scnt
                    j, h = steps[s_next]
                    kpos = seq + 2 * j
                    if h == 0:
                        yield (f"ring_full{kpos % R}", kpos // R)
                    op(f"s_full{scnt & 1}{x}", *([f"ring_empty{kpos % R}"] if last_half[(j, h)] else []))
                    scnt += 1
                    s_next += 1

                yield from issue_s()
                if s_next < len(steps):
                    yield from issue_s()
                for i, (j, h) in enumerate(steps):
                    yield (p_bar(x, pcnt), p_index(pcnt))
                    if i == 0 and ocnt > 0:
                        yield (f"o_free{x}", ocnt - 1)
                    vpos = seq + 2 * j + 1
                    if h == 0:
                        yield (f"ring_full{vpos % R}", vpos // R)
                    op(f"pv_done{x}", *([f"ring_empty{vpos % R}"] if last_half[(j, h)] else []))
                    pcnt += 1
                    if s_next < len(steps):
                        yield from issue_s()
                tensor_queue.append(f"o_ready{x}")
                ocnt += 1
            for j in range(nX, nB):  # stages of tiles past slot A's prefix
                for t in (0, 1):
                    pos = seq + 2 * j + t
                    yield (f"ring_full{pos % R}", pos // R)
                    bars[f"ring_empty{pos % R}"].arrive()
            seq += 2 * nB
            if nX > 0:
                tensor_queue.append(f"q_empty{x}")

    def softmax(x):
        tcnt = bcnt = icnt = 0
        for it in items:
            nX, nrows, kv = (it["nA"], it["nrowsA"], it["kv"]) if x == 0 else (it["nB"], it["nrowsB"], it["kv"])
            if nrows == 0:
                continue
            stag = stagger and it["nA"] > 0
            if stag and x == 0:
                yield ("b_first", bcnt)
            if stag:
                bcnt += 1
            t0 = tcnt
            for j in range(nX):
                for _ in range(2 if kv[j] > 64 else 1):
                    yield (f"s_full{tcnt & 1}{x}", tcnt >> 1)
                    if stag and x == 1 and tcnt == t0:
                        bars["b_first"].arrive()
                    bars[p_bar(x, tcnt)].arrive()
                    tcnt += 1
            if nX > 0:
                yield (f"o_ready{x}", icnt)
                icnt += 1
                bars[f"o_free{x}"].arrive()

    roles = {"producer": producer(), "issuer0": issuer(0), "issuer1": issuer(1)}
    for x in (0, 1):
        for q in range(4):
            roles[f"softmax{x}{q}"] = softmax(x)
    return run(roles, bars, tensor_queue, rng, max_rounds)


def random_items(rng):
    """Items as the planner makes them: equal pairs (GQA heads, frame tiles),
    causal pairs with slot A one tile shorter, lone tiles in slot B; tile
    widths of 16 to 128 keys (one or two half-tile steps)."""
    items = []
    for _ in range(rng.randint(1, 8)):
        nB = rng.randint(1, 12)
        kind = rng.randint(0, 2)
        nA = nB if kind == 0 else (nB - 1 if kind == 1 else 0)
        kv = [rng.choice([16, 48, 64, 80, 128]) for _ in range(nB)]
        items.append(dict(nA=nA, nB=nB, nrowsA=128 if nA > 0 else 0, nrowsB=128, kv=kv))
    return items


def test_half_tile_protocol_has_no_deadlock_or_parity_ambiguity():
    rng = random.Random(11)
    for trial in range(300):
        items = random_items(rng)
        stagger = all(it["nA"] in (0, it["nB"]) for it in items)  # as the host decides it
        r = simulate(items, random.Random(trial), stagger=stagger)
        assert r == "ok", (trial, r)


def test_one_p_barrier_per_slot_is_parity_ambiguous():
    """The model has teeth: with one P barrier per slot (the first version of
    this pipeline, which ran a bounded wait out on the GPU), some schedule
    lets a waiter fall two phases behind."""
    rng = random.Random(3)
    found = False
    for trial in range(200):
        items = random_items(rng)
        r = simulate(items, random.Random(trial), stagger=False, p_per_buffer=False)
        if r != "ok":
            assert "parity ambiguous" in r or "deadlock" in r
            found = True
            break
    assert found
