"""Host models of the mbarrier protocols of the two backward kernels (dK/dV
and dQ), checked for deadlock and parity ambiguity under random schedules.

Each role of a kernel is a generator that yields the barrier phase it waits
for and arrives on barriers directly; tensor-core operations and their
commits go into one queue that completes in issue order at random times (a
commit arrives once everything issued before it has completed).  An
mbarrier wait names only the parity of its phase, so the model fails as soon
as a waiter could be two phases behind its barrier, and fails on a deadlock.
The roles follow the kernels' code: the producer's ring of R stages and its
per-item resident tiles, the MMA issuer's order (two S buffers where the
columns allow, dP issued once the element-wise warps have read the previous
one), the element-wise warps' waits and arrivals, and the hand-over of the
accumulators at the end of an item.  Items with no step (a key tile that no
query sees, a Q tile that sees no key) are included.
"""
import random

import pytest

from protocol_model import Bar, run


def dkdv_model(steps, R, NB, n_ew, rng, p_alternate=None):
    """steps: the number of Q-tile steps of each item (0 allowed).
    p_alternate: P of step t on one of two barriers by the parity of t, as
    the kernel does with two S buffers (the default follows NB), or on a
    single barrier (with two S buffers: the mistake the last test plants)."""
    if p_alternate is None:
        p_alternate = NB == 2
    bars = {n: Bar(c) for n, c in (("fixed_full", 1), ("fixed_empty", 1), ("dp_full", 1), ("p_full0", n_ew),
                                   ("p_full1", n_ew), ("ds_full", n_ew), ("mma_done", 1), ("acc_free", n_ew))}

    def p_bar(t):
        return (f"p_full{t & 1}", t >> 1) if p_alternate else ("p_full0", t)
    for s in range(R):
        bars[f"full{s}"] = Bar(1)
        bars[f"empty{s}"] = Bar(1 + n_ew)
    for x in range(NB):
        bars[f"s_full{x}"] = Bar(1)
    queue = []

    def op(*commits):
        queue.append("op")
        queue.extend(commits)

    def producer():
        g = 0
        for k, n in enumerate(steps):
            if k > 0:
                yield ("fixed_empty", k - 1)
            bars["fixed_full"].arrive()
            for _ in range(n):
                s = g % R
                if g >= R:
                    yield (f"empty{s}", g // R - 1)
                bars[f"full{s}"].arrive()
                g += 1

    def mma():
        g = 0
        for k, n in enumerate(steps):
            yield ("fixed_full", k)
            if n == 0:
                queue.append("fixed_empty")
                continue
            yield (f"full{g % R}", g // R)
            if g > 0:
                yield ("mma_done", g - 1)
            op(f"s_full{g % NB}")                       # S^T(g)
            op("dp_full")                               # dP^T(g)
            if n == 1:
                queue.append("fixed_empty")
            for u in range(n):
                nxt = u + 1 < n
                if NB == 2 and nxt:
                    yield (f"full{(g + 1) % R}", (g + 1) // R)
                    if u >= 1:
                        yield ("mma_done", g - 1)
                    op(f"s_full{(g + 1) % 2}")          # S^T(g+1)
                yield p_bar(g)
                if u == 0 and k > 0:
                    yield ("acc_free", k - 1)
                op()                                    # dV += P^T dO
                yield ("ds_full", g)
                op(f"empty{g % R}", "mma_done")         # dK += dS^T Q
                if nxt:
                    if NB == 1:
                        yield (f"full{(g + 1) % R}", (g + 1) // R)
                        yield ("mma_done", g)
                        op("s_full0")                   # S^T(g+1), one buffer
                    op("dp_full")                       # dP^T(g+1)
                    if u + 2 == n:
                        queue.append("fixed_empty")
                g += 1

    def ew():
        g = 0
        for k, n in enumerate(steps):
            for _ in range(n):
                yield (f"full{g % R}", g // R)
                yield (f"s_full{g % NB}", g // NB)
                bars[p_bar(g)[0]].arrive()              # P written over S
                yield ("dp_full", g)
                bars["ds_full"].arrive()                # dS written behind P
                bars[f"empty{g % R}"].arrive()
                g += 1
            if n > 0:
                yield ("mma_done", g - 1)
            bars["acc_free"].arrive()                   # dV, dK read out

    roles = {"producer": producer(), "mma": mma()}
    for i in range(n_ew):
        roles[f"ew{i}"] = ew()
    return roles, bars, queue


def dq_model(steps, R, NA, n_ew, rng):
    """steps: the number of KV-tile steps of each item (0 allowed)."""
    bars = {n: Bar(c) for n, c in (("fixed_full", 1), ("fixed_empty", 1 + n_ew), ("dp_full", 1),
                                   ("ds_full", n_ew), ("mma_done", 1))}
    for s in range(R):
        bars[f"full{s}"] = Bar(1)
        bars[f"empty{s}"] = Bar(1)
    for x in range(2):
        bars[f"s_full{x}"] = Bar(1)
    for a in range(NA):
        bars[f"acc_free{a}"] = Bar(n_ew)
    queue = []

    def op(*commits):
        queue.append("op")
        queue.extend(commits)

    def producer():
        g = 0
        for k, n in enumerate(steps):
            if k > 0:
                yield ("fixed_empty", k - 1)
            bars["fixed_full"].arrive()
            for _ in range(n):
                s = g % R
                if g >= R:
                    yield (f"empty{s}", g // R - 1)
                bars[f"full{s}"].arrive()
                g += 1

    def mma():
        g = 0
        for k, n in enumerate(steps):
            acc = k % NA
            yield ("fixed_full", k)
            if n == 0:
                queue.append("fixed_empty")
                continue
            yield (f"full{g % R}", g // R)
            if g > 0:
                yield ("mma_done", g - 1)
            op(f"s_full{g & 1}")                        # S(g)
            op("dp_full")                               # dP(g)
            if n == 1:
                queue.append("fixed_empty")
            for j in range(n):
                nxt = j + 1 < n
                if nxt:
                    yield (f"full{(g + 1) % R}", (g + 1) // R)
                    if j >= 1:
                        yield ("mma_done", g - 1)
                    op(f"s_full{(g + 1) & 1}")          # S(g+1)
                yield ("ds_full", g)
                if j == 0 and k >= NA:
                    yield (f"acc_free{acc}", k // NA - 1)
                op(f"empty{g % R}", "mma_done")         # dQ += dS K
                if nxt:
                    op("dp_full")                       # dP(g+1)
                    if j + 2 == n:
                        queue.append("fixed_empty")
                g += 1

    def ew():
        g = 0
        for k, n in enumerate(steps):
            acc = k % NA
            for j in range(n):
                yield (f"s_full{g & 1}", g >> 1)
                if j == 0:                              # D from the resident O and dO
                    yield ("fixed_full", k)
                    bars["fixed_empty"].arrive()
                yield ("dp_full", g)
                bars["ds_full"].arrive()
                g += 1
            if n == 0:
                yield ("fixed_full", k)
                bars["fixed_empty"].arrive()
            if n > 0:
                yield ("mma_done", g - 1)
            bars[f"acc_free{acc}"].arrive()             # dQ read out

    roles = {"producer": producer(), "mma": mma()}
    for i in range(n_ew):
        roles[f"ew{i}"] = ew()
    return roles, bars, queue


def random_steps(rng):
    return [rng.choice([0, 1, 1, 2, 3, 5, 8]) for _ in range(rng.randint(1, 7))]


@pytest.mark.parametrize("R,NB", [(4, 2), (2, 1)])  # d = 64, d = 128
def test_dkdv_protocol_has_no_deadlock_or_parity_ambiguity(R, NB):
    rng = random.Random(17 + R)
    for trial in range(250):
        roles, bars, queue = dkdv_model(random_steps(rng), R, NB, 3, random.Random(trial))
        r = run(roles, bars, queue, random.Random(trial))
        assert r == "ok", (trial, r)


@pytest.mark.parametrize("R,NA", [(4, 2), (2, 1)])  # d = 64, d = 128
def test_dq_protocol_has_no_deadlock_or_parity_ambiguity(R, NA):
    rng = random.Random(29 + R)
    for trial in range(250):
        roles, bars, queue = dq_model(random_steps(rng), R, NA, 3, random.Random(trial))
        r = run(roles, bars, queue, random.Random(trial))
        assert r == "ok", (trial, r)


def test_one_p_barrier_with_s_issued_early_is_parity_ambiguous():
    """The model has teeth: with one P barrier (as the dK/dV kernel had it)
    and S(t+1) issued before the wait for P(t), some schedule lets the
    element-wise warps finish P(t) and P(t+1) before that wait."""
    rng = random.Random(5)
    found = False
    for trial in range(400):
        roles, bars, queue = dkdv_model(random_steps(rng), 4, 2, 3, random.Random(trial), p_alternate=False)
        r = run(roles, bars, queue, random.Random(trial))
        if r != "ok":
            assert "parity ambiguous" in r, r
            found = True
            break
    assert found
