"""Generic engine for the host models of the kernels' mbarrier protocols.

Roles are generators that yield (barrier name, phase index) to wait for a
phase and arrive on barriers directly; tensor-core operations and their
commits go into one queue that completes in issue order at random times ("op"
entries are operations, other entries are barriers a commit arrives on once
everything before it has completed).  `run` interleaves the roles at random
and reports a deadlock, or a waiter that could be two phases behind its
barrier (an mbarrier wait names only the parity of its phase).
"""


class Bar:
    """An mbarrier: `count` arrivals complete a phase."""

    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


def run(roles, bars, queue, rng, max_rounds=400000):
    waiting = {k: None for k in roles}
    finished = set()
    frozen = {k: 0 for k in roles}  # a role that stalls (a warp not scheduled) for some rounds
    for _ in range(max_rounds):
        if len(finished) == len(roles):
            return "ok"
        progressed = skipped = False
        order = list(roles)
        rng.shuffle(order)
        for k in order:
            if k in finished:
                continue
            if frozen[k] > 0:
                frozen[k] -= 1
                skipped = True
                continue
            if rng.random() < 0.02:
                frozen[k] = rng.randint(1, 30)
            for _ in range(rng.randint(1, 3)):
                w = waiting[k]
                if w is not None:
                    name, index = w
                    if bars[name].phase > index + 1:
                        return f"parity ambiguous: {k} waits for phase {index} of {name}, at {bars[name].phase}"
                    if bars[name].phase <= index:
                        break
                    waiting[k] = None
                try:
                    waiting[k] = next(roles[k])
                except StopIteration:
                    finished.add(k)
                    progressed = True
                    break
                progressed = True
        for _ in range(rng.randint(0, 3)):
            if queue:
                entry = queue.pop(0)
                if entry != "op":
                    bars[entry].arrive()
                progressed = True
        if not progressed and skipped:
            continue
        if not progressed:
            if queue:
                entry = queue.pop(0)
                if entry != "op":
                    bars[entry].arrive()
                continue
            return "deadlock: " + ", ".join(f"{k} waits {waiting[k]}" for k in roles if k not in finished)
    return "did not finish"
