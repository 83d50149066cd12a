"""The fused block kernel's barrier protocol (k_block_tc.cu), replayed on the
host.

Roles: the TMA producer (weights once, then one input tile per work item into
a ring of S stages), the MMA issuer (one product per output into a ring of
TMEM accumulator slots) and one or two epilogue warpgroups (warpgroup e reads
the slots of products u with u % nepi == e, then stores).  Each role is a
program of mbarrier arrivals and parity waits in the kernel's order; TMA
copies complete in any order and the issuer's MMA commits complete in issue
order.  Random interleavings must finish with no deadlock,
no wait whose parity could match a phase two or more completions old, and no
tensor-memory or shared-memory hazard: a product never overwrites a slot the
epilogue has not finished reading, and a stage is never reloaded while its
input (or, for the post-norm, its residual tile) is still being read.
"""
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, self.name
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


class Deadlock(Exception):
    pass


def run(ntiles, nparts, S, NS, postnorm, seed, slot_wait=True, nepi=1):
    rng = random.Random(seed)
    bars = {("w_full",): Bar("w_full", 1)}
    for s in range(S):
        bars[("in_full", s)] = Bar(("in_full", s), 1)
        bars[("in_empty", s)] = Bar(("in_empty", s), 2 if postnorm else 1)
    for k in range(NS):
        bars[("slot_full", k)] = Bar(("slot_full", k), 1)
        bars[("slot_empty", k)] = Bar(("slot_empty", k), 4)

    def W(name, k):
        return ("wait", name, k)

    tma = []
    mmaq = []  # FIFO of commit lists (in issue order)
    slot_owner = {}  # slot -> product index whose accumulator it holds
    slot_reading = set()  # slots an epilogue warpgroup is reading
    stage_tile = {}  # stage -> tile whose input it holds
    stage_in_use = {}  # stage -> count of readers (MMA, epilogue residual)

    def producer():
        tma.append(("w_full",))
        for i in range(ntiles):
            s = i % S
            if i >= S:
                yield W(("in_empty", s), i // S - 1)
            assert stage_in_use.get(s, 0) == 0, "stage %d reloaded while read" % s
            stage_tile[s] = i
            tma.append(("in_full", s))

    def mma():
        yield W(("w_full",), 0)
        u = 0
        for i in range(ntiles):
            s = i % S
            yield W(("in_full", s), i // S)
            assert stage_tile[s] == i
            stage_in_use[s] = stage_in_use.get(s, 0) + 1
            for part in range(nparts):
                k = u % NS
                if u >= NS and slot_wait:
                    yield W(("slot_empty", k), u // NS - 1)
                assert k not in slot_reading, "slot %d overwritten while the epilogue reads it" % k
                slot_owner[k] = u
                mmaq.append([("slot_full", k)])
                u += 1
            mmaq.append([("release", s), ("in_empty", s)])

    def epilogue(ew):
        u = 0
        for i in range(ntiles):
            s = i % S
            mine = False
            for part in range(nparts):
                if u % nepi != ew:
                    u += 1
                    continue
                mine = True
                k = u % NS
                yield W(("slot_full", k), u // NS)
                if postnorm:
                    yield W(("in_full", s), i // S)
                    stage_in_use[s] = stage_in_use.get(s, 0) + 1
                assert slot_owner[k] == u, "slot %d holds product %d, expected %d" % (k, slot_owner[k], u)
                slot_reading.add(k)
                yield None  # the reads take time
                slot_reading.discard(k)
                bars[("slot_empty", k)].arrive(4)
                u += 1
            if postnorm and mine:
                stage_in_use[s] -= 1
                bars[("in_empty", s)].arrive()

    roles = {"producer": producer(), "mma": mma()}
    for ew in range(nepi):
        roles["epilogue%d" % ew] = epilogue(ew)
    waiting = {r: None for r in roles}
    alive = set(roles)

    def ready(w):
        _, name, k = w
        c = bars[name].done
        if c >= k + 2:
            raise AssertionError("parity alias on %s: waiting for completion %d, %d done" % (name, k, c))
        return c >= k + 1

    while alive or tma or mmaq:
        cands = [("role", r) for r in alive if waiting[r] is None or ready(waiting[r])]
        if tma:
            cands.append(("tma", None))
        if mmaq:
            cands.append(("mma", None))
        if not cands:
            raise Deadlock({r: waiting[r] for r in alive})
        kind, x = rng.choice(cands)
        if kind == "role":
            try:
                waiting[x] = next(roles[x])
            except StopIteration:
                alive.discard(x)
        elif kind == "tma":
            bars[tma.pop(rng.randrange(len(tma)))].arrive()
        else:
            for c in mmaq.pop(0):
                if c[0] == "release":
                    stage_in_use[c[1]] -= 1
                else:
                    bars[c].arrive()


# (C, nparts, stages, slots) of the kernel's plans: qkv at C = 32, 64, 96;
# post-norm at C = 32 ... 128 (slots = min(6, 512 / C))
PLANS = [(32, 3, 3, 6, False), (64, 3, 3, 6, False), (96, 3, 3, 5, False), (32, 1, 3, 6, True),
         (96, 1, 3, 5, True), (128, 1, 2, 4, True)]


@pytest.mark.parametrize("nepi", [1, 2])
@pytest.mark.parametrize("C,nparts,S,NS,postnorm", PLANS)
@pytest.mark.parametrize("ntiles", [1, 2, 7, 11])
def test_block_protocol(C, nparts, S, NS, postnorm, ntiles, nepi):
    for seed in range(6):
        run(ntiles, nparts, S, NS, postnorm, seed, nepi=nepi)


@pytest.mark.parametrize("nepi", [1, 2])
def test_model_catches_a_missing_slot_wait(nepi):
    with pytest.raises(AssertionError):
        for seed in range(20):
            run(11, 3, 3, 5, False, seed, slot_wait=False, nepi=nepi)
