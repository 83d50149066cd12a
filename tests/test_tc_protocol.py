"""The tensor-core kernel's synchronisation, replayed on the host.

Every role of attn_tc_kernel is a program of mbarrier arrivals and waits in
the kernel's order: the K/V and Q producers (TMA loads), the K and Q prep, one
S-MMA and one PV-MMA issuer per softmax warpgroup, and each of the eight
softmax warps.  TMA copies complete in any order; each issuer thread's MMAs
and commits execute in its issue order, with no order between threads.  Random interleavings run over real per-CTA tile sequences (the
kernel's own host plan, `swin_debug_tc_plan`, decoded tile by tile).

Beyond deadlock freedom and unambiguous parity waits (no wait may see a phase
two or more completions old), the model tracks what every buffer holds and
checks each access against it at the moment it happens:
  * a TMA load may overwrite a K/V stage only after every S and PV MMA that
    reads the stage's previous block has executed, and a Q buffer only after
    all S MMAs of its previous tile and the softmax warps' row-scale reads;
  * an S MMA reads the Q tile and K block it is meant to (loaded and
    prepared), and overwrites S[b % 2] only after the four softmax warps have
    copied S(b - 2) out; a softmax warp reads exactly S(b);
  * a softmax warp writes P(b) only after PV(b - 2) has executed; PV(b) reads
    P(b) written by all four warps and V of its own block;
  * a PV that starts a tile's O runs only after the previous tile's O has
    been read by every warp with rows in it; a rescale or an epilogue read
    of O sees PV(0..b-1) executed and PV(b) not.
Tests also plant mistakes in the model (a missing wait, a ring too small for
resident windows) and check that the model catches each one.
"""
import random

import pytest

from vision_transformer_shifted_window_b200 import swin_attn as sa


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


class Race(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise Race(msg)


def plan_for(B, H, W, heads, M, s, mode, table, sms=148):
    plan, tiles = sa.swin_debug_tc_plan(B, H, W, heads, M, s, mode, table, sms)
    return plan, tiles


def passes(tiles, t0, t1, max_pass):
    t = t0
    while t < t1:
        row = tiles[t]
        ntile, k = int(row[10]), int(row[12])
        n = min(ntile - k, t1 - t, max_pass)
        yield t, n, row
        t += n


def tile_geom(row, k, g):
    """(rows, nq, lane offset) of tile k of the unit in `row` for warpgroup g."""
    ly, lx, R, Rh = int(row[4]), int(row[6]), int(row[7]), int(row[8])
    rows = min(R, ly - k * R)
    nq = rows * lx
    loff = 64 * g if rows <= Rh else 0
    return rows, nq, loff


def run(tiles, plan, t0, t1, mode, seed, rescale_p=0.2, bug=None, nst=None, max_pass=None):
    rng = random.Random(seed)
    nst = plan["nst"] if nst is None else nst
    nqb = plan["nqb"]
    max_pass = plan["max_pass_tiles"] if max_pass is None else max_pass
    ps = list(passes(tiles, t0, t1, max_pass))
    bars = {}

    def bar(name, count):
        bars[name] = Bar(name, count)
    for g in range(2):
        for q in range(nqb):
            bar(("q_full", g, q), 1); bar(("q_ready", g, q), 1); bar(("q_empty", g, q), 5)
        for x in range(2):
            bar(("s_full", g, x), 1); bar(("s_free", g, x), 4); bar(("p_full", g, x), 4); bar(("p_free", g, x), 1)
    for i in range(nst):
        bar(("kv_full", i), 1); bar(("kv_ready", i), 1); bar(("kv_empty", i), 2)

    def W(name, k):
        return ("wait", name, k)

    # ---- buffer contents
    kv = [None] * nst          # stage -> dict(pos, loaded, prepped, reads, expect)
    qb = {}                    # (g, slot) -> dict(tile, loaded, prepped, s_reads, s_expect)
    sm_reads = {}              # tile -> softmax warps done with its Q buffer
    Sb = {(g, x): {"b": None, "reads": 4} for g in range(2) for x in range(2)}
    Pb = {(g, x): {"b": None, "writers": 0} for g in range(2) for x in range(2)}
    pv_exec = [0, 0]           # PVs executed per warpgroup (in order)
    o_epi = {}                 # (g, tile) -> [warps that must read, warps that read]
    prev_tile = {}             # (g, tile) -> previous tile of the warpgroup
    tma = []                   # pending TMA completions
    mmaq = {("S", 0): [], ("S", 1): [], ("PV", 0): [], ("PV", 1): []}

    def wg_of(t):
        return (t - t0) & 1

    # ------------------------------------------------------------ roles
    def kv_producer():
        loads = 0
        for t, n, u in ps:
            for j in range(int(u[11])):
                slot, rnd = loads % nst, loads // nst
                if loads >= nst:
                    yield W(("kv_empty", slot), rnd - 1)
                old = kv[slot]
                if old is not None:
                    check(old["reads"] == old["expect"],
                          "K/V stage %d overwritten with %d of %d reads of position %d done" %
                          (slot, old["reads"], old["expect"], old["pos"]))
                kv[slot] = {"pos": loads, "loaded": False, "prepped": False, "reads": 0, "expect": 2 * n}
                tma.append(("kv", slot))
                loads += 1

    def q_producer():
        qn = [0, 0]
        for t, n, u in ps:
            for i in range(n):
                g = wg_of(t + i)
                slot, rnd = qn[g] % nqb, qn[g] // nqb
                if qn[g] >= nqb:
                    yield W(("q_empty", g, slot), rnd - 1)
                old = qb.get((g, slot))
                if old is not None:
                    check(old["s_reads"] == old["s_expect"] and sm_reads.get(old["tile"], 0) == 4,
                          "Q buffer %s overwritten before its tile was consumed" % ((g, slot),))
                qb[(g, slot)] = {"tile": t + i, "loaded": False, "prepped": False, "s_reads": 0,
                                 "s_expect": int(u[11])}
                tma.append(("q", g, slot))
                qn[g] += 1

    def k_prep():
        cnt = 0
        for t, n, u in ps:
            for j in range(int(u[11])):
                slot, rnd = cnt % nst, cnt // nst
                yield W(("kv_full", slot), rnd)
                check(kv[slot]["pos"] == cnt and kv[slot]["loaded"], "K prep on a stale stage")
                kv[slot]["prepped"] = True
                bars[("kv_ready", slot)].arrive()
                cnt += 1

    def q_prep():
        qn = [0, 0]
        for t, n, u in ps:
            for i in range(n):
                g = wg_of(t + i)
                slot, rnd = qn[g] % nqb, qn[g] // nqb
                yield W(("q_full", g, slot), rnd)
                check(qb[(g, slot)]["tile"] == t + i and qb[(g, slot)]["loaded"], "Q prep on a stale buffer")
                qb[(g, slot)]["prepped"] = True
                bars[("q_ready", g, slot)].arrive()
                qn[g] += 1

    def s_issuer(g):
        """S MMAs of warpgroup g (their own thread)."""
        b = qcnt = base = 0
        for t, n, u in ps:
            nb = int(u[11])
            for i in [i for i in range(n) if wg_of(t + i) == g]:
                qslot, qrnd = qcnt % nqb, qcnt // nqb
                for j in range(nb):
                    pos = base + j
                    slot, rnd = pos % nst, pos // nst
                    if b >= 2 and bug != "s_without_s_free":
                        yield W(("s_free", g, b & 1), (b - 2) >> 1)
                    if j == 0:
                        yield W(("q_ready", g, qslot), qrnd)
                    yield W(("kv_ready", slot), rnd)
                    c = [("S", g, b, slot, pos, qslot, t + i), ("bar", ("s_full", g, b & 1))]
                    if j == nb - 1:
                        c.append(("bar", ("q_empty", g, qslot)))
                        qcnt += 1
                    mmaq[("S", g)].append(c)
                    b += 1
            base += nb

    def pv_issuer(g):
        """PV MMAs of warpgroup g (their own thread)."""
        b = base = 0
        for t, n, u in ps:
            nb = int(u[11])
            mine = [i for i in range(n) if wg_of(t + i) == g]
            last_i = mine[-1] if mine else -1
            for i in mine:
                rel = (2 if n == 1 else 1) if i == last_i else 0
                for j in range(nb):
                    pos = base + j
                    slot = pos % nst
                    if bug != "pv_without_p_full":
                        yield W(("p_full", g, b & 1), b >> 1)
                    c = [("PV", g, b, slot, pos, j > 0, t + i), ("bar", ("p_free", g, b & 1))]
                    c += [("bar", ("kv_empty", slot))] * rel
                    mmaq[("PV", g)].append(c)
                    b += 1
            base += nb

    def softmax_warp(g, wq):
        """One softmax warp, in the kernel's order: S(b + 1) is copied out
        (prefetched) at the top of block b, P(b - 1)'s p_full arrival is
        deferred to the top of block b, and O is touched at the end of a block."""
        steps = []  # (tile id, unit row, tile index k, block j, ring position)
        base = 0
        for t, n, u in ps:
            nb, k0 = int(u[11]), int(u[12])
            for i in range(n):
                if wg_of(t + i) == g:
                    steps += [(t + i, u, k0 + i, j, base + j) for j in range(nb)]
            base += nb
        nblk = len(steps)
        pv_done = 0
        pend, pend_tile = False, None
        last_tile = None
        active = False
        p_pending = False

        def wait_pv(upto):
            nonlocal pv_done
            while pv_done <= upto:
                yield W(("p_free", g, pv_done & 1), pv_done >> 1)
                pv_done += 1

        def read_s(b):
            check(Sb[(g, b & 1)]["b"] == b, "softmax read S(%d) but the buffer holds S(%s)" % (b, Sb[(g, b & 1)]["b"]))
            Sb[(g, b & 1)]["reads"] += 1

        def release_p(b):  # P(b) written by this warp (store landed), then p_full(b)
            Pb[(g, b & 1)]["writers"] = Pb[(g, b & 1)]["writers"] + 1 if Pb[(g, b & 1)].get("for") == b else 1
            Pb[(g, b & 1)]["for"] = b
            bars[("p_full", g, b & 1)].arrive()

        qcnt = 0
        if nblk:
            yield W(("s_full", g, 0), 0)
            read_s(0)
            bars[("s_free", g, 0)].arrive()
        for b, (tid, u, k, j, pos) in enumerate(steps):
            nb = int(u[11])
            slot, rnd = pos % nst, pos // nst
            has_next = b + 1 < nblk
            if has_next:
                yield W(("s_full", g, (b + 1) & 1), (b + 1) >> 1)
                read_s(b + 1)  # the copy is issued here and lands before s_free(b + 1)
            if p_pending:
                release_p(b - 1)
                p_pending = False
            if j == 0:
                rows, nq, loff = tile_geom(u, k, g)
                active = wq * 32 + 31 >= loff and wq * 32 < loff + nq
                prev_tile[(g, tid)] = last_tile
                last_tile = tid
                o_epi.setdefault((g, tid), [0, 0])[0] += 1 if active else 0
                qslot, qrnd = qcnt % nqb, qcnt // nqb
                if mode != 0:
                    yield W(("q_ready", g, qslot), qrnd)
                    check(qb[(g, qslot)]["tile"] == tid and qb[(g, qslot)]["prepped"], "row scale of a stale tile")
                # mode 0 reads nothing from the Q buffer and may release it
                # before the tile has even been loaded
                sm_reads[tid] = sm_reads.get(tid, 0) + 1
                bars[("q_empty", g, qslot)].arrive()
                qcnt += 1
            if active and mode == 1:
                yield W(("kv_ready", slot), rnd)
                check(kv[slot]["pos"] == pos and kv[slot]["prepped"], "1/|k| of a stale stage")
            if b >= 2 and bug != "p_without_pv_wait":
                yield from wait_pv(b - 2)
            if active:
                check(pv_exec[g] >= b - 1, "P(%d) written before PV(%d) executed" % (b, b - 2))
            p_pending = True
            epi = j == 0 and pend
            resc = j > 0 and active and rng.random() < rescale_p
            if epi or resc:
                yield from wait_pv(b - 1)
                check(pv_exec[g] == b, "O read with %d PVs executed at block %d" % (pv_exec[g], b))
                if epi:
                    o_epi[(g, pend_tile)][1] += 1
                    pend = False
            if has_next:
                bars[("s_free", g, (b + 1) & 1)].arrive()
            if j == nb - 1:
                pend, pend_tile = active, tid
        if p_pending:
            release_p(nblk - 1)
        if pend:
            yield from wait_pv(nblk - 1)
            check(pv_exec[g] == nblk, "final O read early")
            o_epi[(g, pend_tile)][1] += 1

    def execute(entry):
        kind = entry[0]
        if kind == "bar":
            bars[entry[1]].arrive()
        elif kind == "S":
            _, g, b, slot, pos, qslot, tile = entry
            check(kv[slot]["pos"] == pos and kv[slot]["prepped"], "S(%d) read K of a stale stage" % b)
            q = qb[(g, qslot)]
            check(q["tile"] == tile and q["prepped"], "S(%d) read a stale Q tile" % b)
            q["s_reads"] += 1
            kv[slot]["reads"] += 1
            check(Sb[(g, b & 1)]["reads"] == 4, "S(%d) overwrote S(%s) before all warps copied it" %
                  (b, Sb[(g, b & 1)]["b"]))
            Sb[(g, b & 1)] = {"b": b, "reads": 0}
        elif kind == "PV":
            _, g, k, slot, pos, acc, tile = entry
            check(kv[slot]["pos"] == pos, "PV(%d) read V of a stale stage" % k)
            kv[slot]["reads"] += 1
            check(Pb[(g, k & 1)].get("for") == k and Pb[(g, k & 1)]["writers"] == 4,
                  "PV(%d) read P before all warps wrote it" % k)
            if not acc:
                prev = prev_tile.get((g, tile))
                if prev is not None:
                    need, done = o_epi[(g, prev)]
                    check(done == need, "tile %d's first PV overwrote O before %d of %d reads" % (tile, done, need))
            check(pv_exec[g] == k, "PVs out of order")
            pv_exec[g] += 1

    roles = {"kvp": kv_producer(), "qp": q_producer(), "kprep": k_prep(), "qprep": q_prep(),
             "s0": s_issuer(0), "s1": s_issuer(1), "pv0": pv_issuer(0), "pv1": pv_issuer(1)}
    for g in range(2):
        for wq in range(4):
            roles["sm%d_%d" % (g, wq)] = softmax_warp(g, wq)
    waiting = {r: None for r in roles}
    alive = set(roles)

    def ready(w):
        _, name, k = w
        c = bars[name].done
        if c >= k + 2:
            raise AssertionError("parity alias on %s: waiting for completion %d, %d done" % (name, k, c))
        return c >= k + 1
    steps = 0
    while alive or tma or any(mmaq.values()):
        steps += 1
        cands = [("role", r) for r in alive if waiting[r] is None or ready(waiting[r])]
        if tma:
            cands.append(("tma", None))
        for key, q in mmaq.items():
            if q:
                cands.append(("mma", key))
        if not cands:
            raise Deadlock({r: waiting[r] for r in alive})
        kind, x = rng.choice(cands)
        if kind == "role":
            try:
                waiting[x] = next(roles[x])
            except StopIteration:
                alive.discard(x)
        elif kind == "tma":
            e = tma.pop(rng.randrange(len(tma)))
            if e[0] == "kv":
                kv[e[1]]["loaded"] = True
                bars[("kv_full", e[1])].arrive()
            else:
                qb[(e[1], e[2])]["loaded"] = True
                bars[("q_full", e[1], e[2])].arrive()
        else:
            for entry in mmaq[x].pop(0):
                execute(entry)
    for g in range(2):
        for key, (need, done) in o_epi.items():
            assert done == need, ("O of a tile never read", key, need, done)
    return steps


WORKLOADS = {  # B, H, W, heads, M, shift, mode, table
    "swin-t-M7": (32, 56, 56, 3, 7, 3, 0, True),
    "swinv2-t-M16": (64, 64, 64, 3, 16, 8, 1, True),
    "flashswin-t-M32": (16, 112, 112, 3, 32, 16, 2, False),
    "swinv2-g-M24": (2, 384, 384, 16, 24, 12, 1, True),
    "ragged-M7": (1, 20, 37, 2, 7, 3, 1, True),
    "ragged-M32": (3, 17, 64, 3, 32, 16, 1, True),
    "M24-no-shift-odd": (1, 100, 60, 5, 24, 0, 0, False),
    "M16-shift0": (2, 33, 33, 1, 16, 0, 2, False),
    "thin-M8": (1, 9, 200, 4, 8, 4, 1, True),
    "M64-streaming": (2, 70, 64, 3, 64, 0, 2, False),
    "M3-tiny": (2, 5, 130, 1, 3, 1, 0, True),
}


def _windows(plan, span):
    """CTA ranges to replay: the first, a middle and the last CTA's range,
    cut to `span` tiles at their start and at their end."""
    cs = plan["cta_start"]
    out = []
    for c in sorted({0, len(cs) // 2 - 1, len(cs) - 2}):
        a, b = cs[c], cs[c + 1]
        out.append((a, min(b, a + span)))
        if b - a > span:
            out.append((b - span, b))
    return out


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_protocol_no_deadlock_no_race(name):
    B, H, W, heads, M, s, mode, table = WORKLOADS[name]
    plan, tiles = plan_for(B, H, W, heads, M, s, mode, table)
    for t0, t1 in _windows(plan, 24):
        for seed in range(3):
            run(tiles, plan, t0, t1, mode, seed)


def test_protocol_small_grids_whole_ranges():
    """Few CTAs, so that each replays a long range end to end."""
    for (B, H, W, heads, M, s, mode, table) in [(1, 40, 36, 3, 16, 8, 1, True), (1, 20, 37, 2, 7, 3, 0, True),
                                                (1, 40, 40, 1, 32, 16, 2, False)]:
        plan, tiles = plan_for(B, H, W, heads, M, s, mode, table, sms=3)
        cs = plan["cta_start"]
        for c in range(len(cs) - 1):
            for seed in range(2):
                run(tiles, plan, cs[c], cs[c + 1], mode, seed)


@pytest.mark.parametrize("bug", ["p_without_pv_wait", "s_without_s_free", "pv_without_p_full"])
def test_model_catches_planted_races(bug):
    B, H, W, heads, M, s, mode, table = WORKLOADS["swinv2-t-M16"]
    plan, tiles = plan_for(B, H, W, heads, M, s, mode, table)
    with pytest.raises((Race, AssertionError)):
        for seed in range(20):
            run(tiles, plan, 0, 12, mode, seed, bug=bug)


def test_model_catches_resident_windows_in_a_short_ring():
    """A pass over every tile of a window needs the ring to hold all of the
    window's blocks plus three; with fewer stages the K/V producer waits for
    a stage that only a later block would free."""
    B, H, W, heads, M, s, mode, table = WORKLOADS["flashswin-t-M32"]
    plan, tiles = plan_for(B, H, W, heads, M, s, mode, table)
    assert plan["max_pass_tiles"] > 8 and plan["nst"] >= 16 + 3
    t0 = next(t for t in range(len(tiles)) if tiles[t][11] == 16 and tiles[t][12] == 0)  # a 32 x 32 window
    with pytest.raises(Deadlock):
        for seed in range(4):
            run(tiles, plan, t0, t0 + 16, mode, seed, nst=12)
    # the same short ring is fine when passes stream (two tiles per pass)
    for seed in range(3):
        run(tiles, plan, t0, t0 + 16, mode, seed, nst=12, max_pass=2)


def test_plan_decodes_every_tile_in_order():
    """The host plan's tile list is the units in order (heads, images, rows and
    columns of rectangles, tiles), enumerated here from the segment geometry."""
    def segs(L, M, s):
        st = list(range(0, L, M)) if s == 0 else [0] + list(range(s, L, M))
        return [(a, min(b, L) - a) for a, b in zip(st, st[1:] + [L])]
    for name, (B, H, W, heads, M, s, mode, table) in WORKLOADS.items():
        plan, tiles = plan_for(B, H, W, heads, M, s, mode, table)
        want = []
        for h in range(heads):
            for b in range(B):
                for y0, ly in segs(H, M, s):
                    for x0, lx in segs(W, M, s):
                        R = 128 // lx
                        for k in range((ly + R - 1) // R):
                            want.append((h, b, y0, ly, x0, lx, k))
        got = [(int(r[0]), int(r[1]), int(r[3]), int(r[4]), int(r[5]), int(r[6]), int(r[12])) for r in tiles]
        assert got == want, name
        cs = plan["cta_start"]
        assert cs[0] == 0 and cs[-1] == len(want) and all(a < b for a, b in zip(cs, cs[1:])), name
