"""The tensor-core kernel's barrier protocol, replayed on the host.

Every role of attn_tc_kernel (TMA producer, operand prep, one MMA issuer per
softmax warpgroup, two softmax warpgroups) is modelled as a program of
mbarrier arrivals and parity waits in the kernel's order; TMA copies complete
in any order, each issuer's MMA commits complete in issue order, and the
online-softmax rescale happens at random.  Random interleavings over the real
per-CTA work-item sequences of every workload must finish with no deadlock and
with no wait whose parity could match a phase two or more completions old.
The tensor-memory hazard is checked too: S(b) overwrites the buffer that
holds P(b - 2), so PV(b - 2) must be issued before it (a thread's MMAs run in
issue order).
"""
import random

import pytest

S = 6  # K/V ring stages of the kernel
KBLK = 96  # keys per K/V block


# segment geometry of the shifted partition (cut at s + kM, clipped)
def nseg(L, M, s):
    if s == 0: return (L + M - 1) // M
    if L <= s: return 1
    return 1 + (L - s + M - 1) // M


def seg_start(k, M, s):
    if s == 0: return k * M
    return 0 if k == 0 else s + (k - 1) * M


def seg_len(k, L, M, s):
    a = seg_start(k, M, s)
    b = (k + 1) * M if s == 0 else s + k * M
    return min(b, L) - a


def items_for(B, H, W, heads, M, s, cta, grid, pos_major=False):
    """Work items of CTA `cta` in the kernel's order: heads outermost, then
    image, then rows of rectangles; item i of a row takes tiles 2i and 2i+1 of
    the row's tile list (rectangles left to right, each split into query
    tiles of floor(128 / lx) rows).  Returns (nb0, nb1, shared) per item: K/V
    blocks of warpgroup 0's and 1's rectangles (nb1 = 0: no second tile) and
    whether both tiles are in one rectangle (K/V blocks shared)."""
    nsy, nsx = nseg(H, M, s), nseg(W, M, s)
    cls = lambda sx: 0 if sx == 0 else (2 if sx == nsx - 1 else 1)
    lxs = [seg_len(0, W, M, s), seg_len(1, W, M, s) if nsx > 2 else seg_len(0, W, M, s), seg_len(nsx - 1, W, M, s)]
    R = [128 // l for l in lxs]
    Rk = [KBLK // l for l in lxs]
    per_hb = []
    for sy in range(nsy):
        ly = seg_len(sy, H, M, s)
        tiles = []
        for sx in range(nsx):
            c = cls(sx)
            nt = (ly + R[c] - 1) // R[c]
            tiles += [(sx, (ly + Rk[c] - 1) // Rk[c])] * nt
        for i in range(0, len(tiles), 2):
            a = tiles[i]
            if i + 1 < len(tiles):
                b = tiles[i + 1]
                per_hb.append((a[1], b[1], a[0] == b[0]))
            else:
                per_hb.append((a[1], 0, False))
    n_items = B * heads * len(per_hb)
    if pos_major:  # item i: position i // (B heads) of (head, image) i % (B heads)
        return [per_hb[it // (B * heads)] for it in range(cta, n_items, grid)]
    return [per_hb[it % len(per_hb)] for it in range(cta, n_items, grid)]


def kv_order(nb0, nb1, shared):
    """Consumers of the item's K/V loads in ring order: shared blocks go to
    both warpgroups; otherwise the two rectangles' blocks alternate, then the
    longer one's remainder follows."""
    if shared:
        return [(0, 1)] * nb0
    mn = min(nb0, nb1)
    out = []
    for j in range(mn):
        out += [(0,), (1,)]
    out += [(0,)] * (nb0 - mn) + [(1,)] * (nb1 - mn)
    return out


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


def run(items, mode, seed, rescale_p=0.2, early_pv=True, pv_lag=2):
    rng = random.Random(seed)
    bars = {}

    def bar(name, count):
        if name not in bars: bars[name] = Bar(name, count)
        return bars[name]
    for g in range(2):
        for b in range(2):
            bar(("q_full", g, b), 1); bar(("q_ready", g, b), 1); bar(("q_empty", g, b), 5)
            bar(("s_full", g, b), 1); bar(("p_full", g, b), 1); bar(("o_done", g, b), 1)
    for i in range(S):
        bar(("kv_full", i), 1); bar(("kv_ready", i), 1); bar(("kv_empty", i), 2)

    def W(name, k):
        """wait for completion k (0-based) of a barrier, by parity"""
        return ("wait", name, k)

    tma = []  # pending async TMA completions (any order)
    mmaq = {0: [], 1: []}  # per issuer FIFO of commit lists

    def producer():
        qu = [0, 0]; ku = 0
        for (nb0, nb1, shared) in items:
            for g, v in ((0, True), (1, nb1 > 0)):
                if not v: continue
                qs = qu[g] & 1
                if qu[g] >= 2: yield W(("q_empty", g, qs), (qu[g] >> 1) - 1)
                tma.append(("q_full", g, qs)); qu[g] += 1
            for _ in kv_order(nb0, nb1, shared):
                st = ku % S
                if ku >= S: yield W(("kv_empty", st), ku // S - 1)
                tma.append(("kv_full", st)); ku += 1

    def prep():
        qu = [0, 0]; ku = 0
        for (nb0, nb1, shared) in items:
            for g, v in ((0, True), (1, nb1 > 0)):
                if not v: continue
                qs = qu[g] & 1
                yield W(("q_full", g, qs), qu[g] >> 1); qu[g] += 1
                bars[("q_ready", g, qs)].arrive()
            for _ in kv_order(nb0, nb1, shared):
                st = ku % S
                yield W(("kv_full", st), ku // S); ku += 1
                bars[("kv_ready", st)].arrive()

    def issuer(g):
        u = qcnt = b = npv = u_last = 0
        pend = [0, 0]

        def issue_pv(k):
            yield W(("p_full", g, k & 1), k >> 1)
            st, acc, rel2 = pend[k & 1]
            c = [("o_done", g, k & 1), ("kv_empty", st)]
            if rel2: c.append(("kv_empty", st))
            mmaq[g].append(c)
        for (nb0, nb1, shared) in items:
            order = kv_order(nb0, nb1, shared)
            u0 = u; u += len(order)
            mine = [u0 + k for k, c in enumerate(order) if g in c]
            if not mine: continue
            qs, qpar = qcnt & 1, (qcnt >> 1)
            qcnt += 1
            rel2 = not shared
            for j, uu in enumerate(mine):
                st = uu % S
                while npv + pv_lag <= b:
                    yield from issue_pv(npv); npv += 1
                if early_pv and npv < b and u_last + S <= uu:
                    yield from issue_pv(npv); npv += 1
                if j == 0: yield W(("q_ready", g, qs), qpar)
                yield W(("kv_ready", st), uu // S)
                assert npv + 2 > b, "S(%d) issued before PV(%d)" % (b, b - 2)
                c = [("s_full", g, b & 1)]
                if j == len(mine) - 1: c.append(("q_empty", g, qs))
                mmaq[g].append(c)
                pend[b & 1] = (st, j > 0, rel2)
                u_last = uu
                b += 1
        while npv < b:
            yield from issue_pv(npv); npv += 1

    def softmax(g):
        qu = ku = blk = 0
        o_cons = [0]
        pend = False

        def consume(upto):
            while o_cons[0] <= upto:
                yield W(("o_done", g, o_cons[0] & 1), o_cons[0] >> 1)
                o_cons[0] += 1
        for (nb0, nb1, shared) in items:
            order = kv_order(nb0, nb1, shared)
            ku0 = ku; ku += len(order)
            mine = [ku0 + k for k, c in enumerate(order) if g in c]
            if not mine: continue
            qs = qu & 1
            yield W(("q_ready", g, qs), qu >> 1); qu += 1
            bars[("q_empty", g, qs)].arrive(4)
            for j, uu in enumerate(mine):
                yield W(("s_full", g, blk & 1), blk >> 1)
                if mode == 1: yield W(("kv_ready", uu % S), uu // S)
                if blk >= 2: o_cons[0] = max(o_cons[0], blk - 1)  # implied by s_full(blk)
                epi = j == 0 and pend
                resc = j > 0 and rng.random() < rescale_p
                if epi or resc: yield from consume(blk - 1)
                bars[("p_full", g, blk & 1)].arrive()
                if epi: pend = False
                blk += 1
            pend = True
        if pend: yield from consume(blk - 1)

    roles = {"producer": producer(), "prep": prep(), "iss0": issuer(0), "iss1": issuer(1),
             "sm0": softmax(0), "sm1": softmax(1)}
    waiting = {k: None for k in roles}
    alive = set(roles)

    def ready(w):
        _, name, k = w
        c = bars[name].done
        if c >= k + 2:
            raise AssertionError("parity alias on %s: waiting for completion %d, %d done" % (name, k, c))
        return c >= k + 1
    steps = 0
    while alive or tma or mmaq[0] or mmaq[1]:
        steps += 1
        cands = []
        for r in alive:
            w = waiting[r]
            if w is None or ready(w): cands.append(("role", r))
        if tma: cands.append(("tma", None))
        for g in (0, 1):
            if mmaq[g]: cands.append(("mma", g))
        if not cands:
            raise Deadlock({r: waiting[r] for r in alive})
        kind, x = rng.choice(cands)
        if kind == "role":
            try:
                waiting[x] = next(roles[x])
            except StopIteration:
                alive.discard(x)
        elif kind == "tma":
            i = rng.randrange(len(tma))
            bars[tma.pop(i)].arrive()
        else:
            for c in mmaq[x].pop(0): bars[c].arrive()
    return steps




WORKLOADS = {  # B, H, W, heads, M, shift, mode
    "swin-t-M7": (32, 56, 56, 3, 7, 3, 0),
    "swinv2-t-M16": (64, 64, 64, 3, 16, 8, 1),
    "flashswin-t-M32": (16, 112, 112, 3, 32, 16, 2),
    "swinv2-g-M24": (2, 384, 384, 16, 24, 12, 1),
    "ragged-M7": (1, 20, 37, 2, 7, 3, 1),
    "ragged-M32": (3, 17, 64, 3, 32, 16, 1),
    "M24-no-shift-odd": (1, 100, 60, 5, 24, 0, 0),
    "M16-shift0": (2, 33, 33, 1, 16, 0, 2),
    "thin-M8": (1, 9, 200, 4, 8, 4, 1),
    "M64-rows": (32, 70, 64, 3, 64, 0, 2),
}


@pytest.mark.parametrize("pos_major", [False, True])
@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_protocol_no_deadlock_no_parity_alias(name, pos_major):
    """Both item orders: heads outermost (a bias table per head) and
    position-major (no table)."""
    B, H, W, heads, M, s, mode = WORKLOADS[name]
    grid = 148 if B * H * W > 20000 else 8
    for cta in (0, 1, grid // 3, grid - 1):
        items = items_for(B, H, W, heads, M, s, cta, grid, pos_major)
        for seed in range(4):
            run(items, mode, seed)


def test_model_catches_the_deadlock_it_guards_against():
    """Without the early PV issue (a pending PV whose K/V slot is a whole
    ring behind the block being waited for) the model deadlocks: with M = 64
    and a 6-row last rectangle row, an item that only warpgroup 0 works on
    fills the ring while warpgroup 1's last PV waits behind its next item."""
    items = items_for(32, 70, 64, 3, 64, 0, 5, 148)
    with pytest.raises(Deadlock):
        for seed in range(8):
            run(items, 2, seed, early_pv=False)
    for seed in range(4):
        run(items, 2, seed)


def test_model_catches_the_tmem_hazard():
    """An issuer that lets PV fall three blocks behind would overwrite P(b - 2)
    with S(b) before PV(b - 2) read it; the model rejects it."""
    items = items_for(16, 112, 112, 3, 32, 16, 0, 148)
    with pytest.raises(AssertionError):
        run(items, 2, 0, pv_lag=3)
