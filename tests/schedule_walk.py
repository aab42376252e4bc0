"""A CPU model of the split kernel's work schedule, for host-side tests.

The producer warp of every CTA walks a cursor over its share of the units
(batch row, KV head, row tile) and cuts it into segments (a contiguous block
range of one unit).  This module restates that walk in Python, step for step
(the balanced cost-space schedule with its per-row fixed costs and the tail
piece taken first, and the uniform schedule), so that a test can walk every
CTA of a launch and check what the kernel relies on: every KV block of every
unit is covered by exactly one CTA, the pieces of a split unit sit in
consecutive CTAs that agree on the first CTA and the piece count, and every
split unit is one a CTA tags before its pieces arrive.

It computes no attention and is not the oracle; nothing outside the tests
uses it.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

BLOCK_TOKENS = {64: 128, 128: 64, 256: 64}


def cdiv(a: int, b: int) -> int:
    return (a + b - 1) // b


def clamp_len(length: int, max_len: int) -> int:
    return 0 if length < 0 else min(length, max_len)


@dataclass
class Problem:
    """One launch: the shape, the rows' lengths and query counts, the plan."""
    B: int
    Hkv: int
    G: int
    q_len: int
    D: int
    lens: list
    q_counts: list          # per row (used when varlen)
    varlen: bool
    schedule: str           # "balanced" or "uniform"
    unit_cost_q: int = 0    # balanced: fixed cost of a unit, quarter blocks
    splits: int = 1         # uniform: pieces per unit
    T: int = field(init=False)
    RT: int = field(init=False)
    max_k: int = field(init=False)
    cu: list = field(init=False)
    total_q: int = field(init=False)
    chunk_blocks: int = field(init=False)

    def __post_init__(self):
        self.T = BLOCK_TOKENS[self.D]
        self.RT = cdiv(self.q_len * self.G, 16)
        self.max_k = max(self.lens + [1])
        self.cu = [0]
        for n in self.q_counts:
            self.cu.append(self.cu[-1] + n)
        self.total_q = self.cu[-1]
        self.chunk_blocks = max(1, cdiv(cdiv(self.max_k, self.T), self.splits))

    def row_queries(self, b: int):
        if self.varlen:
            s = min(max(self.cu[b], 0), self.total_q)
            e = min(max(self.cu[b + 1], s), self.total_q)
            return s, min(e - s, self.q_len)
        return b * self.q_len, self.q_len

    def row_tiles(self, qn: int) -> int:
        return cdiv(qn * self.G, 16)

    def row_cost(self, i: int) -> int:
        """Whole blocks of fixed cost of each unit of row i (the quarter-block
        cost shared out over the rows)."""
        q = self.unit_cost_q
        return ((i + 1) * q) // 4 - (i * q) // 4


@dataclass
class Cursor:
    b: int = 0
    hr: int = 0
    blk: int = 0
    x: int = 0
    end: int = 0
    per_cta: int = 1
    L: int = 0
    nb: int = 0
    L_next: int = 0
    rtb: int = 1
    V: int = 0
    q0: int = 0
    qn: int = 0
    q0_next: int = 0
    qn_next: int = 0


def _enter_row(c: Cursor, p: Problem, length: int):
    c.L = length
    c.nb = cdiv(length, p.T)
    if p.varlen:
        c.q0, c.qn = c.q0_next, c.qn_next
        c.rtb = p.row_tiles(c.qn)
        if c.rtb == 0:
            c.nb = 0  # a row without queries holds no units
        if c.b + 1 < p.B:
            c.q0_next, c.qn_next = p.row_queries(c.b + 1)
    else:
        c.q0, c.qn = c.b * p.q_len, p.q_len
    c.V = p.row_cost(c.b) if p.schedule == "balanced" else 0
    c.L_next = p.lens[c.b + 1] if c.b + 1 < p.B else 0


def _take(c: Cursor, p: Problem) -> dict:
    """The segment at the cursor; the cursor moves past it (and past the
    fixed cost of the unit that follows)."""
    HR = p.Hkv * c.rtb
    n = min(c.nb - c.blk, c.end - c.x)
    s = dict(b=c.b, h=c.hr // c.rtb, rt=c.hr % c.rtb, blk_beg=c.blk, blk_end=c.blk + n, q0=c.q0, qn=c.qn)
    s["kind"] = 0 if (c.blk == 0 and c.blk + n == c.nb) else (1 if c.blk > 0 else 2)
    if p.schedule == "balanced":
        xs = c.x - c.blk  # position of the unit's first block
        s["c_first"] = xs // c.per_cta
        s["n_pieces"] = (xs + c.nb - 1) // c.per_cta - s["c_first"] + 1
    else:
        unit = (c.b * p.Hkv + s["h"]) * p.RT + s["rt"]
        s["c_first"] = unit * p.splits
        s["n_pieces"] = cdiv(c.nb, p.chunk_blocks)
    c.x += n
    c.blk += n
    if c.blk == c.nb:
        c.blk = 0
        c.hr += 1
        if c.hr == HR:
            c.hr = 0
            if c.b + 1 < p.B:
                c.b += 1
                _enter_row(c, p, clamp_len(c.L_next, p.max_k))
                while c.nb == 0 and c.b + 1 < p.B:
                    c.b += 1
                    _enter_row(c, p, clamp_len(p.lens[c.b], p.max_k))
                if c.x + c.V >= c.end:
                    c.end = c.x  # that unit's first block lies past this range
            else:
                c.end = c.x
        c.x += c.V
    return s


def _first_row_past(scan: list, HS: int, x: int, lo: int) -> int:
    """First row (from `lo`) whose positions end past position x."""
    hi = len(scan) - 1
    while lo < hi:
        mid = (lo + hi) // 2
        if HS * scan[mid] > x:
            hi = mid
        else:
            lo = mid + 1
    return lo


def _start(p: Problem, bx: int, grid: int):
    """CTA bx's cursor, and its tail cursor when its range ends inside a unit
    that starts within it (that piece is taken first)."""
    HR = p.Hkv * p.RT
    c = Cursor(rtb=p.RT)
    tail = None
    if p.schedule == "uniform":
        u, si = bx // p.splits, bx % p.splits
        c.b, c.hr = u // HR, u % HR
        c.q0, c.qn = p.row_queries(c.b)
        c.L = clamp_len(p.lens[c.b], p.max_k)
        c.nb = cdiv(c.L, p.T)
        if p.varlen and c.hr % p.RT >= p.row_tiles(c.qn):
            c.nb = 0  # a tile past the row's queries
        beg = si * p.chunk_blocks
        end = min(beg + p.chunk_blocks, c.nb)
        c.blk = c.x = beg
        c.end = max(end, beg)
        return c, tail
    lens, scan, run = [], [], 0
    for i in range(p.B):
        L = clamp_len(p.lens[i], p.max_k)
        lens.append(L)
        nb = cdiv(L, p.T)
        w = nb + p.row_cost(i) if nb > 0 else 0  # positions of one unit of row i
        if p.varlen:
            w *= p.row_tiles(p.row_queries(i)[1])  # one KV head's units of the row
        run += w
        scan.append(run)
    HS = p.Hkv if p.varlen else HR
    NB = HS * run
    c.per_cta = 1 if NB == 0 else cdiv(NB, grid)
    x0 = bx * c.per_cta
    if x0 >= NB:
        return c, tail
    x1 = min(x0 + c.per_cta, NB)
    b0 = _first_row_past(scan, HS, x0, 0)
    pre = scan[b0 - 1] if b0 > 0 else 0
    w = scan[b0] - pre
    off = x0 - HS * pre
    V = p.row_cost(b0)
    uw = cdiv(lens[b0], p.T) + V if p.varlen else w  # positions of one unit of the row
    pos = off % uw
    c.b, c.hr, c.nb, c.V = b0, off // uw, uw - V, V
    if p.varlen:
        c.rtb = w // uw
        c.q0, c.qn = p.row_queries(b0)
        if b0 + 1 < p.B:
            c.q0_next, c.qn_next = p.row_queries(b0 + 1)
    else:
        c.q0, c.qn = b0 * p.q_len, p.q_len
    c.blk = pos - V if pos > V else 0
    c.x = x0 - pos + V + c.blk
    c.end = x1
    c.L = lens[b0]
    c.L_next = lens[b0 + 1] if b0 + 1 < p.B else 0
    xl = x1 - 1
    bl = _first_row_past(scan, HS, xl, b0)
    pre_l = scan[bl - 1] if bl > 0 else 0
    w_l = scan[bl] - pre_l
    off_l = xl - HS * pre_l
    Vl = p.row_cost(bl)
    uw_l = cdiv(lens[bl], p.T) + Vl if p.varlen else w_l
    pos_l = off_l % uw_l
    if pos_l >= Vl:  # xl falls on a KV block of that unit
        nb_l, blk_l = uw_l - Vl, pos_l - Vl
        x_t = xl - blk_l  # position of that unit's first block
        if blk_l + 1 < nb_l and x_t - Vl > x0:
            tail = replace(c, b=bl, hr=off_l // uw_l, blk=0, x=x_t, end=x1, V=Vl, nb=nb_l, L=lens[bl], L_next=0)
            if p.varlen:
                tail.rtb = w_l // uw_l
                tail.q0, tail.qn = p.row_queries(bl)
            else:
                tail.rtb = p.RT
                tail.q0, tail.qn = bl * p.q_len, p.q_len
            c.end = x_t - Vl  # the main walk stops where that unit begins
    return c, tail


def walk_cta(p: Problem, bx: int, grid: int):
    """CTA bx's segments in the order its producer takes them, and the split
    units it tags before any piece is counted (its first unit, if split, and
    its tail unit)."""
    c, tail = _start(p, bx, grid)
    unit_of = lambda k: (k.b * p.Hkv + k.hr // k.rtb) * p.RT + k.hr % k.rtb  # noqa: E731
    tagged = set()
    if c.x < c.end and c.nb > 0:
        if p.schedule == "balanced":
            split = c.blk > 0 or c.x - c.blk + c.nb > c.end
        else:
            split = c.nb > p.chunk_blocks
        if split:
            tagged.add(unit_of(c))
    if tail is not None:
        tagged.add(unit_of(tail))
    segs = []
    if tail is not None:
        segs.append(_take(tail, p))
    while c.x < c.end and c.nb > 0:
        segs.append(_take(c, p))
        assert len(segs) < 1_000_000
    return segs, tagged


def check_launch(p: Problem, grid: int):
    """Walk every CTA and check coverage and the split bookkeeping; raises
    AssertionError on a violation."""
    cover, pieces = {}, {}
    for bx in range(grid):
        segs, tagged = walk_cta(p, bx, grid)
        for s in segs:
            unit = (s["b"] * p.Hkv + s["h"]) * p.RT + s["rt"]
            q0, qn = p.row_queries(s["b"])
            assert (s["q0"], s["qn"]) == (q0, qn), (bx, s)
            assert s["rt"] < p.row_tiles(qn) and s["h"] < p.Hkv, (bx, s)
            assert s["blk_end"] > s["blk_beg"] >= 0, (bx, s)
            for blk in range(s["blk_beg"], s["blk_end"]):
                assert (unit, blk) not in cover, ("block read twice", unit, blk)
                cover[(unit, blk)] = bx
            if s["kind"] != 0:
                assert unit in tagged, ("split unit not tagged", bx, unit)
                pieces.setdefault(unit, []).append((s["blk_beg"], bx, s["kind"], s["c_first"], s["n_pieces"]))
    expected = 0
    for b in range(p.B):
        nb = cdiv(clamp_len(p.lens[b], p.max_k), p.T)
        for h in range(p.Hkv):
            for rt in range(p.row_tiles(p.row_queries(b)[1])):
                unit = (b * p.Hkv + h) * p.RT + rt
                for blk in range(nb):
                    assert (unit, blk) in cover, ("block missed", b, h, rt, blk)
                expected += nb
    assert len(cover) == expected
    for unit, ps in pieces.items():
        ps.sort()
        n, first = ps[0][4], ps[0][3]
        assert len(ps) == n, ("piece count", unit, ps)
        for i, (_, bx, kind, cf, ni) in enumerate(ps):
            assert cf == first and ni == n, ("pieces disagree", unit, ps)
            if p.schedule == "balanced":
                assert bx == first + i, ("pieces not in consecutive CTAs", unit, ps)
                assert kind == (2 if i == 0 else 1), ("piece kinds", unit, ps)
    return len(cover)
