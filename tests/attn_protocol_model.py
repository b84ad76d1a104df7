"""Executable model of the barrier protocol of round_attn_kernel (test infrastructure).

The roles of one CTA -- TMA producer, the two tcgen05 issuing threads, the ring
watcher and the eight softmax warps -- are written as Python generators that
keep the same counters and take the same waits, arrivals and commits, in the
same order, as csrc/wave_attn.cu. A seeded random scheduler interleaves them
with the asynchronous parts: TMA copies land after a random delay, and one
in-order tensor pipe executes MMAs and commits.

mbarriers follow the hardware's phase rules: an arrival counts toward the
current phase, the phase completes when its count is reached, and a parity wait
passes as soon as the completed-phase count has the other parity than the one
waited for. Each wait also records which phase its role meant. The model
reports:
- "early": a wait that passed before that phase had completed (parity aliasing);
- "stall": no role or event can make progress before every role has finished;
- data hazards: an S MMA overwriting an S tile some softmax warp has not loaded;
  a softmax warp loading another tile's S; an MMA reading a K/V slot that does
  not hold its page; P or O read or written at the wrong page; a copy landing
  in a slot an MMA still has to read.

``protocol="original"`` models the protocol before the single-tile fix: both
MMA threads wait for Q_FULL, and the second one, after skipping a single-tile
item, takes its next S_FREE_0 parity wait without first waiting for the
watcher's page count. ``protocol="lean-watcher"`` is the current protocol with
the watcher joining each S_FREE / P_FULL phase without first waiting for the
previous phase to complete (those waits are implied by its other waits).
"""
from __future__ import annotations

import random
from dataclasses import dataclass, field

RING_SLOTS = 5     # d = 128 (the d = 64 kernel has 10)
ITEM_SLOTS = 2
SOFTMAX_WARPS = 4  # per warpgroup


class Violation(Exception):
    pass


class Bar:
    """An mbarrier: `count` arrivals complete a phase."""

    def __init__(self, name: str, count: int):
        self.name, self.count = name, count
        self.done = 0          # completed phases
        self.pending = count   # arrivals still missing in the current phase

    def arrive(self, n: int = 1):
        if n > self.pending:
            raise Violation(f"{self.name}: {n} arrivals into a phase missing {self.pending}")
        self.pending -= n
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def parity_passes(self, phase: int) -> bool:
        """What `mbarrier.try_wait.parity` with the parity of `phase` returns."""
        return (self.done & 1) != (phase & 1)


@dataclass
class Item:
    id: int
    n: int       # key pages
    two: bool    # two query tiles (else one)


@dataclass
class State:
    items: list
    rng: random.Random
    protocol: str = "current"
    slots: int = RING_SLOTS
    bars: dict = field(default_factory=dict)
    item_q: list = field(default_factory=lambda: [None] * ITEM_SLOTS)
    s_done: int = 0
    # data
    ring: list = field(default_factory=list)          # per slot: (kind, page, landed)
    ring_readers: list = field(default_factory=list)  # per slot: MMAs queued on it
    q_buf: object = None                  # (item id, landed)
    s_buf: object = None                  # (tile, page)
    s_loaded: set = field(default_factory=set)
    p_buf: list = field(default_factory=lambda: [dict(), dict()])   # warp -> page
    p_queued: list = field(default_factory=lambda: [0, 0])         # P.V queued on P_w
    o_pages: list = field(default_factory=lambda: [0, 0])
    o_read: list = field(default_factory=lambda: [True, True])
    pipe: list = field(default_factory=list)
    copies: list = field(default_factory=list)   # [delay, action]
    early: list = field(default_factory=list)    # (role, barrier) of early passes

    def bar(self, name):
        return self.bars[name]


def make_bars(slots: int = RING_SLOTS):
    b = {}
    def add(name, count):
        b[name] = Bar(name, count)
    add("Q_FULL", 1)
    add("Q_EMPTY", 1)
    for w in range(2):
        add(f"S_FULL{w}", 1)
        add(f"S_FREE{w}", SOFTMAX_WARPS + 1)
        add(f"P_FULL{w}", SOFTMAX_WARPS + 1)
        add(f"P_FREE{w}", 1)
        add(f"O_FULL{w}", 1)
        add(f"O_EMPTY{w}", SOFTMAX_WARPS)
    for k in range(ITEM_SLOTS):
        add(f"ITEM_FULL{k}", 1)
        add(f"ITEM_EMPTY{k}", 3 + 2 * SOFTMAX_WARPS)
    for s in range(slots):
        add(f"RING_FULL{s}", 1)
        add(f"RING_EMPTY{s}", 2)
    return b


# ---------------------------------------------------------------- asynchronous parts

def copy(st: State, action):
    st.copies.append([st.rng.randint(1, 12), action])


def mma(st: State, op):
    st.pipe.append([st.rng.randint(1, 4), op])


def commit(st: State, bar_name):
    st.pipe.append([1, ("commit", bar_name)])


def execute(st: State, op):
    kind = op[0]
    if kind == "commit":
        st.bar(op[1]).arrive()
    elif kind == "S":
        _, w, page, item = op
        if st.s_buf is not None and len(st.s_loaded) < SOFTMAX_WARPS:
            raise Violation(f"S_{w}({page}) overwrites S{st.s_buf} loaded by {len(st.s_loaded)} warps")
        slot = (2 * page) % st.slots
        if st.ring[slot] != ("K", page, True):
            raise Violation(f"S_{w}({page}) reads K slot {slot} holding {st.ring[slot]}")
        st.ring_readers[slot] -= 1
        if st.q_buf != (item, True):
            raise Violation(f"S_{w}({page}) of item {item} reads Q {st.q_buf}")
        st.s_buf, st.s_loaded = (w, page), set()
    elif kind == "PV":
        _, w, page, acc = op
        slot = (2 * page + 1) % st.slots
        if st.ring[slot] != ("V", page, True):
            raise Violation(f"PV_{w}({page}) reads V slot {slot} holding {st.ring[slot]}")
        st.ring_readers[slot] -= 1
        if any(pg != page for pg in st.p_buf[w].values()) or len(st.p_buf[w]) < SOFTMAX_WARPS:
            raise Violation(f"PV_{w}({page}) reads P_{w} {st.p_buf[w]}")
        st.p_queued[w] -= 1
        if not acc:
            if not st.o_read[w]:
                raise Violation(f"PV_{w}({page}) starts O_{w} before the epilogue read it")
            st.o_pages[w], st.o_read[w] = 0, False
        st.o_pages[w] += 1


# ---------------------------------------------------------------- roles

def wait(bar: str, phase: int):
    return ("bar", bar, phase)


def producer(st: State):
    r = it = 0
    k = 0
    while True:
        slot = k % ITEM_SLOTS
        if k >= ITEM_SLOTS:
            yield wait(f"ITEM_EMPTY{slot}", k // ITEM_SLOTS - 1)
        w = st.items[k] if k < len(st.items) else None
        st.item_q[slot] = w
        st.bar(f"ITEM_FULL{slot}").arrive()
        if w is None:
            return
        if it > 0:
            yield wait("Q_EMPTY", it - 1)
        st.q_buf = (w.id, False)

        def q_lands(item=w.id):
            st.q_buf = (item, True)
            st.bar("Q_FULL").arrive()
        copy(st, q_lands)
        it += 1
        for _ in range(w.n):
            for kind in ("K", "V"):
                s = r % st.slots
                if r >= st.slots:
                    yield wait(f"RING_EMPTY{s}", r // st.slots - 1)
                if st.ring_readers[s]:
                    raise Violation(f"copy into slot {s} with {st.ring_readers[s]} MMAs to read it")
                page = r // 2
                st.ring[s] = (kind, page, False)

                def lands(s=s, kind=kind, page=page):
                    st.ring[s] = (kind, page, True)
                    st.bar(f"RING_FULL{s}").arrive()
                copy(st, lands)
                r += 1
        k += 1


def next_item(st: State, k: int):
    yield wait(f"ITEM_FULL{k % ITEM_SLOTS}", k // ITEM_SLOTS)
    w = st.item_q[k % ITEM_SLOTS]
    st.bar(f"ITEM_EMPTY{k % ITEM_SLOTS}").arrive()
    return w


def watcher(st: State):
    g = 0
    sf, pf = [0, 0], [0, 0]

    def next_phase(base, q, n):
        if n[q] > 0 and st.protocol != "lean-watcher":
            yield wait(f"{base}{q}", n[q] - 1)
        st.bar(f"{base}{q}").arrive()
        n[q] += 1
    k = 0
    while True:
        w = yield from next_item(st, k)
        if w is None:
            return
        nq = 2 if w.two else 1
        for t in range(w.n):
            for q in range(nq):
                if q == nq - 1 and t + 1 < w.n:
                    yield wait(f"RING_FULL{(2 * g + 2) % st.slots}", (2 * g + 2) // st.slots)
                yield from next_phase("S_FREE", q, sf)
            yield wait(f"S_FREE{nq - 1}", sf[nq - 1] - 1)
            st.s_done = g + 1
            st.bar(f"RING_EMPTY{(2 * g) % st.slots}").arrive(2)
            yield wait(f"RING_FULL{(2 * g + 1) % st.slots}", (2 * g + 1) // st.slots)
            for q in range(nq):
                yield from next_phase("P_FULL", q, pf)
            g += 1
        k += 1


def issuer(st: State, mw: int):
    g = it = pv = itw = 0
    sc = [0, 0]
    s_last = -1
    resync = False

    def take_s(w):
        nonlocal s_last
        sc[w] += 1
        s_last = w

    def issue_s(t, item):
        if s_last >= 0:
            yield wait(f"S_FREE{s_last}", sc[s_last] - 1)
        st.ring_readers[(2 * t) % st.slots] += 1
        mma(st, ("S", mw, t, item))
        commit(st, f"S_FULL{mw}")
        take_s(mw)

    def issue_pv(t, acc):
        nonlocal pv
        yield wait(f"P_FULL{mw}", pv)
        if not acc and itw > 0:
            yield wait(f"O_EMPTY{mw}", itw - 1)
        st.ring_readers[(2 * t + 1) % st.slots] += 1
        st.p_queued[mw] += 1
        mma(st, ("PV", mw, t, acc))
        commit(st, f"P_FREE{mw}")
        pv += 1

    def release_v(t, nq):
        commit(st, f"RING_EMPTY{(2 * t + 1) % st.slots}")
        if nq == 1:
            commit(st, f"RING_EMPTY{(2 * t + 1) % st.slots}")
    k = 0
    while True:
        w = yield from next_item(st, k)
        k += 1
        if w is None:
            return
        n, nq = w.n, 2 if w.two else 1
        qit = it
        it += 1
        if mw >= nq:
            for _ in range(n):
                take_s(0)
            g += n
            resync = st.protocol != "original"
            continue
        if mw == 0 or st.protocol == "original":
            yield wait("Q_FULL", qit)
        if resync:
            yield ("until", lambda need=g: st.s_done >= need)
            resync = False
        for j in range(n):
            if mw == 1:
                take_s(0)
            if mw == 0 and j == 0:
                yield wait(f"RING_FULL{(2 * g) % st.slots}", (2 * g) // st.slots)
            yield from issue_s(g, w.id)
            if mw == nq - 1 and j == n - 1:
                commit(st, "Q_EMPTY")
            if mw == 0 and nq == 2:
                take_s(1)
            if j > 0:
                yield from issue_pv(g - 1, j > 1)
                release_v(g - 1, nq)
            g += 1
        yield from issue_pv(g - 1, n > 1)
        commit(st, f"O_FULL{mw}")
        release_v(g - 1, nq)
        itw += 1


def softmax_warp(st: State, wq: int, warp: int):
    g = pw = it = gp = 0
    k = 0
    while True:
        w = yield from next_item(st, k)
        k += 1
        if w is None:
            return
        if wq == 1 and not w.two:
            gp += w.n
            continue
        for t in range(w.n):
            yield wait(f"S_FULL{wq}", g)
            if st.s_buf != (wq, gp):
                raise Violation(f"softmax {wq}.{warp} loads S{st.s_buf}, wants ({wq}, {gp})")
            st.s_loaded.add(warp)
            st.bar(f"S_FREE{wq}").arrive()
            grow = t > 0 and st.rng.random() < 0.3
            p_free = pw == 0
            if grow:
                yield wait(f"P_FREE{wq}", pw - 1)
                p_free = True
                if st.p_queued[wq]:
                    raise Violation(f"softmax {wq}.{warp} rescales O_{wq} under a queued P.V")
            if not p_free:
                yield wait(f"P_FREE{wq}", pw - 1)
            if st.p_queued[wq]:
                raise Violation(f"softmax {wq}.{warp} writes P_{wq} under a queued P.V")
            st.p_buf[wq][warp] = gp
            st.bar(f"P_FULL{wq}").arrive()
            pw += 1
            g += 1
            gp += 1
        yield wait(f"O_FULL{wq}", it)
        if st.o_pages[wq] != w.n:
            raise Violation(f"epilogue {wq} reads O of {st.o_pages[wq]} pages, item has {w.n}")
        st.bar(f"O_EMPTY{wq}").arrive()
        if st.bar(f"O_EMPTY{wq}").pending == SOFTMAX_WARPS:  # the phase just completed
            st.o_read[wq] = True
        it += 1


# ---------------------------------------------------------------- scheduler

def run(items, seed: int, protocol: str = "current", early_fatal: bool = True,
        slots: int = RING_SLOTS, max_steps: int = 200000):
    """Interleave every role and event at random until all roles finish.
    Raises Violation on a stall or a data hazard, and on an early pass unless
    ``early_fatal`` is False (then early passes are listed in ``state.early``)."""
    st = State(items=list(items), rng=random.Random(seed), protocol=protocol, slots=slots)
    st.ring, st.ring_readers = [None] * slots, [0] * slots
    st.bars = make_bars(slots)
    roles = {"producer": producer(st), "issuer0": issuer(st, 0), "issuer1": issuer(st, 1),
             "watcher": watcher(st)}
    for wq in range(2):
        for warp in range(SOFTMAX_WARPS):
            roles[f"softmax{wq}.{warp}"] = softmax_warp(st, wq, warp)
    waiting = {name: None for name in roles}   # None: runnable

    def ready(name):
        cond = waiting[name]
        if cond is None:
            return True
        if cond[0] == "until":
            return cond[1]()
        return st.bar(cond[1]).parity_passes(cond[2])

    for _ in range(max_steps):
        choices = [("role", n) for n in roles if ready(n)]
        choices += [("copy", i) for i in range(len(st.copies))]
        if st.pipe:
            choices.append(("pipe", 0))
        if not choices:
            if roles:
                raise Violation("stall: " + ", ".join(f"{n} on {waiting[n]}" for n in roles))
            return st
        kind, x = st.rng.choice(choices)
        if kind == "copy":
            ev = st.copies[x]
            ev[0] -= 1
            if ev[0] == 0:
                st.copies.pop(x)
                ev[1]()
        elif kind == "pipe":
            head = st.pipe[0]
            head[0] -= 1
            if head[0] == 0:
                st.pipe.pop(0)
                execute(st, head[1])
        else:
            cond = waiting[x]
            if cond is not None and cond[0] == "bar" and st.bar(cond[1]).done <= cond[2]:
                msg = (f"early: {x} passed {cond[1]} phase {cond[2]} "
                       f"with {st.bar(cond[1]).done} phases complete")
                if early_fatal:
                    raise Violation(msg)
                st.early.append((x, cond[1]))
            try:
                waiting[x] = next(roles[x])
            except StopIteration:
                del roles[x]
                del waiting[x]
    raise Violation("step limit")


def random_items(rng: random.Random, count: int, max_pages: int = 4, p_single: float = 0.4):
    return [Item(i, rng.randint(1, max_pages), rng.random() >= p_single) for i in range(count)]
