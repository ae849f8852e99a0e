"""Model check of the forward's O staging-turn protocol (CPU).

The persistent forward gives each work item two 128-row Q tiles, and their 16
softmax warps (8 per tile) share one shared-memory staging tile for O.  The
turns go tile 0, tile 1, item after item.  In its turn, each warp of the tile
writes its rows.  The last of the 8 warps (counted in shared memory) resets the
count and issues the TMA store.  When the store has read the tile, that thread
arrives on a turn barrier.  A tile that lies past N writes nothing, but its
last warp still passes the turn on.

This file models that protocol step by step, with these parts:
- mbarrier phases (count 1);
- parity waits with the hardware's semantics: a wait on parity p succeeds once
  the phase of that parity before the current one is complete, so a waiter two
  phases ahead of the barrier cannot be told from one zero phases ahead;
- asynchronous stores;
- the o_free dependency, under which a tile's warps cannot finish the next
  item's work before all 8 have written their rows for the previous one.

A seeded random scheduler interleaves the warps and stores, with random delays
and now and then a long stall of one of them.
The checks:
- no warp writes the tile while another turn's writes or store are in flight;
- every turn is stored exactly once;
- nothing deadlocks.

The protocol the kernel uses waits on one barrier per tile (stg_done[t ^ 1],
phase n of the other tile's turns), and must pass every run.  The earlier
protocol used one barrier for both tiles (parity t ^ 1), and some run must
catch it writing over a store in flight.  That race was found on the GPU only
under timing stress.
"""
import random

import pytest


class Barrier:
    """An mbarrier whose phases complete on one arrival."""

    def __init__(self):
        self.phase = 0  # index of the phase in progress

    def arrive(self):
        self.phase += 1

    def test_wait(self, parity):
        # true once the phase of this parity before the current one is complete
        return parity != (self.phase & 1)


def simulate(protocol, items, seed, max_idle=600):
    """Runs one random interleaving.  items: list of (tile 0 has rows, tile 1 has
    rows) per item (tile 0 always does).  Returns (violation or None, turns
    stored or passed on, in order)."""
    rng = random.Random(seed)
    per_tile = protocol.startswith("per_tile")
    first_passes = protocol == "per_tile_first_passes"
    bars = [Barrier(), Barrier()] if per_tile else [Barrier()]
    passed = set()               # turns passed on (first_passes form)
    count = [0]                  # warps of the current turn done writing
    writers = {}                 # turn -> warps writing it now
    reading = set()              # turns whose store still reads the tile
    stored = []
    done_writes = {0: [0] * len(items), 1: [0] * len(items)}
    found = []

    def check(turn):
        others = [u for u, k in writers.items() if k > 0 and u != turn] + [u for u in reading if u != turn]
        if others and not found:
            found.append("turn %s touches the tile while %s is in flight" % (turn, sorted(others)))

    def turn_bar(t):
        return bars[t] if per_tile else bars[0]

    def wait_target(t, n, has_rows):
        if per_tile:
            return bars[t ^ 1], (n & 1) ^ t ^ 1
        return bars[0], (t ^ 1) if has_rows else 0

    def store(turn, t):
        for _ in range(rng.randint(1, 60)):
            yield "read"
        reading.discard(turn)
        stored.append(turn)
        turn_bar(t).arrive()

    def warp(t):
        for n, rows in enumerate(items):
            has_rows = rows[t]
            prev = [m for m in range(n) if items[m][t]]
            if has_rows and prev:
                # o_free: the tile's previous O has been read by all 8 warps
                while done_writes[t][prev[-1]] < 8:
                    yield "blocked"
            for _ in range(rng.randint(0, 30) if has_rows else rng.randint(0, 3)):
                yield "work"
            bar, parity = wait_target(t, n, has_rows)
            while not bar.test_wait(parity):
                yield "blocked"
            turn = (n, t)
            if not has_rows and first_passes:
                # the earlier pass-on: the first warp to see the tile free passes it on
                if turn not in passed:
                    passed.add(turn)
                    stored.append(turn)
                    turn_bar(t).arrive()
                yield "work"
                continue
            if has_rows:
                check(turn)
                writers[turn] = writers.get(turn, 0) + 1
                for _ in range(rng.randint(1, 8)):
                    yield "write"
                    check(turn)
                writers[turn] -= 1
                done_writes[t][n] += 1
            count[0] += 1
            if count[0] == 8:
                count[0] = 0
                if has_rows:
                    check(turn)
                    reading.add(turn)
                    pool.append(store(turn, t))
                else:
                    stored.append(turn)
                    turn_bar(t).arrive()
            yield "work"

    pool = [warp(t) for t in range(2) for _ in range(8)]
    asleep = {}                  # entity -> pass at which it runs again
    idle, tick = 0, 0
    while pool:
        tick += 1
        progressed = False
        order = list(pool)
        rng.shuffle(order)
        for g in order:
            if asleep.get(g, 0) > tick:
                continue
            if rng.random() < 0.3:
                continue  # uneven speeds
            if rng.random() < 0.004:
                asleep[g] = tick + rng.randint(20, 300)  # a long stall (descheduled, slow memory)
                continue
            try:
                progressed |= next(g) != "blocked"
            except StopIteration:
                pool.remove(g)
                progressed = True
        idle = 0 if progressed else idle + 1
        if idle > max_idle:
            return (found[0] if found else "deadlock: every warp and store blocked"), stored
    return (found[0] if found else None), stored


def _workloads(rng, n):
    out = []
    for _ in range(n):
        items = [(True, rng.random() < 0.75) for _ in range(rng.randint(2, 7))]
        out.append(items)
    return out


def test_per_tile_turn_barriers_never_overlap_and_never_deadlock():
    rng = random.Random(2024)
    for k, items in enumerate(_workloads(rng, 300)):
        violation, stored = simulate("per_tile", items, seed=k)
        assert violation is None, (items, violation)
        # every turn (tile 0 and tile 1 of every item) is stored or passed on once, in order
        assert stored == [(n, t) for n in range(len(items)) for t in (0, 1)], (items, stored)


def test_one_shared_barrier_is_caught_writing_over_a_store_in_flight():
    """The earlier form: both tiles wait on one barrier by parity t ^ 1.  A fast
    warp whose previous turn is not yet stored sees the phase two before its
    own as complete.  The model must find such an interleaving."""
    rng = random.Random(7)
    found = None
    for k, items in enumerate(_workloads(rng, 300)):
        violation, _ = simulate("shared", items, seed=k)
        if violation and "in flight" in violation:
            found = (items, violation)
            break
    assert found is not None


def test_turn_passed_on_by_the_first_warp_deadlocks():
    """The first form of the pass-on for a tile past N: the first of its warps to
    see the tile free passes the turn on.  A slower warp of that tile then
    meets the phase after the one it waits for, waits for a later phase, and the
    next item needs it: the model must find the deadlock (on the GPU a bounded
    wait expired)."""
    items = [(True, False), (True, True), (True, True), (True, False), (True, True)]
    outcomes = [simulate("per_tile_first_passes", items, seed=k)[0] for k in range(200)]
    assert any(o and o.startswith("deadlock") for o in outcomes)


@pytest.mark.parametrize("items", [
    [(True, False)] * 6,                  # every item's tile 1 past N: pass-ons only
    [(True, True)] * 6,                   # both tiles with rows throughout
    [(True, False), (True, True)] * 3,    # alternating
])
def test_per_tile_protocol_on_fixed_item_mixes(items):
    for seed in range(200):
        violation, stored = simulate("per_tile", items, seed=seed)
        assert violation is None, (seed, violation)
        assert stored == [(n, t) for n in range(len(items)) for t in (0, 1)]


# ---------------------------------------------------------------------------
# Exhaustive search over small scopes: every interleaving of W warps per tile
# and the stores, for short item sequences (the random runs above sample the
# 8-warp case).  A state is (warp states, barrier phases, turn count, writers,
# stores reading, warps done writing per item, turns passed on); every enabled
# step of every warp or store is explored.  Checked in every reachable state:
# no warp enters or stays in a turn's writes, and no store starts, while
# another turn's writes or store are in flight; a state with no enabled step
# is the end (every turn stored or passed on once, in order) and not a
# deadlock.

def explore(protocol, items, W=2):
    per_tile = protocol.startswith("per_tile")
    first_passes = protocol == "per_tile_first_passes"
    nbar = 2 if per_tile else 1
    M = len(items)
    OFREE, WAIT, WRITE, INC, END = range(5)

    def bar_of(t):
        return t if per_tile else 0

    def wait_of(t, n, rows):
        if per_tile:
            return t ^ 1, (n & 1) ^ t ^ 1
        return 0, (t ^ 1) if rows else 0

    # state: warps (tuple of (n, phase) per warp, t = i // W), phases, count,
    # writers (tuple of (turn, k)), reading (frozenset of turns), done (tuple per
    # tile of per-item counts), passed (frozenset), stored (tuple of turns)
    start = (tuple((0, OFREE) for _ in range(2 * W)), (0,) * nbar, 0, (), frozenset(),
             ((0,) * M, (0,) * M), frozenset(), ())
    seen, stack = {start}, [start]
    while stack:
        st = stack.pop()
        warps, phases, count, writers, reading, done, passed, stored = st
        wr = dict(writers)
        succ = []

        def other_active(turn):
            return any(k > 0 and u != turn for u, k in wr.items()) or any(u != turn for u in reading)

        for i, (n, ph) in enumerate(warps):
            t = i // W
            if ph == END:
                continue
            rows = items[n][t]
            turn = (n, t)
            nxt = (n + 1, OFREE) if n + 1 < M else (n + 1, END)
            if ph == OFREE:
                prev = [m for m in range(n) if items[m][t]]
                if rows and prev and done[t][prev[-1]] < W:
                    continue
                succ.append((i, (n, WAIT), phases, count, wr, reading, done, passed, stored))
            elif ph == WAIT:
                b, parity = wait_of(t, n, rows)
                if parity == (phases[b] & 1):
                    continue  # that phase is not complete
                if not rows and first_passes:
                    if turn in passed:
                        succ.append((i, nxt, phases, count, wr, reading, done, passed, stored))
                    else:
                        ph2 = list(phases)
                        ph2[bar_of(t)] += 1
                        succ.append((i, nxt, tuple(ph2), count, wr, reading, done, passed | {turn},
                                     stored + (turn,)))
                    continue
                if rows:
                    if other_active(turn):
                        return "turn %s writes while another turn is in flight" % (turn,)
                    w2 = dict(wr)
                    w2[turn] = w2.get(turn, 0) + 1
                    succ.append((i, (n, WRITE), phases, count, w2, reading, done, passed, stored))
                else:
                    succ.append((i, (n, INC), phases, count, wr, reading, done, passed, stored))
            elif ph == WRITE:
                if other_active(turn):
                    return "turn %s writes while another turn is in flight" % (turn,)
                w2 = dict(wr)
                w2[turn] -= 1
                d2 = [list(done[0]), list(done[1])]
                d2[t][n] += 1
                succ.append((i, (n, INC), phases, count, w2, reading, (tuple(d2[0]), tuple(d2[1])), passed, stored))
            elif ph == INC:
                c = count + 1
                if c < W:
                    succ.append((i, nxt, phases, c, wr, reading, done, passed, stored))
                elif rows:
                    if any(k > 0 and u != turn for u, k in wr.items()):
                        return "turn %s's store starts while another turn writes" % (turn,)
                    succ.append((i, nxt, phases, 0, wr, reading | {turn}, done, passed, stored))
                else:
                    ph2 = list(phases)
                    ph2[bar_of(t)] += 1
                    succ.append((i, nxt, tuple(ph2), 0, wr, reading, done, passed, stored + (turn,)))
        for turn in reading:  # a store finishes reading: its turn ends
            ph2 = list(phases)
            ph2[bar_of(turn[1])] += 1
            succ.append((None, None, tuple(ph2), count, wr, reading - {turn}, done, passed, stored + (turn,)))
        if not succ:
            if all(ph == END for _, ph in warps) and not reading:
                if list(stored) != [(n, t) for n in range(M) for t in (0, 1)]:
                    return "turns ended out of order: %s" % (stored,)
                continue
            return "deadlock"
        for i, w_new, ph2, c2, w2, r2, d2, p2, s2 in succ:
            ws = list(warps)
            if i is not None:
                ws[i] = w_new
            ns = (tuple(ws), ph2, c2, tuple(sorted((u, k) for u, k in w2.items() if k)), r2, d2, p2, s2)
            if ns not in seen:
                seen.add(ns)
                stack.append(ns)
    return None


def _mixes(max_items):
    import itertools
    for m in range(1, max_items + 1):
        for rows1 in itertools.product((True, False), repeat=m):
            yield [(True, r) for r in rows1]


def test_per_tile_protocol_holds_in_every_interleaving_of_small_scopes():
    for items in _mixes(4):
        assert explore("per_tile", items) is None, items


def test_every_interleaving_search_finds_both_earlier_forms_wrong():
    shared = [explore("shared", items) for items in _mixes(3)]
    # the one-barrier form: from two items on, some interleaving overlaps a turn's
    # writes with another turn's store
    assert all((r is not None) == (len(items) > 1) for r, items in zip(shared, _mixes(3)))
    assert any(r and ("in flight" in r or "store starts" in r) for r in shared)
    first = [explore("per_tile_first_passes", items) for items in _mixes(4)]
    assert any(r == "deadlock" for r in first)
