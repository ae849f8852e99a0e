"""Model check of the forward's work queue (CPU).

The persistent forward's CTAs take their first work item by index.  They take
the rest from a 64-bit word in a small device array (shared by all launches
on a device), picked by the launch's number modulo the array size.  The word
packs:
- the claiming launch's 24-bit identity;
- a DONE bit;
- a 9-bit count of the CTAs taking items;
- a 30-bit counter.

This file restates the device function's steps (one atomic access per step)
and the host's choice of identities.  A seeded random scheduler runs the CTAs
of several launches, interleaving every access.  The checks:
- every launch processes every one of its items;
- a launch that hands items out by the counter hands each out once, even when
  one of its CTAs starts after the hand-out is over (it must recognise its own
  launch's finished word rather than claim the word again);
- no CTA ever draws from a counter claimed by another launch;
- no CTA gets stuck;
- the word is left free (zero, or DONE with no takers).

The scenarios:
- one launch;
- launches with different identities sharing one word at the same time (more
  launches in flight than words);
- identities that agree in their low 16 bits.

The host rule also gets a check: a launch that will use the queue never
receives the identity of the last launch that used the same word, even across
the 24-bit wrap.  So a finished word with a launch's own identity can only be
its own hand-out.
"""
import random

import pytest

COUNT = (1 << 30) - 1
TAKER = 1 << 30
TAKERS = 0x1FF << 30
DONE = 1 << 39
M64 = (1 << 64) - 1


def is_free(w):
    return w == 0 or ((w & DONE) != 0 and (w & TAKERS) == 0)


class Word:
    def __init__(self, value=0):
        self.v = value


def cta(word, ticket, total, grid, b, rec, rng):
    """One CTA of a launch: yields between atomic accesses; records in rec the
    items it processes and, for each counter draw, the launch identity the word
    held at that moment.  `ticket` is the launch's 24-bit identity."""
    yield
    rec["items"].append(b)             # first item: its index
    for _ in range(rng.randint(0, 6)):
        yield
    mode, next_fixed, tries = "undecided", 0, 0
    while True:
        item = None
        while mode == "undecided":
            tries += 1
            if tries > 4096:
                rec["stuck"] = True
                return
            w = word.v
            yield
            own = w != 0 and (w >> 40) == ticket
            if is_free(w):
                if own:
                    mode = "finished"  # this launch's hand-out is over
                    break
                want = (ticket << 40) | TAKER | (grid + 1)
                if word.v != w:        # compare and swap
                    yield
                    continue
                word.v = want
                yield
                mode = "taking"
                rec["draws"].append(ticket)
                if grid + 1 >= total:
                    word.v |= DONE
                    yield
                    word.v = (word.v - TAKER) & M64
                    yield
                    mode = "finished"
                item = grid
                break
            if own:
                if w & DONE:
                    mode = "finished"
                    break
                old = word.v            # atomic add of one taker
                word.v = (old + TAKER) & M64
                yield
                if old != 0 and (old >> 40) == ticket and not (old & DONE):
                    mode = "taking"
                else:
                    word.v = (word.v - TAKER) & M64
                    yield
                continue
            mode = "fixed"
            next_fixed = b + grid
        if item is None:
            if mode == "taking":
                old = word.v            # atomic add of one to the counter
                word.v = (old + 1) & M64
                rec["draws"].append(old >> 40)
                yield
                c = old & COUNT
                if c < total:
                    item = c
                else:
                    if c == total:
                        word.v |= DONE
                        yield
                    word.v = (word.v - TAKER) & M64
                    yield
                    mode = "finished"
            elif mode == "fixed":
                it = next_fixed
                next_fixed += grid
                if it < total:
                    item = it
                else:
                    mode = "finished"
        if item is None:
            return
        rec["items"].append(item)
        for _ in range(rng.randint(0, 6)):
            yield


def run(launches, seed, word=None, late=None):
    """launches: list of (ticket, total, grid, start_tick).  Returns per-launch
    records and the word."""
    rng = random.Random(seed)
    word = word or Word()
    recs = [{"items": [], "draws": [], "stuck": False} for _ in launches]
    pending = []
    for li, (ticket, total, grid, start) in enumerate(launches):
        for b in range(grid):
            delay = late if (late is not None and li == 0 and b == grid - 1) else rng.randint(0, 3)
            pending.append((start + delay, li, b))
    live, tick = [], 0
    while pending or live:
        tick += 1
        for p in [p for p in pending if p[0] <= tick]:
            pending.remove(p)
            _, li, b = p
            ticket, total, grid, _ = launches[li]
            live.append(cta(word, ticket, total, grid, b, recs[li], rng))
        rng.shuffle(live)
        for g in list(live):
            if rng.random() < 0.3:
                continue
            try:
                next(g)
            except StopIteration:
                live.remove(g)
        assert tick < 200000, "no progress"
    return recs, word


def check(launches, recs, word):
    for (ticket, total, grid, _), r in zip(launches, recs):
        assert not r["stuck"]
        assert set(r["items"]) == set(range(total)), (ticket, sorted(set(range(total)) - set(r["items"])))
        # every draw from a counter was from this launch's own claim
        assert all(t == ticket for t in r["draws"]), (ticket, r["draws"][:5])
    assert is_free(word.v), hex(word.v)


@pytest.mark.parametrize("grid,total", [(1, 2), (3, 4), (3, 10), (8, 9), (8, 45), (16, 200)])
def test_one_launch_hands_every_item_out_once(grid, total):
    for seed in range(150):
        launches = [(5, total, grid, 0)]
        recs, word = run(launches, seed)
        check(launches, recs, word)
        # handed out by the counter: no item twice
        assert sorted(recs[0]["items"]) == list(range(total)), seed


def test_concurrent_launches_sharing_one_word():
    rng = random.Random(99)
    for seed in range(300):
        launches = [(t, rng.randint(2, 60), rng.randint(1, 12), rng.randint(0, 40)) for t in (1, 2, 3)]
        launches = [(t, max(total, grid + 1), grid, s) for t, total, grid, s in launches]
        recs, word = run(launches, seed)
        check(launches, recs, word)


def test_identities_equal_in_their_low_16_bits_take_the_word_over():
    """A launch 65536 launches after another on the same word agrees with it in
    the low 16 bits of its identity but not in the top 8: it must hand out all
    its items through the counter."""
    for seed in range(200):
        first = [(7, 30, 6, 0)]
        recs, word = run(first, seed)
        check(first, recs, word)
        again = [(7 | (1 << 16), 41, 8, 0)]
        recs, word = run(again, seed + 1000, word)
        check(again, recs, word)
        assert sorted(recs[0]["items"]) == list(range(41))


def test_a_cta_that_starts_after_the_hand_out_does_not_repeat_it():
    """One CTA of a launch starts after the launch's other CTAs have drawn every
    item (its SM was busy): it must find its own launch's finished word and
    stop after its first item, not claim the word and redo the rest alone."""
    for seed in range(200):
        launches = [(11, 60, 6, 0)]
        recs, word = run(launches, seed, late=5000)
        check(launches, recs, word)
        assert sorted(recs[0]["items"]) == list(range(60)), seed


class Host:
    """The host's choice of a launch's identity and word: a per-device launch
    number; the word is the number modulo `slots`, the identity its low 24
    bits, and a launch that will use the queue skips a number whose identity
    equals that of the last queue user of its word."""

    def __init__(self, slots, start=0):
        self.slots, self.serial, self.last = slots, start, {}

    def launch(self, uses_queue):
        while True:
            n = self.serial
            self.serial += 1
            slot, ident = n % self.slots, n & 0xFFFFFF
            if not uses_queue:
                return slot, ident
            if self.last.get(slot) != ident:
                self.last[slot] = ident
                return slot, ident


def test_host_never_repeats_the_last_queue_users_identity_on_a_word():
    rng = random.Random(3)
    for slots in (1, 2, 64):
        # start just below the 24-bit wrap, with a history of queue users
        host = Host(slots, start=(1 << 24) - 3 * slots)
        last_user = {}
        for _ in range(20 * slots + 100):
            uses = rng.random() < 0.3
            slot, ident = host.launch(uses)
            if uses:
                assert last_user.get(slot) != ident
                last_user[slot] = ident
    # the exact case: the only queue user on a word 2^24 launches ago
    host = Host(1)
    assert host.launch(True) == (0, 0)
    for _ in range((1 << 24) - 1):
        host.serial += 1  # launches that do not use the queue
    slot, ident = host.launch(True)
    assert ident != 0


def test_many_launches_in_sequence_and_overlapping():
    """Rounds of one to four launches on one word, identities from the host's
    rule (starting near the 24-bit wrap), each round starting on the word the
    last one left."""
    rng = random.Random(5)
    for seed in range(100):
        word = Word()
        host = Host(1, start=(1 << 24) - rng.randint(1, 8))
        for rnd in range(4):
            launches = []
            for _ in range(rng.randint(1, 4)):
                grid = rng.randint(1, 10)
                total = max(rng.randint(2, 40), grid + 1)
                launches.append((host.launch(True)[1], total, grid, rng.randint(0, 20)))
            recs, word = run(launches, seed * 10 + rnd, word)
            check(launches, recs, word)


# ---------------------------------------------------------------------------
# Exhaustive search over small scopes.  Each CTA is a small state machine over
# the same steps as `cta` above (each atomic access of the word one step; a
# CTA's start -- when it takes its first item and, in the earlier form, reads
# its snapshot of the word -- is a step too, so every start order, late starts
# included, is explored).  Every interleaving of the CTAs of one or two
# launches on one word is visited.  Checked in every terminal state: each
# launch processed every item; a launch none of whose CTAs fell back to the
# fixed order processed no item twice; no draw came from another launch's
# counter; the word is free.  (With two launches on one word, a CTA that starts
# after its own launch's hand-out AND another launch's later hand-out on the
# same word are both over finds a free word of another identity and hands its
# launch's items out again: identical results, only repeated work.  With 64
# words the other launch is 64 launches later, so this is checked for single
# launches only.)  The earlier form ("snapshot": a 16-bit ticket
# and a claim epoch, a free word with the launch's own ticket taken for its own
# only if it differs from the CTA's snapshot) is kept as a mutant: the search
# must find its late-start double hand-out.

def explore(launches, protocol="identity", word0=0, allow_repeats=False):
    """launches: list of (identity, total, grid).  Returns None or a failure."""
    (START, READ, DECIDE, CAS, JOIN_ADD, JOIN_UNDO, DRAW, OR_DONE_LAST, LEAVE_LAST,
     OR_DONE_CLAIM, LEAVE_CLAIM, FIXED, END) = range(13)
    snapshot = protocol == "snapshot"
    shift = 48 if snapshot else 40
    ctas = [(li, b) for li, (_, _, grid) in enumerate(launches) for b in range(grid)]
    # CTA: (pc, next_fixed, w (value read / old value), snap, items, n_items, draws_ok, fixed)
    init = (word0, tuple((START, 0, 0, 0, frozenset(), 0, True, False) for _ in ctas))
    seen, stack = {init}, [init]
    terminal = 0
    while stack:
        word, cs = stack.pop()
        moved = False
        for k, (li, b) in enumerate(ctas):
            ident, total, grid = launches[li]
            pc, nf, w, snap, items, n_items, ok, fixed = cs[k]
            if pc == END:
                continue
            nw = word
            npc, nnf, nwv, nsnap, nitems, nn, nok, nfixed = pc, nf, w, snap, items, n_items, ok, fixed

            def take(item):
                return items | {item}, n_items + 1

            if pc == START:
                nsnap = word
                nitems, nn = take(b)
                npc = READ
            elif pc == READ:
                nwv, npc = word, DECIDE
            elif pc == DECIDE:
                own = w != 0 and (w >> shift) == ident
                if is_free(w):
                    if own and (not snapshot or w != snap):
                        npc = END
                    else:
                        npc = CAS
                elif own:
                    npc = END if (w & DONE) else JOIN_ADD
                else:
                    npc, nnf, nfixed = FIXED, b + grid, True
            elif pc == CAS:
                if word != w:
                    npc = READ
                else:
                    ep = (((w >> 40) + 1) & 0xFF) << 40 if snapshot else 0
                    nw = (ident << shift) | ep | TAKER | (grid + 1)
                    nitems, nn = take(grid)
                    npc = OR_DONE_CLAIM if grid + 1 >= total else DRAW
            elif pc == OR_DONE_CLAIM:
                nw, npc = word | DONE, LEAVE_CLAIM
            elif pc == LEAVE_CLAIM:
                nw, npc = (word - TAKER) & M64, END
            elif pc == JOIN_ADD:
                old = word
                nw = (old + TAKER) & M64
                if old != 0 and (old >> shift) == ident and not (old & DONE):
                    npc = DRAW
                else:
                    npc = JOIN_UNDO
            elif pc == JOIN_UNDO:
                nw, npc = (word - TAKER) & M64, READ
            elif pc == DRAW:
                old = word
                nw = (old + 1) & M64
                if (old >> shift) != ident:
                    nok = False
                c = old & COUNT
                if c < total:
                    nitems, nn = take(c)
                elif c == total:
                    npc = OR_DONE_LAST
                else:
                    npc = LEAVE_LAST
            elif pc == OR_DONE_LAST:
                nw, npc = word | DONE, LEAVE_LAST
            elif pc == LEAVE_LAST:
                nw, npc = (word - TAKER) & M64, END
            elif pc == FIXED:
                if nf < total:
                    nitems, nn = take(nf)
                    nnf = nf + grid
                else:
                    npc = END
            ncs = list(cs)
            ncs[k] = (npc, nnf, nwv, nsnap, nitems, nn, nok, nfixed)
            ns = (nw, tuple(ncs))
            moved = True
            if ns not in seen:
                seen.add(ns)
                stack.append(ns)
        if not moved:
            terminal += 1
            for li, (ident, total, grid) in enumerate(launches):
                mine = [cs[k] for k, (lj, _) in enumerate(ctas) if lj == li]
                got = set().union(*(c[4] for c in mine))
                if got != set(range(total)):
                    return "launch %d missed items %s" % (li, sorted(set(range(total)) - got))
                if not allow_repeats and not any(c[7] for c in mine) and sum(c[5] for c in mine) != total:
                    return "launch %d handed items out twice (%d for %d)" % (li, sum(c[5] for c in mine), total)
                if not all(c[6] for c in mine):
                    return "launch %d drew from another launch's counter" % li
            if not is_free(word):
                return "word left held: %x" % word
    return None if terminal else "no terminal state"


SMALL_SCOPES = [[(1, 2, 1)], [(1, 3, 2)], [(1, 4, 2)], [(1, 5, 3)], [(1, 6, 3)]]
TWO_LAUNCHES = [[(1, 2, 1), (2, 2, 1)], [(1, 3, 2), (2, 2, 1)], [(1, 3, 1), (2, 3, 1)], [(1, 2, 1), (2, 4, 2)]]


@pytest.mark.parametrize("launches", SMALL_SCOPES)
def test_every_interleaving_of_one_launch_hands_each_item_out_once(launches):
    assert explore(launches) is None, launches


@pytest.mark.parametrize("launches", TWO_LAUNCHES)
def test_every_interleaving_of_two_launches_on_one_word(launches):
    assert explore(launches, allow_repeats=True) is None, launches


@pytest.mark.parametrize("launches", SMALL_SCOPES[:4])
def test_every_interleaving_from_a_word_an_older_launch_left(launches):
    """The word starts as an older launch left it: free (DONE, no takers) with
    another identity, or with the same low 16 bits of identity."""
    for word0 in ((9 << 40) | DONE | 7, ((launches[0][0] | (1 << 16)) << 40) | DONE | 3):
        assert explore(launches, word0=word0) is None, (launches, hex(word0))


def test_the_snapshot_form_hands_items_out_twice_after_a_late_start():
    """The earlier form: some interleaving (a CTA starting after its launch's
    hand-out is over) hands items out a second time."""
    found = [explore(launches, protocol="snapshot") for launches in SMALL_SCOPES]
    assert any(r and "twice" in r for r in found), found
