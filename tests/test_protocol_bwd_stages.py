"""Model check of the backward's per-tile Q and dO stages (CPU).

The backward walks an item's query tiles T.  Each tile's Q_T, its LSE2 and D
vectors and its dO_T come into shared memory from the producer:
- Q and the vectors use a ring of two stages (tile T in stage T mod 2),
  released by the MMA warp's commit after the tile's dK product (the last
  MMA that reads Q_T).
- dO at d = 64 rides in the same stage under the same barrier.  Its readers,
  dP^T(T) issued at the end of the previous tile's step and dV(T) at the start
  of this one, are issued before that dK.
- dO at d = 128 has one buffer with its own barriers (released after dV(T);
  dP^T(T + 1) waits for its load).
The softmax warps read the vectors of stage T mod 2 while they form P(T)
(LSE2) and dS(T) (D).

This model restates, for both forms, the MMA warp's issue order per tile:
- dV(T);
- S^T(T + 1);
- dK(T), then the stage's release;
- dQ(T);
- dP^T(T + 1).
It runs the tensor pipe in order, the softmax and the producer as the code
has them, under a seeded random scheduler with long stalls.  It checks that
no load overwrites a stage (Q, vectors or dO) that an issued MMA or the
softmax still reads.  Mutants must be caught: releasing the stage after dV
instead of dK, and, at d = 64, dO in one buffer with no barrier of its own.
"""
import random

import pytest


class Bar:
    def __init__(self, count=1):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return parity != (self.phase & 1)


def simulate(n_tiles, seed, do_with_q=True, mutant=None, max_idle=800):
    rng = random.Random(seed)
    SMW = 2
    q_full = [Bar(), Bar()]
    q_empty = [Bar(), Bar()]
    do_full, do_empty = Bar(), Bar()
    s_full, dp_full, dq_full, dq_empty = Bar(), Bar(), Bar(), Bar()
    p_ready, dp_read, ds_ready = Bar(SMW), Bar(SMW), Bar(SMW)
    # buffers: ("Q", s), ("V", s) vectors, ("O", s) dO stage (d = 64) or ("O", 0) (d = 128)
    readers = {}
    writing = set()
    pipe, loads, ran, problems = [], [], set(), []
    do_single = (not do_with_q) or mutant == "do_single_no_bar"

    def dbuf(T):
        return ("O", 0) if do_single else ("O", T & 1)

    def read(buf, who):
        if buf in writing and not problems:
            problems.append("%s reads %s while a load writes it" % (who, buf))
        readers[buf] = readers.get(buf, 0) + 1

    def unread(buf):
        readers[buf] -= 1

    def wait(bar, parity):
        while not bar.done(parity):
            yield "blocked"

    def tensor_pipe():
        while True:
            if not pipe:
                yield "idle"
                continue
            op = pipe[0]
            if op[0] == "mma":
                for _ in range(rng.randint(1, 6)):
                    yield "work"
                for b in op[1]:
                    unread(b)
                ran.add(op[2])
            else:
                op[1].arrive()
            pipe.pop(0)
            yield "work"

    def issue(bufs, tag):
        for b in bufs:
            read(b, tag)
        pipe.append(("mma", bufs, tag))

    def commit(bar):
        pipe.append(("commit", bar))

    def loader():
        while True:
            if not loads:
                yield "idle"
                continue
            op = rng.choice(loads)
            if rng.random() < 0.2:
                loads.remove(op)
                for b in op[0]:
                    writing.discard(b)
                op[1].arrive()
            yield "work"

    def load(bufs, bar):
        for b in bufs:
            if readers.get(b, 0) and not problems:
                problems.append("load overwrites %s while %d readers remain" % (b, readers[b]))
            writing.add(b)
        loads.append((bufs, bar))

    def producer():
        for T in range(n_tiles):
            s = T & 1
            yield from wait(q_empty[s], ((T >> 1) & 1) ^ 1)
            bufs = [("Q", s), ("V", s)]
            if not do_single or mutant == "do_single_no_bar":
                bufs.append(dbuf(T))  # dO with Q, under the stage's barrier
            load(bufs, q_full[s])
            if do_single and mutant != "do_single_no_bar":
                yield from wait(do_empty, (T & 1) ^ 1)
                load([dbuf(T)], do_full)
            yield "work"

    def mma():
        yield from wait(q_full[0], 0)
        issue([("Q", 0)], "S0")
        commit(s_full)
        if do_single and mutant != "do_single_no_bar":
            yield from wait(do_full, 0)
        issue([dbuf(0)], "dP0")
        commit(dp_full)
        for T in range(n_tiles):
            s = T & 1
            more = T + 1 < n_tiles
            yield from wait(p_ready, T & 1)
            issue([dbuf(T)], "dV%d" % T)
            if mutant == "release_after_dv":
                commit(q_empty[s])
            if do_single and mutant != "do_single_no_bar":
                commit(do_empty)
            yield from wait(dp_read, T & 1)
            if more:
                yield from wait(q_full[(T + 1) & 1], ((T + 1) >> 1) & 1)
                issue([("Q", (T + 1) & 1)], "S%d" % (T + 1))
                commit(s_full)
            yield from wait(ds_ready, T & 1)
            issue([("Q", s)], "dK%d" % T)
            if mutant != "release_after_dv":
                commit(q_empty[s])
            if T > 0:
                # dQ's TMEM region: the dQ warps have read the previous tile's dQ out
                yield from wait(dq_empty, (T - 1) & 1)
            issue([], "dQ%d" % T)
            commit(dq_full)
            if more:
                if do_single and mutant != "do_single_no_bar":
                    yield from wait(do_full, (T + 1) & 1)
                issue([dbuf(T + 1)], "dP%d" % (T + 1))
                commit(dp_full)
            yield "work"

    def softmax():
        for T in range(n_tiles):
            s = T & 1
            yield from wait(s_full, T & 1)
            yield from wait(q_full[s], (T >> 1) & 1)
            read(("V", s), "softmax P")
            for _ in range(rng.randint(1, 4)):
                yield "work"
            unread(("V", s))
            p_ready.arrive()
            yield from wait(dp_full, T & 1)
            dp_read.arrive()
            read(("V", s), "softmax dS")
            for _ in range(rng.randint(1, 4)):
                yield "work"
            unread(("V", s))
            ds_ready.arrive()

    def dq_warps():
        for T in range(n_tiles):
            yield from wait(dq_full, T & 1)
            yield "work"
            dq_empty.arrive()

    workers = [producer(), mma(), softmax(), softmax(), dq_warps()]
    daemons = [tensor_pipe(), loader()]
    asleep, idle, tick = {}, 0, 0
    while workers:
        tick += 1
        progressed = False
        order = workers + daemons
        rng.shuffle(order)
        for g in order:
            if asleep.get(id(g), 0) > tick or rng.random() < 0.3:
                continue
            if g in workers and rng.random() < 0.003:
                asleep[id(g)] = tick + rng.randint(20, 200)
                continue
            try:
                progressed |= next(g) not in ("blocked", "idle")
            except StopIteration:
                workers.remove(g)
                progressed = True
        if problems:
            return problems[0]
        idle = 0 if progressed else idle + 1
        if idle > max_idle:
            return "deadlock"
    for _ in range(5000):
        if not pipe:
            break
        next(daemons[0])
    if problems:
        return problems[0]
    missing = [tag for T in range(n_tiles) for tag in ("dV%d" % T, "dK%d" % T) if tag not in ran]
    return "products never ran: %s" % missing[:4] if missing else None


@pytest.mark.parametrize("do_with_q", [True, False])
@pytest.mark.parametrize("n_tiles", [1, 2, 3, 6])
def test_q_and_do_stages_are_never_overwritten_while_read(n_tiles, do_with_q):
    for seed in range(150):
        r = simulate(n_tiles, seed, do_with_q=do_with_q)
        assert r is None, (n_tiles, do_with_q, seed, r)


@pytest.mark.parametrize("mutant,do_with_q", [("release_after_dv", True), ("release_after_dv", False),
                                              ("do_single_no_bar", True)])
def test_wrong_forms_are_caught(mutant, do_with_q):
    found = None
    for n_tiles in (3, 6):
        for seed in range(200):
            r = simulate(n_tiles, seed, do_with_q=do_with_q, mutant=mutant)
            if r is not None and r != "deadlock":
                found = r
                break
        if found:
            break
    assert found, mutant
