"""Model check of the forward's tensor-memory protocol per Q tile (CPU).

Each of the forward's two Q tiles owns two TMEM regions: the S columns, where
P overwrites S once formed, and the O accumulator.  Per item, per key tile j,
the MMA warp issues:
- P V(j), which reads P and accumulates into O, after the softmax has
  published P(j) (p_full);
- then S(j + 1), which overwrites the S columns, with a commit to s_full.
After the tile's last P V it commits o_full.  The first P V of an item
overwrites O (no accumulate), so it waits for o_free: the previous item's
epilogue has read O.

The softmax warps of the tile wait for s_full, then:
- read S;
- when the running max moves, rescale O in TMEM (the P V before this S is
  complete, since S's commit covers every earlier MMA);
- write P over S and arrive on p_full.
After the item's last key tile they wait for o_full, read O for the
epilogue and arrive on o_free.  The next item's first S is issued as soon as
its Q and K are in, while the softmax may still be in the epilogue.

This model runs both tiles' MMAs on one in-order tensor pipe and both tiles'
softmax, with random rescales, under a seeded random scheduler with long
stalls.  No agent writes a region while another's access to it is in flight.
Mutants must be caught:
- o_full committed before the last P V;
- P V issued without waiting for p_full.
The o_free wait turns out to be implied: the same softmax warps read O in
their epilogue before they form the next item's first P, and the first P V
waits for all of them on p_full.  Dropping it must therefore cause no
conflict; it costs the MMA warp one satisfied wait per item and tile.
"""
import random

import pytest


class Bar:
    def __init__(self):
        self.phase = 0

    def arrive(self):
        self.phase += 1

    def done(self, parity):
        return parity != (self.phase & 1)


def simulate(items, seed, mutant=None, max_idle=800):
    rng = random.Random(seed)
    s_full, p_full, o_full, o_free = ([Bar(), Bar()] for _ in range(4))
    inflight = {(r, t): [] for r in ("S", "O") for t in range(2)}
    pipe, ran, problems = [], set(), []

    def touch(agent, reg, kind):
        for a, k in inflight[reg]:
            if a != agent and (kind == "w" or k == "w") and not problems:
                problems.append("%s %ss %s while %s has a %s in flight" % (agent, "write" if kind == "w" else "read", reg, a, k))
        inflight[reg].append((agent, kind))

    def release(agent, reg, kind):
        inflight[reg].remove((agent, kind))

    def wait(bar, parity):
        while not bar.done(parity):
            yield "blocked"

    def issue(acc, tag):
        for reg, kind in acc:
            touch("mma", reg, kind)
        pipe.append(("mma", acc, tag))

    def tensor_pipe():
        while True:
            if not pipe:
                yield "idle"
                continue
            op = pipe[0]
            if op[0] == "mma":
                for _ in range(rng.randint(1, 6)):
                    yield "work"
                for reg, kind in op[1]:
                    release("mma", reg, kind)
                ran.add(op[2])
            else:
                op[1].arrive()
            pipe.pop(0)
            yield "work"

    def mma():
        pc = [0, 0]      # key tiles done per Q tile (p_full phases)
        nact = [0, 0]    # items in which the tile took part (o_full / o_free phases)
        for n, nk in enumerate(items):
            for t in range(2):
                if nk[t] > 0:
                    issue([(("S", t), "w")], "S%d_%d(0)" % (n, t))
                    pipe.append(("commit", s_full[t]))
            for j in range(max(nk)):
                for t in range(2):
                    if j >= nk[t]:
                        continue
                    if mutant != "no_p_wait":
                        yield from wait(p_full[t], pc[t] & 1)
                    if j == 0 and nact[t] > 0 and mutant != "no_o_free":
                        yield from wait(o_free[t], (nact[t] - 1) & 1)
                    last = j == nk[t] - 1
                    if last and mutant == "early_o_full":
                        pipe.append(("commit", o_full[t]))
                    issue([(("S", t), "r"), (("O", t), "w")], "PV%d_%d(%d)" % (n, t, j))
                    pc[t] += 1
                    if last and mutant != "early_o_full":
                        pipe.append(("commit", o_full[t]))
                    if j + 1 < nk[t]:
                        issue([(("S", t), "w")], "S%d_%d(%d)" % (n, t, j + 1))
                        pipe.append(("commit", s_full[t]))
                yield "work"
            for t in range(2):
                nact[t] += 1 if nk[t] > 0 else 0

    def softmax(t):
        agent = "soft%d" % t
        pc = oc = 0
        for n, nk in enumerate(items):
            for j in range(nk[t]):
                yield from wait(s_full[t], pc & 1)
                touch(agent, ("S", t), "r")
                yield "read"
                release(agent, ("S", t), "r")
                if j > 0 and rng.random() < 0.3:  # the running max moved: rescale O in TMEM
                    touch(agent, ("O", t), "w")
                    yield "write"
                    release(agent, ("O", t), "w")
                touch(agent, ("S", t), "w")  # P over S
                yield "write"
                release(agent, ("S", t), "w")
                p_full[t].arrive()
                pc += 1
            if nk[t] > 0:
                yield from wait(o_full[t], oc & 1)
                oc += 1
                touch(agent, ("O", t), "r")
                for _ in range(rng.randint(1, 5)):
                    yield "read"
                release(agent, ("O", t), "r")
                o_free[t].arrive()

    workers = [mma(), softmax(0), softmax(1)]
    daemons = [tensor_pipe()]
    asleep, idle, tick = {}, 0, 0
    while workers:
        tick += 1
        progressed = False
        order = workers + daemons
        rng.shuffle(order)
        for g in order:
            if asleep.get(id(g), 0) > tick or rng.random() < 0.3:
                continue
            if g in workers and rng.random() < 0.004:
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
    want = sum(sum(nk) for nk in items) * 2
    return None if len(ran) == want else "only %d of %d products ran" % (len(ran), want)


ITEMS = [[(1, 2), (3, 4), (5, 6)], [(4, 4), (4, 4)], [(2, 0), (3, 4), (1, 0), (2, 2)], [(1, 1)] * 5]


@pytest.mark.parametrize("items", ITEMS)
def test_tmem_regions_are_never_accessed_in_conflict(items):
    for seed in range(150):
        r = simulate(items, seed)
        assert r is None, (items, seed, r)


@pytest.mark.parametrize("mutant", ["early_o_full", "no_p_wait"])
def test_wrong_forms_are_caught(mutant):
    found = None
    for items in ITEMS:
        for seed in range(150):
            r = simulate(items, seed, mutant=mutant)
            if r is not None and r != "deadlock":
                found = r
                break
        if found:
            break
    assert found, mutant


def test_o_free_is_implied_by_p_full():
    for items in ITEMS:
        for seed in range(100):
            assert simulate(items, seed, mutant="no_o_free") is None, (items, seed)
