"""Model check of the forward's K/V ring (CPU).

The persistent forward's producer streams each item's K_j and V_j tiles
through a ring of shared-memory stages: K_0, V_0, K_1, V_1, and so on.  The
MMA warp issues, for an item:
- S_t(0) for each Q tile t that has key tiles;
- then, for each key step j: P V_t(j) (reads V_j) and S_t(j + 1) (reads
  K_{j+1}), tile 0 before tile 1.
The tensor pipe completes MMAs in issue order.

No MMA commits the ring stages' release.  One softmax thread of the Q tile
with the most key tiles (tile 1 unless it lies past N) releases them: when its
S(j) is complete, K_j and V_{j-1} are consumed (V_{j-1} at j = 0 is the
previous item's last V).  Causal items give tile 0 fewer key tiles than
tile 1.

This model runs the producer, the MMA warp, both tiles' softmax and the
in-order tensor pipe under a seeded random scheduler with long stalls.  It
checks that:
- no load overwrites a stage that an issued MMA has not finished reading;
- nothing deadlocks;
- every product runs.
Mutants of the release rule must be caught: releasing on tile 0's S(j), or
always releasing from tile 0.
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


def simulate(items, stages, seed, release="last_tile", max_idle=800):
    """items: list of (n_kv0, n_kv1) with n_kv0 >= 1 and n_kv0 <= n_kv1 or
    n_kv1 == 0 (tile 1 past N)."""
    rng = random.Random(seed)
    kv_full = [Bar() for _ in range(stages)]
    kv_empty = [Bar() for _ in range(stages)]
    s_full = [Bar(), Bar()]
    p_full = [Bar(), Bar()]
    readers = [0] * stages      # issued MMAs that read the stage and have not completed
    writing = [False] * stages  # a load is writing the stage
    pipe, loads, ran, problems = [], [], set(), []

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
                readers[op[1]] -= 1
                ran.add(op[2])
            else:
                op[1].arrive()
            pipe.pop(0)
            yield "work"

    def issue(stage, tag):
        if writing[stage] and not problems:
            problems.append("%s reads stage %d while a load writes it" % (tag, stage))
        readers[stage] += 1
        pipe.append(("mma", stage, tag))

    def loader():
        while True:
            if not loads:
                yield "idle"
                continue
            s = rng.choice(loads)
            if rng.random() < 0.2:
                loads.remove(s)
                writing[s] = False
                kv_full[s].arrive()
            yield "work"

    def producer():
        it = 0
        for n, (a, b) in enumerate(items):
            for j in range(max(a, b)):
                for _kind in range(2):
                    s = it % stages
                    yield from wait(kv_empty[s], ((it // stages) & 1) ^ 1)
                    if readers[s] and not problems:
                        problems.append("load overwrites stage %d while %d MMAs read it" % (s, readers[s]))
                    writing[s] = True
                    loads.append(s)
                    it += 1
                    yield "work"

    def mma():
        it = 0
        pc = [0, 0]
        for n, nk in enumerate(items):
            nmax = max(nk)
            sK = it % stages
            yield from wait(kv_full[sK], (it // stages) & 1)
            it += 1
            for t in range(2):
                if nk[t] > 0:
                    issue(sK, "S%d_%d(0)" % (n, t))
                    pipe.append(("commit", s_full[t]))
            for j in range(nmax):
                sV = it % stages
                yield from wait(kv_full[sV], (it // stages) & 1)
                it += 1
                sKn = None
                if j + 1 < nmax:
                    sKn = it % stages
                    yield from wait(kv_full[sKn], (it // stages) & 1)
                    it += 1
                for t in range(2):
                    if j >= nk[t]:
                        continue
                    yield from wait(p_full[t], pc[t] & 1)
                    issue(sV, "PV%d_%d(%d)" % (n, t, j))
                    pc[t] += 1
                    if j + 1 < nk[t]:
                        issue(sKn, "S%d_%d(%d)" % (n, t, j + 1))
                        pipe.append(("commit", s_full[t]))
            yield "work"

    def softmax(t):
        pc = 0
        ring0 = 0
        for n, nk in enumerate(items):
            if release == "last_tile":
                releaser = 1 if nk[1] > 0 else 0
            elif release == "tile0":
                releaser = 0
            else:  # "first_tile": on tile 0's S whenever tile 0 has that key tile
                releaser = None
            for j in range(nk[t]):
                yield from wait(s_full[t], pc & 1)
                if releaser is None:
                    me = t == (0 if j < nk[0] else 1)
                else:
                    me = t == releaser
                if me:
                    k_slot = ring0 + 2 * j
                    kv_empty[k_slot % stages].arrive()
                    if k_slot > 0:
                        kv_empty[(k_slot - 1) % stages].arrive()
                for _ in range(rng.randint(0, 4)):
                    yield "work"
                p_full[t].arrive()
                pc += 1
            ring0 += 2 * max(nk)

    workers = [producer(), mma(), softmax(0), softmax(1)]
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
    want = sum(sum(nk) for nk in items) * 2
    return None if len(ran) == want else "only %d of %d products ran" % (len(ran), want)


ITEMS = [
    [(1, 2), (3, 4), (5, 6)],          # causal pairs: tile 0 one key tile short
    [(4, 4), (4, 4), (4, 4)],          # non-causal
    [(2, 0), (3, 4), (1, 0)],          # items whose tile 1 lies past N
    [(1, 1), (2, 2), (1, 2), (3, 3)],
]


@pytest.mark.parametrize("stages", [4, 8])
@pytest.mark.parametrize("items", ITEMS)
def test_ring_release_by_the_last_tile_is_safe(items, stages):
    for seed in range(100):
        r = simulate(items, stages, seed)
        assert r is None, (items, stages, seed, r)


@pytest.mark.parametrize("release", ["first_tile", "tile0"])
def test_wrong_release_rules_are_caught(release):
    found = None
    for items in ITEMS:
        for seed in range(100):
            r = simulate(items, 4, seed, release=release)
            if r is not None and r != "deadlock":
                found = r
                break
        if found:
            break
    assert found, release
