"""Model check of the d = 128 persistent backward's buffer protocol (CPU).

A persistent backward CTA walks several (head, key tile) items.  At d = 128
one set of buffers serves consecutive items:
- a K, V buffer that holds an item's keys and then its dV staging;
- the dS^T buffer and the dQ staging tile, which hold the dS^T of each query
  tile and the first and second halves of its dQ, and then the item's dK
  staging;
- the TMEM regions of dV and dK.

This file models the agents that touch those buffers, with the barriers the
kernel uses:
- the TMA producer (the next item's K, V loads);
- the MMA warp (the S^T, dP^T, dV, dK and dQ products of every tile, issued in
  order to the tensor pipe, with commits);
- two softmax warps (dS^T, then the item's epilogue: dV and dK staged and
  stored by TMA);
- the dQ warps' issuing thread (dQ staged in two halves and reduce-added by
  TMA);
- the tensor pipe and the TMA engine, as asynchronous agents.

A seeded random scheduler interleaves them, with long stalls.  In every state
it checks that no agent writes a buffer while an access by another agent is
still in flight:
- an MMA that reads it, issued and not yet complete;
- a TMA store or reduce-add that has not finished reading it;
- a TMA load still writing it;
- an epilogue still reading dV or dK out of TMEM.

It also checks that nothing deadlocks and that every item's products run.
Per-tile Q and dO traffic and the TMEM regions of S^T and dP^T are left out;
the tile pipeline's own barriers (s_full, p_ready, dp_full, dp_read,
ds_ready, dq_full, dq_empty, ds_free) are kept, since they order the buffer
accesses.  Mutants that drop one protocol step must each be caught.
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


def simulate(item_tiles, seed, drop=None, max_idle=800):
    rng = random.Random(seed)
    K = len(item_tiles)
    tiles = [(k, t) for k in range(K) for t in range(item_tiles[k])]  # global order, T = index
    NT = len(tiles)
    SMW = 2
    B = {n: Bar() for n in ("kv_full", "kv_empty", "s_full", "dp_full", "dq_full", "dq_empty_m", "dkdv_done",
                            "dq_stg_free", "epi_free", "ds_free", "epi_kv", "dv_free", "dk_free")}
    B["p_ready"] = Bar(SMW)
    B["dp_read"] = Bar(SMW)
    B["ds_ready"] = Bar(SMW)
    B["dv_staged"] = Bar(SMW)
    B["dk_staged"] = Bar(SMW)
    B["dv_free"] = Bar(SMW)
    B["dk_free"] = Bar(SMW)
    # buffer accesses in flight: buffer -> list of (agent, kind) ; kind "r" or "w"
    inflight = {b: [] for b in ("KV", "DS", "STG", "DV", "DK")}
    problems = []
    pipe = []            # queued tensor-pipe ops: ("mma", reads, writes, tag) or ("commit", bar)
    tma = []             # TMA ops in flight: dicts
    groups = {"soft": [], "dq": []}  # per issuing thread: list of committed groups (lists of ops)
    ran = set()

    def touch(agent, buf, kind):
        for a, k in inflight[buf]:
            if a != agent and (kind == "w" or k == "w"):
                if not problems:
                    problems.append("%s %ss %s while %s has a %s in flight" % (agent, "write" if kind == "w" else "read", buf, a, k))
        inflight[buf].append((agent, kind))

    def release(agent, buf, kind):
        inflight[buf].remove((agent, kind))

    def wait(bar, parity):
        while not B[bar].done(parity):
            yield "blocked"

    def issue(reads, writes, tag):
        # an MMA counts as in flight on its buffers from issue to completion; the
        # pipe runs them in order, so MMAs never conflict with each other
        for b in reads:
            touch("mma", b, "r")
        for b in writes:
            touch("mma", b, "w")
        pipe.append(("mma", reads, writes, tag))

    def commit(bar):
        pipe.append(("commit", bar))

    def tensor_pipe():
        while True:
            if not pipe:
                yield "idle"
                continue
            op = pipe[0]
            if op[0] == "mma":
                for _ in range(rng.randint(1, 6)):
                    yield "work"
                _, reads, writes, tag = op
                for b in reads:
                    release("mma", b, "r")
                for b in writes:
                    release("mma", b, "w")
                ran.add(tag)
            else:
                B[op[1]].arrive()
            pipe.pop(0)
            yield "work"

    def tma_engine():
        while True:
            if not tma:
                yield "idle"
                continue
            op = rng.choice(tma)
            op["left"] -= 1
            if op["left"] <= 0:
                tma.remove(op)
                release(op["agent"], op["buf"], op["kind"])
                op["done"] = True
                if op.get("bar"):
                    B[op["bar"]].arrive()
            yield "work"

    def tma_op(agent, buf, kind, bar=None, group=None):
        touch(agent, buf, kind)
        op = {"agent": agent, "buf": buf, "kind": kind, "left": rng.randint(1, 40), "bar": bar, "done": False}
        tma.append(op)
        return op

    def wait_groups(owner, keep):
        # cp.async.bulk.wait_group.read keep: all but the newest `keep` groups have read
        while any(not op["done"] for g in groups[owner][: max(0, len(groups[owner]) - keep)] for op in g):
            yield "blocked"

    def producer():
        for k in range(K):
            if k > 0 and drop != "kv_empty":
                yield from wait("kv_empty", (k & 1) ^ 1)
            tma_op("load", "KV", "w", bar="kv_full")
            yield "work"

    def mma():
        yield from wait("kv_full", 0)
        issue(["KV"], [], "S0")
        commit("s_full")
        issue(["KV"], [], "dP0")
        commit("dp_full")
        for T, (k, t) in enumerate(tiles):
            last = t + 1 == item_tiles[k]
            more = T + 1 < NT
            yield from wait("p_ready", T & 1)
            if t == 0 and k > 0 and drop != "dv_free":
                yield from wait("dv_free", (k - 1) & 1)
            issue([], ["DV"], "dV%d" % T)
            yield from wait("dp_read", T & 1)
            if more and not last:
                issue(["KV"], [], "S%d" % (T + 1))
                commit("s_full")
            yield from wait("ds_ready", T & 1)
            if t == 0 and k > 0 and drop != "dk_free":
                yield from wait("dk_free", (k - 1) & 1)
            issue(["DS"], ["DK"], "dK%d" % T)
            issue(["DS", "KV"], [], "dQ%d" % T)
            commit("dq_full")
            if last:
                commit("dkdv_done")
            if more and last:
                yield from wait("kv_full", (k + 1) & 1)
                issue(["KV"], [], "S%d" % (T + 1))
                commit("s_full")
            if more:
                yield from wait("dq_empty_m", T & 1)
                issue(["KV"], [], "dP%d" % (T + 1))
                commit("dp_full")
            yield "work"

    def softmax(w):
        # the softmax warps write disjoint halves (query halves of dS^T, column
        # halves of the dV and dK staging): one agent against all others
        agent = "soft"
        for T, (k, t) in enumerate(tiles):
            last = t + 1 == item_tiles[k]
            yield from wait("s_full", T & 1)
            for _ in range(rng.randint(0, 5)):
                yield "work"
            B["p_ready"].arrive()
            yield from wait("dp_full", T & 1)
            B["dp_read"].arrive()
            if T > 0 and drop != "ds_free":
                yield from wait("ds_free", (T - 1) & 1)
            touch(agent, "DS", "w")
            for _ in range(rng.randint(1, 4)):
                yield "write"
            release(agent, "DS", "w")
            B["ds_ready"].arrive()
            if not last:
                continue
            # epilogue of item k
            yield from wait("dkdv_done", k & 1)
            for which in (0, 1):
                if which == 1 and drop != "dq_stg_free":
                    yield from wait("dq_stg_free", k & 1)
                acc = "DV" if which == 0 else "DK"
                areas = ["KV"] if which == 0 else ["DS", "STG"]
                touch(agent, acc, "r")
                for a in areas:
                    touch(agent, a, "w")
                for _ in range(rng.randint(1, 4)):
                    yield "write"
                release(agent, acc, "r")
                for a in areas:
                    release(agent, a, "w")
                B["dv_free" if which == 0 else "dk_free"].arrive()
                B["dv_staged" if which == 0 else "dk_staged"].arrive()
                if w == 0:  # the issuing thread
                    yield from wait("dv_staged" if which == 0 else "dk_staged", k & 1)
                    ops = [tma_op("store", a, "r") for a in areas]
                    groups["soft"].append(ops)
                    yield from wait_groups("soft", 0)
                    B["kv_empty" if which == 0 else "epi_free"].arrive()
            if drop != "epi_free":
                yield from wait("epi_free", k & 1)

    def dq_warp():
        agent = "dq"
        for T, (k, t) in enumerate(tiles):
            last = t + 1 == item_tiles[k]
            yield from wait("dq_full", T & 1)
            # first half staged in the dS^T buffer (free: this tile's dK, dQ are complete)
            touch(agent, "DS", "w")
            yield "write"
            release(agent, "DS", "w")
            B["dq_empty_m"].arrive()   # dQ read out of TMEM
            g1 = [tma_op("reduce", "DS", "r")]
            groups["dq"].append(g1)
            # second half: the previous reduce-add from the staging tile has read it
            if drop != "stg_wait":
                yield from wait_groups("dq", 1)
            touch(agent, "STG", "w")
            yield "write"
            release(agent, "STG", "w")
            groups["dq"].append([tma_op("reduce", "STG", "r")])
            yield from wait_groups("dq", 1)
            B["ds_free"].arrive()
            if last:
                yield from wait_groups("dq", 0)
                B["dq_stg_free"].arrive()

    workers = [producer(), mma(), softmax(0), softmax(1), dq_warp()]
    daemons = [tensor_pipe(), tma_engine()]
    asleep, idle, tick = {}, 0, 0
    while workers:
        tick += 1
        progressed = False
        order = workers + daemons
        rng.shuffle(order)
        for g in order:
            if asleep.get(id(g), 0) > tick:
                continue
            if rng.random() < 0.3:
                continue
            if g in workers and rng.random() < 0.003:
                asleep[id(g)] = tick + rng.randint(20, 200)
                continue
            try:
                r = next(g)
                progressed |= r not in ("blocked", "idle")
            except StopIteration:
                workers.remove(g)
                progressed = True
        if problems:
            return problems[0]
        idle = 0 if progressed else idle + 1
        if idle > max_idle:
            return "deadlock"
    # drain the pipe and the TMA engine
    for _ in range(5000):
        if not pipe and not tma:
            break
        for g in daemons:
            next(g)
    if problems:
        return problems[0]
    missing = [tag for T in range(NT) for tag in ("dV%d" % T, "dK%d" % T, "dQ%d" % T) if tag not in ran]
    if missing:
        return "products never ran: %s" % missing[:4]
    return None


ITEM_MIXES = [[1, 1, 1], [2, 1, 3], [3, 2], [1, 3, 1, 2], [2, 2, 2]]


@pytest.mark.parametrize("items", ITEM_MIXES)
def test_buffer_protocol_holds_under_random_interleavings(items):
    for seed in range(120):
        r = simulate(items, seed)
        assert r is None, (items, seed, r)


@pytest.mark.parametrize("drop", ["kv_empty", "dq_stg_free", "epi_free", "ds_free", "stg_wait"])
def test_each_protocol_step_is_needed(drop):
    """Leaving out any one of these waits lets some interleaving write a buffer
    that is still being read, or read one that is still being written."""
    found = None
    for items in ITEM_MIXES:
        for seed in range(120):
            r = simulate(items, seed, drop=drop)
            if r is not None and r != "deadlock":
                found = r
                break
        if found:
            break
    assert found, drop


@pytest.mark.parametrize("drop", ["dv_free", "dk_free"])
def test_dv_dk_free_are_implied_at_d128(drop):
    """The MMA warp's waits for dV and dK to have been read out of TMEM before
    an item's first dV and dK products are implied at d = 128: the softmax warps
    read them out in their epilogue before they form the next item's first P,
    which those products wait for.  (At d = 64 the dQ warps write the epilogue
    while the softmax warps run the next item, and the waits are needed.)"""
    for items in ITEM_MIXES:
        for seed in range(60):
            assert simulate(items, seed, drop=drop) is None, (items, seed)


# ---------------------------------------------------------------------------
# d = 64: two K, V buffers (item k in buffer k % 2, released by an MMA commit
# after the item's last product), dQ in its own TMEM region, the whole dQ
# staged in the staging tile, and the dQ warps writing an item's dV (into the
# dV staging area) and dK (into the staging tile) while the other warps run
# the next item.

def simulate64(item_tiles, seed, drop=None, max_idle=800):
    rng = random.Random(seed)
    K = len(item_tiles)
    tiles = [(k, t) for k in range(K) for t in range(item_tiles[k])]
    NT = len(tiles)
    SMW = 2
    B = {n: Bar() for n in ("kv_full0", "kv_full1", "kv_empty0", "kv_empty1", "s_full", "dp_full", "dq_full",
                            "dq_empty", "dkdv_done", "dv_free", "dk_free")}
    for n in ("p_ready", "dp_read", "ds_ready"):
        B[n] = Bar(SMW)
    inflight = {b: [] for b in ("KV0", "KV1", "DS", "STG", "EPI", "DV", "DK", "DQ")}
    problems, pipe, tma, groups, ran = [], [], [], [], set()

    def touch(agent, buf, kind):
        for a, k in inflight[buf]:
            if a != agent and (kind == "w" or k == "w") and not problems:
                problems.append("%s %ss %s while %s has a %s in flight" % (agent, "write" if kind == "w" else "read", buf, a, k))
        inflight[buf].append((agent, kind))

    def release(agent, buf, kind):
        inflight[buf].remove((agent, kind))

    def wait(bar, parity):
        while not B[bar].done(parity):
            yield "blocked"

    def issue(reads, writes, tag):
        for b in reads:
            touch("mma", b, "r")
        for b in writes:
            touch("mma", b, "w")
        pipe.append(("mma", reads, writes, tag))

    def commit(bar):
        pipe.append(("commit", bar))

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
                    release("mma", b, "r")
                for b in op[2]:
                    release("mma", b, "w")
                ran.add(op[3])
            else:
                B[op[1]].arrive()
            pipe.pop(0)
            yield "work"

    def tma_engine():
        while True:
            if not tma:
                yield "idle"
                continue
            op = rng.choice(tma)
            op["left"] -= 1
            if op["left"] <= 0:
                tma.remove(op)
                release(op["agent"], op["buf"], op["kind"])
                op["done"] = True
                if op.get("bar"):
                    B[op["bar"]].arrive()
            yield "work"

    def tma_op(agent, buf, kind, bar=None):
        touch(agent, buf, kind)
        op = {"agent": agent, "buf": buf, "kind": kind, "left": rng.randint(1, 40), "bar": bar, "done": False}
        tma.append(op)
        return op

    def wait_groups(keep):
        while any(not op["done"] for g in groups[: max(0, len(groups) - keep)] for op in g):
            yield "blocked"

    def kv(k):
        return "KV%d" % (k & 1)

    def producer():
        for k in range(K):
            b = k & 1
            if drop != "kv_empty":
                yield from wait("kv_empty%d" % b, ((k >> 1) & 1) ^ 1)
            tma_op("load", kv(k), "w", bar="kv_full%d" % b)
            yield "work"

    def mma():
        yield from wait("kv_full0", 0)
        issue([kv(0)], [], "S0")
        commit("s_full")
        issue([kv(0)], [], "dP0")
        commit("dp_full")
        for T, (k, t) in enumerate(tiles):
            cross = t + 1 == item_tiles[k]
            more = T + 1 < NT
            nk = k + 1 if cross else k
            yield from wait("p_ready", T & 1)
            if t == 0 and k > 0 and drop != "dv_free":
                yield from wait("dv_free", (k - 1) & 1)
            issue([], ["DV"], "dV%d" % T)
            yield from wait("dp_read", T & 1)
            if more:
                if cross:
                    yield from wait("kv_full%d" % (nk & 1), (nk >> 1) & 1)
                issue([kv(nk)], [], "S%d" % (T + 1))
                commit("s_full")
            yield from wait("ds_ready", T & 1)
            if t == 0 and k > 0 and drop != "dk_free":
                yield from wait("dk_free", (k - 1) & 1)
            issue(["DS"], ["DK"], "dK%d" % T)
            if T > 0:
                yield from wait("dq_empty", (T - 1) & 1)
            issue(["DS", kv(k)], ["DQ"], "dQ%d" % T)
            commit("dq_full")
            if cross:
                commit("dkdv_done")
                commit("kv_empty%d" % (k & 1))
            if more:
                issue([kv(nk)], [], "dP%d" % (T + 1))
                commit("dp_full")
            yield "work"

    def softmax(w):
        for T, (k, t) in enumerate(tiles):
            yield from wait("s_full", T & 1)
            for _ in range(rng.randint(0, 5)):
                yield "work"
            B["p_ready"].arrive()
            yield from wait("dp_full", T & 1)
            B["dp_read"].arrive()
            touch("soft", "DS", "w")
            for _ in range(rng.randint(1, 4)):
                yield "write"
            release("soft", "DS", "w")
            B["ds_ready"].arrive()

    def dq_warps():
        agent = "dq"
        for T, (k, t) in enumerate(tiles):
            last = t + 1 == item_tiles[k]
            yield from wait("dq_full", T & 1)
            touch(agent, "DQ", "r")
            yield "read"
            release(agent, "DQ", "r")
            B["dq_empty"].arrive()
            if drop != "stg_wait":
                yield from wait_groups(0)  # the previous reduce-add (or epilogue store) has read its staging
            touch(agent, "STG", "w")
            yield "write"
            release(agent, "STG", "w")
            groups.append([tma_op("reduce", "STG", "r")])
            if not last:
                continue
            # epilogue of item k, while the other warps run the next item
            if drop != "epi_wait":
                yield from wait_groups(0)
            yield from wait("dkdv_done", k & 1)
            for acc, area, bar in (("DV", "EPI", "dv_free"), ("DK", "STG", "dk_free")):
                touch(agent, acc, "r")
                touch(agent, area, "w")
                yield "write"
                release(agent, acc, "r")
                release(agent, area, "w")
                B[bar].arrive()
            groups.append([tma_op("store", "EPI", "r"), tma_op("store", "STG", "r")])

    workers = [producer(), mma(), softmax(0), softmax(1), dq_warps()]
    daemons = [tensor_pipe(), tma_engine()]
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
        if not pipe and not tma:
            break
        for g in daemons:
            next(g)
    if problems:
        return problems[0]
    missing = [tag for T in range(NT) for tag in ("dV%d" % T, "dK%d" % T, "dQ%d" % T) if tag not in ran]
    return "products never ran: %s" % missing[:4] if missing else None


@pytest.mark.parametrize("items", ITEM_MIXES)
def test_d64_buffer_protocol_holds_under_random_interleavings(items):
    for seed in range(120):
        r = simulate64(items, seed)
        assert r is None, (items, seed, r)


@pytest.mark.parametrize("drop", ["kv_empty", "dv_free", "dk_free", "stg_wait", "epi_wait"])
def test_d64_each_protocol_step_is_needed(drop):
    found = None
    for items in ITEM_MIXES:
        for seed in range(150):
            r = simulate64(items, seed, drop=drop)
            if r is not None and r != "deadlock":
                found = r
                break
        if found:
            break
    assert found, drop
