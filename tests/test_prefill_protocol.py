"""A CPU model of the tcgen05 prefill kernel's synchronisation protocol (no GPU).

The model runs every role of one CTA as a coroutine -- the producer warp, the two
MMA issuer threads and the eight softmax warps -- over the kernel's shared objects:
the unit queue, the Q buffers, the K/V ring, the per-tile S / P / P V barriers and
the per-tile S-read counters.  Asynchronous copies and MMAs complete at once (the
roles still order themselves only through the barriers, which is what matters for
deadlock).  A scheduler interleaves the roles in a random order every round; every
parity wait is checked against the barrier's true phase count, so a wait that would
take a later (or earlier) phase for the one it wants -- parity aliasing -- fails the
test, and so does a round in which no role can move (deadlock).  Each role takes one to
three steps per round, so the roles interleave at the granularity of single barrier
operations.

What it mirrors from the kernel: the unit list (units bucketed by the KV tiles of
tile A, longest first, dealt to CTAs in a snake); the producer publishing each unit
and then loading Q and the K/V tiles into a 5-slot ring (a slot freed by one commit
per tile that reads it, two by tile A for the tiles B does not read); the S columns
shared by the two tiles in the order A0 B0 A1 B1 ..., each S issued only once the S
before it has been read by all four warps of its tile (a monotonic counter); each
issuer taking S_t(j+1) and P_t(j) V_j in whichever order their inputs are ready; the
softmax reading S, waiting for the previous P V before writing P, and the epilogue
waiting for the last P V.
"""

from __future__ import annotations

import itertools
import random

KRING, USLOTS, READERS = 5, 4, 10       # ring slots, unit-queue slots, unit readers


class Bar:
    """An mbarrier: `count` arrivals complete a phase; waits are by phase parity."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"too many arrivals on {self.name}"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, k):
        """Parity test for phase index k, checked against the true phase count."""
        by_parity = (self.phase & 1) != (k & 1)
        assert by_parity == (self.phase > k), \
            f"parity aliasing on {self.name}: phase {k} wanted, barrier at {self.phase}"
        return by_parity


def cta_units(cached, new, group, cta, grid):
    """(KV tiles of tile A, of tile B, keys tile A reads) of CTA `cta`'s units."""
    qpt = 128 // group
    seqs = []
    for c, q in zip(cached, new):
        T = -(-q // qpt)
        seqs.append((q, c + q, T, (T + 1) // 2))
    lst = []
    for b in range(-(-max(k for _, k, _, _ in seqs) // 128), 0, -1):
        for q, k, T, P in seqs:
            c = k - q

            def first_pair(bb):
                if c + q <= bb * 128:
                    return 0
                R = bb * 128 - c
                if R < 0:
                    return P
                return min(max((T - R // qpt + 1) // 2, 1), P)

            for pp in range(first_pair(b), first_pair(b - 1)):
                ta, tb = T - 1 - 2 * pp, T - 2 - 2 * pp
                kv_end = c + min(q, (ta + 1) * qpt)
                nb = -(-(c + min(q, (tb + 1) * qpt)) // 128) if tb >= 0 else 0
                lst.append((-(-kv_end // 128), nb, kv_end))
    mine = []
    for kk in itertools.count():
        pos = (kk >> 1) * 2 * grid + ((2 * grid - 1 - cta) if kk & 1 else cta)
        if pos >= len(lst):
            return mine
        mine.append(lst[pos])


def run(units, rnd, mistake=None):
    """Runs one CTA's roles over `units`; returns None, or the roles stuck in a deadlock.

    Besides the parity checks, the shared S columns are tracked as data: writing an S
    asserts that all four warps of the S it replaces have read it, and each warp's read
    asserts that the columns hold its own S.  `mistake` plants one error for the tests
    that show the model can fail: "no_read_counter" issues an S without waiting for the
    previous S's readers, "single_release" has tile A free the ring slots of the K/V
    tiles tile B skips once instead of twice, "early_p" writes P without waiting for the
    previous P V."""
    bars, reads = {}, {0: 0, 1: 0}
    s_cols = {"owner": None, "reads": 4}

    def bar(name, count=1):
        return bars.setdefault(name, Bar(name, count))

    for t in (0, 1):
        for n in ("q_full", "q_empty", "s_full", "pv_done"):
            bar(f"{n}{t}")
        bar(f"p_full{t}", 4)
    for s in range(KRING):
        bar(f"kv_full{s}")
        bar(f"kv_empty{s}", 2)
    for s in range(USLOTS):
        bar(f"unit_full{s}")
        bar(f"unit_empty{s}", READERS)
    desc = [None] * USLOTS

    def wait(name, k):
        return ("wait", name, k)

    def arrive(name):
        return ("arrive", name)

    def producer():
        kv_i, qn = 0, [0, 0]
        for k in range(len(units) + 1):
            us = k % USLOTS
            if k >= USLOTS:
                yield wait(f"unit_empty{us}", k // USLOTS - 1)
            desc[us] = units[k] if k < len(units) else (0, 0, 0)
            yield arrive(f"unit_full{us}")
            if k == len(units):
                return
            n, nb, _ = units[k]
            for t, nt in ((0, n), (1, nb)):
                if nt:
                    if qn[t]:
                        yield wait(f"q_empty{t}", qn[t] - 1)
                    yield arrive(f"q_full{t}")
                    qn[t] += 1
            for _ in range(2 * n):
                slot = kv_i % KRING
                if kv_i >= KRING:
                    yield wait(f"kv_empty{slot}", kv_i // KRING - 1)
                yield arrive(f"kv_full{slot}")
                kv_i += 1

    def take(k):
        us = k % USLOTS
        yield wait(f"unit_full{us}", k // USLOTS)
        u = desc[us]
        yield arrive(f"unit_empty{us}")
        return u

    def issuer(t):
        kv_i = qc = pc = ra = rb = 0
        last = None                                 # the previous unit's last S: (tile, index)
        for k in itertools.count():
            n, nb, _ = yield from take(k)
            if n == 0:
                return
            nt = (n, nb)[t]
            if nt:
                def pred(j):
                    if t == 1:
                        return (0, ra + j)
                    if j == 0:
                        return last
                    return (1, rb + j - 1) if j - 1 < nb else (0, ra + j - 1)

                def s_ready(p):
                    if mistake == "no_read_counter":
                        return True
                    return p is None or reads[p[0]] >= 4 * (p[1] + 1)

                def release(slot, j):
                    yield arrive(f"kv_empty{slot}")
                    if t == 0 and j >= nb and mistake != "single_release":
                        yield arrive(f"kv_empty{slot}")

                yield wait(f"q_full{t}", qc)
                qc += 1
                yield wait(f"kv_full{kv_i % KRING}", kv_i // KRING)
                while not s_ready(pred(0)):
                    yield ("spin",)
                yield ("write_s", t, (ra, rb)[t])
                yield arrive(f"s_full{t}")
                if nt == 1:
                    yield arrive(f"q_empty{t}")
                yield from release(kv_i % KRING, 0)
                for j in range(nt):
                    iv = kv_i + 2 * j + 1
                    kn = iv + 1
                    s_todo, pv_todo = j + 1 < nt, True
                    p = pred(j + 1) if s_todo else None
                    while s_todo or pv_todo:
                        moved = False
                        for which in rnd.sample((0, 1), 2):
                            if which == 0 and s_todo and s_ready(p) and \
                                    bars[f"kv_full{kn % KRING}"].done(kn // KRING):
                                yield ("write_s", t, (ra, rb)[t] + j + 1)
                                yield arrive(f"s_full{t}")
                                if j + 2 == nt:
                                    yield arrive(f"q_empty{t}")
                                yield from release(kn % KRING, j + 1)
                                s_todo, moved = False, True
                            if which == 1 and pv_todo and \
                                    bars[f"kv_full{iv % KRING}"].done(iv // KRING) and \
                                    bars[f"p_full{t}"].done(pc):
                                pc += 1
                                yield arrive(f"pv_done{t}")
                                yield from release(iv % KRING, j)
                                pv_todo, moved = False, True
                        if not moved:
                            yield ("spin",)
            last = (1, rb + nb - 1) if nb == n else (0, ra + n - 1)
            ra, rb, kv_i = ra + n, rb + nb, kv_i + 2 * n

    def softmax(t):
        sc = pvc = kv_i = 0
        for k in itertools.count():
            n, nb, kv_end = yield from take(k)
            if n == 0:
                return
            kv_unit, kv_i = kv_i, kv_i + 2 * n
            nt = (n, nb)[t]
            for j in range(nt):
                yield wait(f"s_full{t}", sc)
                yield ("read", t, sc)
                sc += 1
                if j and mistake != "early_p":
                    yield wait(f"pv_done{t}", pvc)
                    pvc += 1
                if j == n - 1 and (kv_end - j * 128) & 15:   # zeroing the last V tile's tail
                    iv = kv_unit + 2 * j + 1
                    yield wait(f"kv_full{iv % KRING}", iv // KRING)
                yield arrive(f"p_full{t}")
            if nt:
                if mistake == "early_p":
                    pvc += nt - 1
                yield wait(f"pv_done{t}", pvc)
                pvc += 1

    roles = {"producer": producer(), "issuerA": issuer(0), "issuerB": issuer(1)}
    for t in (0, 1):
        for w in range(4):
            roles[f"softmax{'AB'[t]}{w}"] = softmax(t)
    pending = {r: None for r in roles}
    while roles:
        moved = False
        order = list(roles)
        rnd.shuffle(order)
        for r in order:
            g = roles[r]
            for _ in range(rnd.randint(1, 3)):     # a few steps of each role per round
                op = pending[r]
                if op is None:
                    try:
                        op = next(g)
                    except StopIteration:
                        del roles[r]
                        moved = True
                        break
                if op[0] == "wait":
                    if bars[op[1]].done(op[2]):
                        pending[r], moved = None, True
                        continue
                    pending[r] = op
                    break
                if op[0] == "spin":
                    pending[r] = None
                    break
                if op[0] == "write_s":
                    assert s_cols["reads"] == 4, \
                        f"S {op[1:]} written over S {s_cols['owner']} before all its readers"
                    s_cols["owner"], s_cols["reads"] = op[1:], 0
                elif op[0] == "read":
                    assert s_cols["owner"] == op[1:], \
                        f"tile {op[1]} reads S {op[2]}, the columns hold {s_cols['owner']}"
                    s_cols["reads"] += 1
                    reads[op[1]] += 1
                else:
                    bars[op[1]].arrive()
                pending[r], moved = None, True
        if not moved:
            return {r: pending[r] for r in roles}
    return None


def test_ragged_batch_all_grids_random_schedules():
    cached = [0, 0, 0, 17, 256, 300, 0, 5, 1024]
    new = [1, 63, 129, 47, 1, 200, 256, 64, 65]
    for seed in range(10):
        rnd = random.Random(seed)
        for group in (1, 3, 7):
            for grid in (1, 3, 148):
                for cta in range(min(grid, 3)):
                    assert run(cta_units(cached, new, group, cta, grid), rnd) is None


def test_random_unit_lists():
    rnd = random.Random(11)
    for _ in range(400):
        units = []
        for _ in range(rnd.randint(1, 10)):
            na = rnd.randint(1, 17)
            nb = rnd.choice([0, na, max(0, na - 1), rnd.randint(0, na)])
            units.append((na, nb, (na - 1) * 128 + rnd.randint(1, 128)))
        assert run(units, rnd) is None, units


def _fails(units, mistake, seeds=20):
    """True when some schedule of `units` with `mistake` planted trips a check."""
    for seed in range(seeds):
        try:
            if run(units, random.Random(seed), mistake) is not None:
                return True
        except AssertionError:
            return True
    return False


def test_the_model_catches_planted_mistakes():
    units = [(3, 2, 300), (2, 2, 200), (4, 1, 450), (1, 0, 5)]
    for mistake in ("no_read_counter", "single_release", "early_p"):
        assert _fails(units, mistake), mistake
    assert not _fails(units, None)
