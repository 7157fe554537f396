"""The prefill kernel's work list, checked on the CPU against brute force (no GPU).

The tcgen05 prefill kernel splits every (sequence, KV head) into units of two
consecutive query tiles (tile A the later one, B the one before), lists the units
from the most KV tiles tile A reads to the fewest, and deals the list to the
persistent CTAs in a snake.  It never builds the list: a warp walks it, finding the
pairs of a sequence whose tile A reads exactly b KV tiles from a closed form in
the sequence's lengths.  This file restates that closed form (the same arithmetic as
the kernel's first-pair helper) and checks it against a plain enumeration of every
pair: every pair lands in exactly one bucket, the bucket is the pair's KV-tile
count, and the snake deal hands every list position to exactly one CTA.  The GPU
parity tests check the outputs the walk produces; this pins the formula itself on
cases too many for them (groups of 1 to 128 heads, one-query sequences, cached
prefixes that are and are not tile aligned).
"""

from __future__ import annotations

import random

KEYS = 128           # keys per KV tile
ROWS = 128           # packed (query, head) rows per query tile


def tiles(q_len: int, qpt: int) -> tuple[int, int]:
    """Query tiles T of a sequence and its pairs P (the last pair may lack tile B)."""
    T = -(-q_len // qpt)
    return T, (T + 1) // 2


def kv_tiles_of_pair(cached: int, q_len: int, qpt: int, pp: int) -> tuple[int, int]:
    """KV tiles read by tile A and tile B of pair pp (0 = the sequence's last two tiles)."""
    T, _ = tiles(q_len, qpt)
    ta, tb = T - 1 - 2 * pp, T - 2 - 2 * pp
    na = -(-(cached + min(q_len, (ta + 1) * qpt)) // KEYS)
    nb = -(-(cached + min(q_len, (tb + 1) * qpt)) // KEYS) if tb >= 0 else 0
    return na, nb


def first_pair(cached: int, q_len: int, qpt: int, b: int) -> int:
    """First pair whose tile A reads at most b KV tiles (P when none does): pair pp's
    tile A ends at query min(q_len, (T - 2 pp) qpt), so its KV tiles fall as pp grows."""
    T, P = tiles(q_len, qpt)
    if cached + q_len <= b * KEYS:
        return 0
    R = b * KEYS - cached
    if R < 0:
        return P
    return min(max((T - R // qpt + 1) // 2, 1), P)


def unit_list(cached: list[int], new: list[int], qpt: int, hkv: int):
    """The kernel's list: buckets from the most KV tiles down, then sequence, pair, KV head."""
    top = max(-(-(c + q) // KEYS) for c, q in zip(cached, new))
    out = []
    for b in range(top, 0, -1):
        for s, (c, q) in enumerate(zip(cached, new)):
            for pp in range(first_pair(c, q, qpt, b), first_pair(c, q, qpt, b - 1)):
                for h in range(hkv):
                    out.append((b, s, pp, h))
    return out


def snake_owner(pos: int, grid: int) -> int:
    """CTA that takes list position pos: c, 2G-1-c, 2G+c, 4G-1-c, ..."""
    r = pos % (2 * grid)
    return r if r < grid else 2 * grid - 1 - r


def check_case(cached, new, group, hkv, grid):
    qpt = ROWS // group
    lst = unit_list(cached, new, qpt, hkv)
    # every (sequence, pair, KV head) exactly once, in the bucket of its own KV tiles
    seen = {}
    for b, s, pp, h in lst:
        assert (s, pp, h) not in seen, (s, pp, h)
        seen[(s, pp, h)] = b
    want = set()
    for s, (c, q) in enumerate(zip(cached, new)):
        _, P = tiles(q, qpt)
        for pp in range(P):
            na, nb = kv_tiles_of_pair(c, q, qpt, pp)
            assert nb <= na
            for h in range(hkv):
                want.add((s, pp, h))
                assert seen.get((s, pp, h)) == na, (s, pp, h, seen.get((s, pp, h)), na)
    assert set(seen) == want
    # the list is ordered from the most KV tiles to the fewest
    buckets = [b for b, _, _, _ in lst]
    assert buckets == sorted(buckets, reverse=True)
    # the snake deal: each CTA's positions, taken k = 0, 1, 2, ... as the kernel does,
    # cover the list once
    owners = [snake_owner(p, grid) for p in range(len(lst))]
    per_cta = {}
    for c in range(grid):
        k, mine = 0, []
        while True:
            pos = (k >> 1) * 2 * grid + ((2 * grid - 1 - c) if k & 1 else c)
            if pos >= len(lst):
                break
            mine.append(pos)
            k += 1
        per_cta[c] = mine
        assert all(owners[p] == c for p in mine)
    assert sorted(p for m in per_cta.values() for p in m) == list(range(len(lst)))


def test_ragged_batch_of_the_parity_tests():
    cached = [0, 0, 0, 17, 256, 300, 0, 5, 1024]
    new = [1, 63, 129, 47, 1, 200, 256, 64, 65]
    for group in (1, 2, 3, 7, 20, 128):
        for grid in (1, 7, 148):
            check_case(cached, new, group, 4, grid)


def test_random_batches():
    rnd = random.Random(23)
    for _ in range(300):
        n = rnd.randint(1, 12)
        cached = [rnd.choice([0, 0, rnd.randint(0, 3000), 128 * rnd.randint(0, 20)]) for _ in range(n)]
        new = [rnd.choice([1, rnd.randint(1, 300), rnd.randint(1, 3000)]) for _ in range(n)]
        group = rnd.choice([1, 2, 3, 4, 5, 7, 8, 16, 20, 64, 128])
        check_case(cached, new, group, rnd.choice([1, 2, 4, 8]), rnd.choice([1, 3, 148]))


def test_first_pair_edges():
    """Tile A's KV tiles fall as the pair index grows, and the closed form's bucket edges
    match a scan of the pairs (one-query sequences, exact tile boundaries)."""
    for qpt in (1, 6, 18, 42, 64, 128):
        for cached in (0, 1, 127, 128, 129, 1000):
            for q_len in (1, qpt, qpt + 1, 2 * qpt, 2 * qpt + 1, 1000):
                T, P = tiles(q_len, qpt)
                counts = [kv_tiles_of_pair(cached, q_len, qpt, pp)[0] for pp in range(P)]
                assert counts == sorted(counts, reverse=True)
                for b in range(0, max(counts) + 2):
                    scan = next((pp for pp in range(P) if counts[pp] <= b), P)
                    assert first_pair(cached, q_len, qpt, b) == scan, (qpt, cached, q_len, b)
