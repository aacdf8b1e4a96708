"""Host-side model of the flat decode gather's work partition (the long-list kernel of
decode_gather.cu), checked on random list mixes: CTA ranges of the flat key list, stages that
never cross a list's end, the partial slot each split list writes, and the ticket count its
merge waits for.  The arithmetic below restates the kernel's formulas; the checks are the
invariants they must satisfy (every key streamed exactly once, no two partials in one slot,
the merge finding every partial of its list)."""
import random

STAGE = 64


def partition(counts, grid):
    off = [0]
    for k in counts:
        off.append(off[-1] + k)
    T = off[-1]
    if T == 0:
        return None
    G = min(grid, max(1, T // 32))  # CTAs in use: at most one per 32 keys
    return off, T, G


def owner(x, T, G):
    return ((x + 1) * G - 1) // T


def walk(off, lo, hi):
    """The stages of one CTA range, as (list, first key, end key)."""
    P = len(off) - 1
    p, ph = 0, P - 1
    while p < ph:  # the largest p with off[p] <= lo
        mid = (p + ph + 1) // 2
        if off[mid] <= lo:
            p = mid
        else:
            ph = mid - 1
    g = lo
    while g < hi:
        g1 = min(g + STAGE, min(off[p + 1], hi))
        yield p, g, g1
        g = g1
        while g < hi and off[p + 1] <= g:
            p += 1


def check(counts, grid):
    part = partition(counts, grid)
    if part is None:
        return
    off, T, G = part
    seen = [0] * T
    slots, tickets, whole = {}, {}, set()
    for c in range(G):
        lo, hi = T * c // G, T * (c + 1) // G
        assert lo < hi
        for p, g0, g1 in walk(off, lo, hi):
            assert off[p] <= g0 < g1 <= off[p + 1] and g1 - g0 <= STAGE
            for x in range(g0, g1):
                seen[x] += 1
            seg_lo, seg_hi = max(off[p], lo), min(off[p + 1], hi)
            if g1 != seg_hi:
                continue
            if seg_lo == off[p] and seg_hi == off[p + 1]:
                whole.add(p)
                continue
            slot = 2 * c if seg_lo > off[p] else 2 * c + 1
            assert slot not in slots and slot < 2 * G
            slots[slot] = p
            tickets[p] = tickets.get(p, 0) + 1
    assert seen == [1] * T
    for p, k in enumerate(counts):
        if k == 0:
            continue
        cf, cl = owner(off[p], T, G), owner(off[p + 1] - 1, T, G)
        if p in whole:
            assert cf == cl and p not in tickets
            continue
        assert tickets[p] == cl - cf + 1
        for cc in range(cf, cl + 1):  # the merge's view of each partial's slot
            lo_c = T * cc // G
            assert slots[2 * cc if lo_c > off[p] else 2 * cc + 1] == p


def test_flat_gather_partition_random_mixes():
    rng = random.Random(7)
    for _ in range(1500):
        P = rng.randint(1, 60)
        r = rng.random()
        if r < 0.3:
            counts = [rng.randint(0, 5) for _ in range(P)]
        elif r < 0.6:
            counts = [rng.randint(0, 400) for _ in range(P)]
        else:
            counts = [rng.choice([0, 1, 7, 64, 65, 128, 1000, 5000]) for _ in range(P)]
        check(counts, rng.choice([1, 2, 3, 148, 160]))


def test_flat_gather_partition_workload_shapes():
    check([131072] * 40, 148)   # p = 1 at 128K, B = 8
    check([1048576] * 5, 148)   # p = 1 at 1M
    check([5918] * 40, 148)     # clustered 128K (mean set)
    check([0, 0, 5], 148)       # empty lists before a short one
    check([1], 148)             # a single key
