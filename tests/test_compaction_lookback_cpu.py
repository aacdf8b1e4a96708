"""Host-side model of the clustered selection's single-pass compaction (cluster.cu): chunks take
indices in start order, publish their own count, then look back over their predecessors' flags
32 at a time to the nearest inclusive count.  The model runs the protocol under random
interleavings of the chunks' steps and checks the invariants the kernel relies on: every chunk
gets the exact exclusive prefix of the counts before it, flags left by an earlier launch (an
older epoch) are never taken, and no chunk waits on one that has not started."""
import random

VALUE_BITS = 38


def flag(epoch, status, value):
    return (epoch << 40) | (status << 38) | (value & ((1 << VALUE_BITS) - 1))


def unpack(f):
    return f >> 40, (f >> 38) & 3, f & ((1 << VALUE_BITS) - 1)


def lookback_step(flags, chunk, top, epoch):
    """One warp-wide step of chunk `chunk`'s look-back from predecessor `top` down: returns
    (ready, add, done) -- whether the needed flags are published, the sum they add, and whether
    an inclusive count was reached."""
    lanes = []
    for lane in range(32):
        j = top - lane
        if j < 0:
            lanes.append((True, True, 0))  # before chunk 0: an inclusive count of 0
            continue
        ep, st, v = unpack(flags[j])
        ok = ep == epoch and st != 0
        lanes.append((ok, ok and st == 2, v))
    inc = [i for i, (_, inc_, _) in enumerate(lanes) if inc_]
    L = inc[0] if inc else 31
    if not all(lanes[i][0] for i in range(L + 1)):
        return False, 0, False
    add = sum(v for i, (_, _, v) in enumerate(lanes[:L + 1]) if top - i >= 0)
    return True, add, bool(inc)


def run_launch(counts, flags, epoch, rng):
    n = len(counts)
    started, state = [], {}
    order = list(range(n))  # CTAs start in some order; chunk indices follow start order
    rng.shuffle(order)
    next_chunk = 0
    pending = list(order)
    result = {}
    steps = 0
    while len(result) < n:
        steps += 1
        assert steps < 200000, "no progress"
        # either start a new CTA or advance a running one
        if pending and (not state or rng.random() < 0.4):
            pending.pop()
            c = next_chunk
            next_chunk += 1
            started.append(c)
            if c == 0:
                flags[0] = flag(epoch, 2, counts[0])
                result[0] = 0
            else:
                flags[c] = flag(epoch, 1, counts[c])
                state[c] = [c - 1, 0]
            continue
        c = rng.choice(list(state))
        top, prefix = state[c]
        assert all(j in started for j in range(max(0, top - 31), top + 1)), "waits on an unstarted chunk"
        ready, add, done = lookback_step(flags, c, top, epoch)
        if not ready:
            continue
        prefix += add
        if done:
            flags[c] = flag(epoch, 2, prefix + counts[c])
            result[c] = prefix
            del state[c]
        else:
            state[c] = [top - 32, prefix]
    return result


def test_lookback_gives_exact_prefixes_under_random_interleavings():
    rng = random.Random(11)
    flags = [0] * 300
    epoch = 0
    for trial in range(200):
        epoch += 1
        n = rng.choice([1, 2, 5, 31, 32, 33, 64, 100, 256])
        counts = [rng.choice([0, 0, 1, 7, 4096, rng.randint(0, 4096)]) for _ in range(n)]
        got = run_launch(counts, flags, epoch, rng)
        want, acc = {}, 0
        for c in range(n):
            want[c] = acc
            acc += counts[c]
        assert got == want


def test_stale_flags_of_an_older_epoch_are_never_taken():
    rng = random.Random(3)
    flags = [flag(5, 2, 999999)] * 64  # inclusive counts left by an earlier launch
    counts = [rng.randint(0, 100) for _ in range(64)]
    got = run_launch(counts, flags, 6, rng)
    acc = 0
    for c in range(64):
        assert got[c] == acc
        acc += counts[c]
