"""Host-side model of the decode's stream-K work split and of the merge's
record lookup, checked by brute force on random layouts.

The decode kernel gives CTA i of P the units [W*i/P, W*(i+1)/P) of the total
W; a work pair (sequence, KV head, column group) owns a contiguous run of
units (its full tiles, then its tail weight).  A CTA that decodes any of a
pair's tiles writes one partial record at slot pair + i, and the merge grid
reads the records of CTAs owner(pst) .. owner(pst + nt - 1), where
owner(u) = ((u + 1) * P - 1) // W, skipping CTAs whose range misses the
tiles when W < P.  These are the kernel's formulas restated; the checks
are the properties the kernel relies on: the ranges partition the units,
owner() inverts them, every record slot is unique and inside the workspace
((pairs + P) slots), and the merge reads exactly the records written.
"""
import random


def sk_begin(W, P, i):
    return W * i // P


def sk_owner(W, P, u):
    return ((u + 1) * P - 1) // W


def check_layout(tiles, tail_units, P):
    pairs = len(tiles)
    units = [t + tu for t, tu in zip(tiles, tail_units)]
    starts = [0]
    for u in units:
        starts.append(starts[-1] + u)
    W = starts[-1]
    assert W > 0
    # the ranges partition [0, W) in order
    prev = 0
    for i in range(P):
        b, e = sk_begin(W, P, i), sk_begin(W, P, i + 1)
        assert b == prev and b <= e
        prev = e
    assert prev == W
    # owner() returns the CTA whose range holds the unit
    for u in range(W):
        o = sk_owner(W, P, u)
        assert 0 <= o < P and sk_begin(W, P, o) <= u < sk_begin(W, P, o + 1)
    # records written: CTA i writes slot pair + i for each pair whose tiles its range meets
    written = {}
    for i in range(P):
        b, e = sk_begin(W, P, i), sk_begin(W, P, i + 1)
        for p in range(pairs):
            t0, t1 = starts[p], starts[p] + tiles[p]
            if max(b, t0) < min(e, t1):
                slot = p + i
                assert slot not in written, "two records share a slot"
                assert slot < pairs + P
                written[slot] = (p, i)
    # the merge's lookup reads exactly the records written for each pair
    dense = W >= P
    for p in range(pairs):
        pst, nt = starts[p], tiles[p]
        want = {i for (q, i) in written.values() if q == p}
        got = set()
        if nt > 0:
            lo, hi = sk_owner(W, P, pst), sk_owner(W, P, pst + nt - 1)
            for i in range(lo, hi + 1):
                live = dense or max(sk_begin(W, P, i), pst) < min(sk_begin(W, P, i + 1), pst + nt)
                if live:
                    got.add(i)
        assert got == want, (p, sorted(got), sorted(want))


def test_stream_k_small_exhaustive():
    for pairs in range(1, 5):
        for P in range(1, 12):
            for t in range(0, 6):
                check_layout([t] * pairs, [14 if t % 2 else 3] * pairs, P)


def test_stream_k_random_layouts():
    rng = random.Random(2024)
    for _ in range(300):
        pairs = rng.randint(1, 40)
        P = rng.choice([1, 2, 7, 64, 148, 296, 320])
        tiles = [rng.choice([0, 0, 1, 2, 5, 31, 128, rng.randint(0, 300)]) for _ in range(pairs)]
        tails = [rng.choice([3, 14, 14 + 32]) for _ in range(pairs)]
        check_layout(tiles, tails, P)


def test_stream_k_model_catches_a_wrong_owner():
    """The checks are sharp: an owner() off by one fails them."""
    global sk_owner
    good = sk_owner
    try:
        sk_owner = lambda W, P, u: min(P - 1, good(W, P, u) + (1 if u % 7 == 3 else 0))
        failed = False
        try:
            check_layout([5, 9, 2, 0, 30], [14, 3, 14, 3, 14], 7)
        except AssertionError:
            failed = True
        assert failed
    finally:
        sk_owner = good
