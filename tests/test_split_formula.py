"""Host logic of the range-balanced work split (MLA decode: 64-token tiles with a weight of
8 positions per sequence; FP8 paged decode: 16-token pages, no weight), restated here:

* the kernel side: range c of P takes positions [N c / P, N (c + 1) / P) of a space in
  which a non-empty sequence of n units takes SEG + n positions (unit u at SEG + u) and
  writes one partial per sequence whose units it holds (its segments);
* the merge side: the ranges meeting sequence b run from the one holding its first unit
  to the one holding its last, c = floor(((x + 1) P - 1) / N) for position x.

Checked on random layouts (empty sequences, single-unit sequences, more ranges than
units): every unit is computed by exactly one range, and the merge reads exactly the
partials the kernel writes."""
import numpy as np


def segments(units, P, SEG):
    N = sum(n + SEG for n in units if n > 0)
    out = {}
    for c in range(P):
        lo, hi = N * c // P, N * (c + 1) // P
        s = 0
        for b, n in enumerate(units):
            if n == 0:
                continue
            first = s + SEG
            a, e = max(lo - first, 0), min(hi - first, n)
            if e > a:
                out.setdefault(b, []).append((c, a, e))
            s += n + SEG
    return N, out


def merge_ranges(units, P, SEG, N):
    got = {}
    s = 0
    for b, n in enumerate(units):
        if n == 0:
            continue
        f, e = s + SEG, s + SEG + n
        c0, c1 = ((f + 1) * P - 1) // N, (e * P - 1) // N
        got[b] = [c for c in range(c0, c1 + 1) if N * (c + 1) // P > N * c // P]
        s += n + SEG
    return got


def test_split_and_merge_agree_on_random_layouts():
    rng = np.random.default_rng(2026)
    for trial in range(3000):
        B = int(rng.integers(1, 40))
        kind = trial % 3
        if kind == 0:
            units = rng.integers(0, 600, B)
        elif kind == 1:
            units = rng.integers(0, 3, B)  # many empty and one-unit sequences
        else:
            units = np.where(rng.random(B) < 0.3, 0, rng.integers(1, 40, B))
        units = [int(u) for u in units]
        for P, SEG in ((74, 8), (74, 0), (148, 0), (3, 8)):
            if sum(units) == 0:
                continue
            N, segs = segments(units, P, SEG)
            for b, n in enumerate(units):
                tiles = sorted(t for c, a, e in segs.get(b, []) for t in range(a, e))
                assert tiles == list(range(n)), (units, P, SEG, b)
            want = merge_ranges(units, P, SEG, N)
            for b, n in enumerate(units):
                if n:
                    assert [c for c, _, _ in segs[b]] == want[b], (units, P, SEG, b)
            # slot c + b is unique over all (range, sequence) pairs that write one
            slots = [c + b for b, lst in segs.items() for c, _, _ in lst]
            assert len(slots) == len(set(slots))
