"""The decode split: P equal slices of the flattened cache rows, pieces (slice w, sequence b)
stored in slot w + b, merged per sequence by the combine step.  This mirrors the index
arithmetic of the kernels on the CPU and checks coverage and slot uniqueness."""
import random

import pytest


def slice_start(N, w, P):
    return (N * w) // P


def slice_of(r, N, P):
    return ((r + 1) * P + N - 1) // N - 1


def pieces(seqlens, P):
    off = [0]
    for s in seqlens:
        off.append(off[-1] + max(s, 0))
    N = off[-1]
    out = []   # (w, b, row0, row1)
    for w in range(P):
        start, end = slice_start(N, w, P), slice_start(N, w + 1, P)
        if start >= end:
            continue
        b = max(i for i in range(len(seqlens)) if off[i] <= start)
        row = start
        while row < end:
            seg_end = min(end, off[b + 1])
            if seg_end > row:
                out.append((w, b, row, seg_end))
            row = seg_end
            b += 1
    return off, N, out


def combine_view(off, N, P, b):
    s0, s1 = off[b], off[b + 1]
    if s1 <= s0:
        return []
    lo, hi = slice_of(s0, N, P), slice_of(s1 - 1, N, P)
    return [w for w in range(lo, hi + 1) if slice_start(N, w + 1, P) > slice_start(N, w, P)]


@pytest.mark.parametrize("seed", range(40))
def test_partition_covers_rows_once_and_slots_are_unique(seed):
    rnd = random.Random(seed)
    B = rnd.choice([1, 2, 3, 7, 64, 200])
    hi = rnd.choice([1, 5, 40, 2000, 32768])
    seqlens = [rnd.randint(1, hi) for _ in range(B)]
    if seed % 5 == 0:
        seqlens[rnd.randrange(B)] = 0   # an invalid (empty) sequence
    P = rnd.choice([1, 4, 37, 296, 1184])
    off, N, ps = pieces(seqlens, P)
    covered = sorted((r0, r1) for _, _, r0, r1 in ps)
    pos = 0
    for r0, r1 in covered:
        assert r0 == pos and r1 > r0
        pos = r1
    assert pos == N
    slots = [w + b for w, b, _, _ in ps]
    assert len(set(slots)) == len(slots)
    assert all(0 <= s < P + B for s in slots)
    for w, b, r0, r1 in ps:
        assert off[b] <= r0 < r1 <= off[b + 1]
    for b in range(B):
        assert sorted(w for w, bb, _, _ in ps if bb == b) == combine_view(off, N, P, b)


def test_slice_of_inverts_slice_start():
    for N in [1, 2, 3, 10, 295, 296, 297, 1000, 1048576 + 7]:
        for P in [1, 3, 296, 1184]:
            for r in sorted({0, 1, N // 3, N // 2, N - 2, N - 1} & set(range(N))):
                w = slice_of(r, N, P)
                assert slice_start(N, w, P) <= r < slice_start(N, w + 1, P)
