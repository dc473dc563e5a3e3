"""A model of the decode gate's top-k (moba_decode_select_kernel in k_decode.cuh), checked against a plain
sort on the cases that parity data rarely reaches: equal scores, rows of -inf scores (what a NaN score
ranks as) and slices with fewer blocks than k - 1.

The kernel splits the c candidate blocks into 16 contiguous slices (one per warp). A block's rank in its
slice is the number of the slice's blocks that rank before it by (score desc, index asc), and the
blocks of rank < k - 1 are the slice's list. The head's k - 1 blocks are the list entries of rank
< k - 1 among all listed entries, returned in ascending block order. The model follows those steps;
the reference is the sorted order itself. A planted mistake (ranks by score alone, without the index
tie-break) must be caught.
"""
import math
import random

NW = 16


def before(s2, j2, s, j):
    return s2 > s or (s2 == s and j2 < j)


def kernel_select(scores, kp, before=before):
    c = len(scores)
    sc = [(-math.inf if s != s else s) for s in scores]  # a NaN score ranks as -inf
    listed = []
    for w in range(NW):
        lo, hi = c * w // NW, c * (w + 1) // NW
        for i in range(lo, hi):
            rank = sum(before(sc[k], k, sc[i], i) for k in range(lo, hi))
            if rank < kp:
                listed.append((sc[i], i))
    kept = []
    for s, j in listed:
        rank = sum(before(s2, j2, s, j) for s2, j2 in listed)
        if rank < kp:
            kept.append(j)
    return sorted(kept)


def reference_select(scores, kp):
    keyed = [(-(-math.inf if s != s else s), j) for j, s in enumerate(scores)]
    return sorted(j for _, j in sorted(keyed)[:kp])


def test_rank_count_selection_equals_a_sort():
    rng = random.Random(7)
    for trial in range(400):
        c = rng.choice([12, 13, 16, 17, 31, 40, 63, 100, 255, 400])
        kp = rng.choice([1, 2, 3, 11, 31, 63])
        if kp >= c:
            continue
        kind = trial % 4
        if kind == 0:    # distinct scores
            scores = [rng.gauss(0, 1) for _ in range(c)]
        elif kind == 1:  # heavy ties: a few distinct values
            vals = [rng.gauss(0, 1) for _ in range(3)]
            scores = [rng.choice(vals) for _ in range(c)]
        elif kind == 2:  # NaN scores (rank as -inf) mixed in
            scores = [float("nan") if rng.random() < 0.3 else rng.gauss(0, 1) for _ in range(c)]
        else:            # every score NaN: the lowest block indices are kept
            scores = [float("nan")] * c
        assert kernel_select(scores, kp) == reference_select(scores, kp), (trial, c, kp, kind)


def test_all_nan_row_keeps_the_lowest_blocks():
    assert kernel_select([float("nan")] * 40, 11) == list(range(11))


def test_model_catches_ranks_without_the_index_tie_break():
    rng = random.Random(3)
    wrong = lambda s2, j2, s, j: s2 > s
    caught = 0
    for _ in range(50):
        vals = [rng.gauss(0, 1) for _ in range(3)]
        scores = [rng.choice(vals) for _ in range(64)]
        caught += kernel_select(scores, 11, before=wrong) != reference_select(scores, 11)
    assert caught > 25
