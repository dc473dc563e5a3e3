"""A model of how the backward kernel (k_backward.cuh) packs P^T and dS^T into TMEM with two threads
per key row.

Threads h = 0 and 1 of a key row each take two 32-query chunks qq = 2h and 2h + 1: they read the fp32
columns [32 qq, 32 qq + 32) of S^T (and of dP^T), then store that chunk's 16 packed bf16 pairs at
column 64h + 16 (qq - 2h). The products dV += P^T dO and dK += dS^T Q read the 16 queries of k-step k
at column 8k + 32 [k >= 4]. The model checks, over every interleaving of the two threads' steps, that
no store lands on a column the other thread has still to read, and that the packed columns hold the
queries each k-step's product expects. Two planted mistakes must be caught: the one-thread-per-row
layout (chunk qq packed at column 16 qq) kept with two threads, and products that read k-step k at
column 8k, as they did with one thread per row.
"""
import itertools


def kernel_layout(h, qq):
    """First packed column of chunk qq, stored by thread h (the kernel's rule)."""
    return 64 * h + 16 * (qq - 2 * h)


def naive_layout(h, qq):
    """The single-thread layout: chunk qq at column 16 qq."""
    return 16 * qq


def mma_column(k):
    """Packed column the products read for queries 16k .. 16k + 15."""
    return 8 * k + (32 if k >= 4 else 0)


def thread_ops(h, layout):
    ops = []
    for qq in (2 * h, 2 * h + 1):
        ops.append(("read", h, set(range(32 * qq, 32 * qq + 32))))
        c0 = layout(h, qq)
        ops.append(("write", h, set(range(c0, c0 + 16)), qq))
    return ops


def interleavings(a, b):
    n, m = len(a), len(b)
    for pos in itertools.combinations(range(n + m), n):
        seq, ia, ib = [], 0, 0
        for i in range(n + m):
            if i in pos:
                seq.append(a[ia]); ia += 1
            else:
                seq.append(b[ib]); ib += 1
        yield seq


def check(layout, mma_col=mma_column):
    """Returns the list of violations over all interleavings (empty when the layout is safe)."""
    bad = []
    ops0, ops1 = thread_ops(0, layout), thread_ops(1, layout)
    need = {0: set().union(*(o[2] for o in ops0 if o[0] == "read")),
            1: set().union(*(o[2] for o in ops1 if o[0] == "read"))}
    for seq in interleavings(ops0, ops1):
        read = {0: set(), 1: set()}
        packed = {}  # column -> (query chunk, offset in the chunk's 16 columns)
        for op in seq:
            if op[0] == "read":
                read[op[1]] |= op[2]
            else:
                h, cols, qq = op[1], op[2], op[3]
                other = 1 - h
                clobbered = (need[other] - read[other]) & cols
                if clobbered:
                    bad.append(f"thread {h} stores chunk {qq} over columns {sorted(clobbered)[:4]}.. "
                               f"that thread {other} has not read")
                mine_unread = (need[h] - read[h]) & cols
                if mine_unread:
                    bad.append(f"thread {h} stores chunk {qq} over its own unread columns")
                for i, c in enumerate(sorted(cols)):
                    packed[c] = (qq, i)
        # every k-step reads its queries' pairs: column 8k + 32 [k >= 4] + i holds queries 16k + 2i, + 1
        for k in range(8):
            for i in range(8):
                col = mma_col(k) + i
                q = 16 * k + 2 * i  # first query of the pair
                want = (q // 32, (q % 32) // 2)
                if packed.get(col) != want:
                    bad.append(f"k-step {k}: column {col} holds {packed.get(col)}, the product expects {want}")
                    break
    return bad


def test_two_thread_packing_is_race_free_and_matches_the_products():
    assert check(kernel_layout) == []


def test_model_catches_the_single_thread_layout_with_two_threads():
    bad = check(naive_layout)
    assert any("has not read" in b for b in bad)


def test_model_catches_products_reading_the_single_thread_columns():
    bad = check(kernel_layout, mma_col=lambda k: 8 * k)
    assert any("the product expects" in b for b in bad)
