"""Work accounting for the MoBA causal prefill forward (host arithmetic only).

Attention work is counted in attended (query, key) pairs: a query in block
c = floor(t / B) attends min(c, k - 1) full past blocks plus the keys of its own
block up to and including itself. Each pair costs 2d FLOPs for q.k and 2d for
p.v. The nominal sparsity 1 - B k / N is the figure the "KIMI MoBA" blog uses in
its section 3 block_size / top_k table.
"""
from __future__ import annotations


def nblocks(N: int, block_size: int) -> int:
    return (N + block_size - 1) // block_size


def nominal_sparsity(N: int, block_size: int, topk: int) -> float:
    """1 - B k / N: the share of a length-N context that one query does not read."""
    return 1.0 - block_size * topk / N


def useful_pairs_per_head(N: int, block_size: int, topk: int) -> int:
    """Sum over t of min(c(t), k-1) * B + (t - c(t) * B + 1)."""
    total = 0
    for c in range(nblocks(N, block_size)):
        n_c = min(block_size, N - c * block_size)
        total += n_c * min(c, topk - 1) * block_size + n_c * (n_c + 1) // 2
    return total


def dense_causal_pairs_per_head(N: int) -> int:
    return N * (N + 1) // 2


def useful_flops(B: int, Hq: int, N: int, d: int, block_size: int, topk: int) -> float:
    return 4.0 * d * B * Hq * useful_pairs_per_head(N, block_size, topk)


def dense_causal_flops(B: int, Hq: int, N: int, d: int) -> float:
    return 4.0 * d * B * Hq * dense_causal_pairs_per_head(N)


def gate_scores(B: int, Hq: int, N: int, block_size: int) -> int:
    """Number of past-block scores the gate forms: sum over t of c(t)."""
    total = 0
    for c in range(nblocks(N, block_size)):
        total += min(block_size, N - c * block_size) * c
    return B * Hq * total


def min_io_bytes(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    """Q, K, V read once and out (bf16) plus lse (fp32) written once."""
    return 2 * B * N * d * (2 * Hq + 2 * Hkv) + 4 * B * Hq * N
