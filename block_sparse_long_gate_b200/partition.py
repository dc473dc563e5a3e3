"""Split of one MoBA forward across ranks by groups of kv heads (one process per GPU).

Every query head h reads exactly one kv head, h // G (G = Hq / Hkv), and gates,
attends and merges on its own ("MoBA project hub", Steps 2-3: the gate scores a
query against the mean-pooled keys of its own head; nothing mixes heads). So the
forward of a contiguous range of kv heads, together with the G query heads of
each, depends on nothing outside that range: a rank runs the ordinary
single-GPU forward on its own contiguous head slices and no data moves between
ranks. This module is host logic only: which heads a rank owns, and how the
per-rank results fit back into the whole layout.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class HeadSlice:
    rank: int
    hkv0: int  # kv heads [hkv0, hkv1)
    hkv1: int
    hq0: int   # query heads [hq0, hq1) = [hkv0 * G, hkv1 * G)
    hq1: int

    @property
    def n_kv(self) -> int:
        return self.hkv1 - self.hkv0

    @property
    def n_q(self) -> int:
        return self.hq1 - self.hq0


def can_split(Hq: int, Hkv: int, world: int) -> bool:
    """True when every rank can own at least one kv head."""
    return world >= 1 and Hkv >= world and Hq % Hkv == 0


def head_slices(Hq: int, Hkv: int, world: int) -> list[HeadSlice]:
    """Contiguous, balanced kv-head ranges, one per rank (sizes differ by at most one),
    covering every head exactly once."""
    if not can_split(Hq, Hkv, world):
        raise ValueError(f"cannot split Hkv={Hkv} kv heads (Hq={Hq}) over {world} ranks")
    G = Hq // Hkv
    out = []
    for r in range(world):
        h0 = (r * Hkv) // world
        h1 = ((r + 1) * Hkv) // world
        out.append(HeadSlice(r, h0, h1, h0 * G, h1 * G))
    return out


def assemble(parts, Hq: int, Hkv: int):
    """Whole (out [B, N, Hq, d], lse [B, Hq, N]) from the per-rank results.

    `parts` is a list of (HeadSlice, out_r [B, N, n_q, d], lse_r [B, n_q, N]) torch tensors
    (any order, on one device)."""
    import torch

    parts = sorted(parts, key=lambda p: p[0].hq0)
    covered = [h for s, _, _ in parts for h in range(s.hq0, s.hq1)]
    if covered != list(range(Hq)):
        raise ValueError("the parts do not cover every query head exactly once")
    out = torch.cat([o for _, o, _ in parts], dim=2)
    lse = torch.cat([l for _, _, l in parts], dim=1)
    return out, lse
