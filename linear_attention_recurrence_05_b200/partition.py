"""Data-parallel sharding of a prefill or decode batch over the ranks of a job.

Packed sequences (and decode rows) are independent: the gated delta rule of page
"ARCHITECTURE PREVIEW / FIELD NOTES", section 03 runs each sequence's state on its own, so a
batch shards by sequence with no exchange at all.  Prefill work is proportional to a
sequence's tokens, so sequences are spread to balance tokens; decode rows all cost the same
and are split evenly.  Host-side planning only: no arithmetic of the method happens here.
"""
from __future__ import annotations

import heapq

__all__ = ["balance_sequences", "split_rows", "rank_pack"]


def balance_sequences(lengths, world: int):
    """Sequence indices per rank, balancing tokens: longest sequence first, each to the rank
    holding the fewest tokens so far (ties to the lower rank).  The largest load is at most
    the mean load plus the longest sequence, and at most 4/3 of the best possible.  Each rank's
    list is returned in ascending index order (the packing order of its sub-batch)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    heap = [(0, r) for r in range(world)]
    parts = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        parts[r].append(i)
        heapq.heappush(heap, (load + int(lengths[i]), r))
    return [sorted(p) for p in parts]


def split_rows(n_rows: int, world: int):
    """Contiguous, near-equal ranges of decode rows per rank (the first n_rows % world ranks get
    one more row)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    base, extra = divmod(int(n_rows), world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append(range(lo, hi))
        lo = hi
    return out


def rank_pack(lengths, index):
    """Token ranges (start, stop) in the packed batch of the sequences `index` and the
    cu_seqlens of their own packed sub-batch."""
    starts, acc = [], 0
    for L in lengths:
        starts.append(acc)
        acc += int(L)
    spans = [(starts[i], starts[i] + int(lengths[i])) for i in index]
    cu, acc = [0], 0
    for a, b in spans:
        acc += b - a
        cu.append(acc)
    return spans, cu
