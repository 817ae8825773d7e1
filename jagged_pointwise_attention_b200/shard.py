"""Sharding a jagged batch across GPUs (host logic, no CUDA).

The attention forward has no cross-sequence term: every (sequence, head) pair
is an independent problem, and the layer's projections and LayerNorm are
row-local. A batch therefore splits across ranks by whole sequences with no
collective in the data path. Each sequence of length n costs about n(n+1)
causal score pairs, so sequences are assigned longest-processing-time first:
largest cost to the currently least-loaded rank.
"""

from __future__ import annotations

import heapq
from typing import List, Tuple

import numpy as np


def sequence_costs(lengths) -> np.ndarray:
    n = np.asarray(lengths, dtype=np.int64)
    return n * (n + 1)


def partition_sequences(lengths, world: int) -> List[np.ndarray]:
    """Indices of the sequences each rank owns (ascending within a rank).
    Deterministic: ties break by sequence index, then by rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = sequence_costs(lengths)
    order = sorted(range(len(cost)), key=lambda s: (-int(cost[s]), s))
    heap = [(0, r) for r in range(world)]
    owned: List[List[int]] = [[] for _ in range(world)]
    for s in order:
        load, r = heapq.heappop(heap)
        owned[r].append(s)
        heapq.heappush(heap, (load + int(cost[s]), r))
    return [np.array(sorted(o), dtype=np.int64) for o in owned]


def shard_offsets(seq_offsets, seqs) -> Tuple[np.ndarray, np.ndarray]:
    """For the listed sequences of a jagged batch: the token indices to gather
    (in order) and the local seq_offsets of the shard."""
    off = np.asarray(seq_offsets, dtype=np.int64)
    seqs = np.asarray(seqs, dtype=np.int64)
    lens = off[seqs + 1] - off[seqs]
    local = np.zeros(len(seqs) + 1, dtype=np.int64)
    np.cumsum(lens, out=local[1:])
    if len(seqs):
        tokens = np.concatenate([np.arange(off[s], off[s + 1]) for s in seqs])
    else:
        tokens = np.zeros(0, dtype=np.int64)
    return tokens, local
