"""Host-side sharding of a packed variable-length batch across ranks.

Every (sequence, head) of the mixer is independent, so a batch shards across
GPUs by sequence with no collective on the data path: each rank runs the
mixer on its own sequences and the outputs are scattered back by token index.
Sequences are assigned longest first to the least-loaded rank (token count),
which bounds the imbalance by one sequence.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np


def assign_sequences(lengths, world_size: int) -> List[List[int]]:
    """Sequence indices per rank, longest-processing-time-first greedy."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    lengths = np.asarray(lengths, dtype=np.int64)
    load = np.zeros(world_size, dtype=np.int64)
    out: List[List[int]] = [[] for _ in range(world_size)]
    for n in sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i)):
        r = int(np.argmin(load))
        out[r].append(n)
        load[r] += int(lengths[n])
    for r in range(world_size):
        out[r].sort()
    return out


def shard_tokens(cu_seqlens, seq_ids) -> Tuple[np.ndarray, np.ndarray]:
    """(token indices of the given sequences in packed order, their cu_seqlens)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    idx = [np.arange(cu[n], cu[n + 1], dtype=np.int64) for n in seq_ids]
    tok = np.concatenate(idx) if idx else np.zeros(0, np.int64)
    lens = [int(cu[n + 1] - cu[n]) for n in seq_ids]
    new_cu = np.zeros(len(seq_ids) + 1, dtype=np.int32)
    new_cu[1:] = np.cumsum(lens)
    return tok, new_cu
