"""Host-side helpers for running the forward on several GPUs, one process per GPU.

Attention is independent per (sequence, head), so a packed varlen batch partitions across ranks
with no exchange at all: every rank takes a subset of the sequences, packs its own TND batch and
calls attn_fwd on it. These helpers choose the subset (balanced by algorithmic work) and build
the rank's packed index; the only collectives are for timing (barrier, max over ranks).
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np


def sequence_work(lq: int, lk: int, causal: bool) -> int:
    """Visible (query, key) pairs of one sequence (top-left causal when `causal`)."""
    if not causal:
        return int(lq) * int(lk)
    n = min(int(lq), int(lk))
    return n * (n + 1) // 2 + max(0, int(lq) - n) * int(lk)


def balanced_partition(lengths_q: Sequence[int], world: int, lengths_kv: Sequence[int] = None,
                       causal: bool = True) -> List[List[int]]:
    """Assign every sequence to one rank, longest-processing-time first (heaviest sequence to the
    least-loaded rank). Returns, per rank, the sorted sequence indices."""
    lengths_kv = lengths_q if lengths_kv is None else lengths_kv
    work = [sequence_work(a, b, causal) for a, b in zip(lengths_q, lengths_kv)]
    order = sorted(range(len(work)), key=lambda i: (-work[i], i))
    load = [0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda x: (load[x], x))
        parts[r].append(i)
        load[r] += work[i]
    return [sorted(p) for p in parts]


def local_token_index(cu_seqlens: Sequence[int], seqs: Sequence[int]) -> np.ndarray:
    """Token indices (into the global packed batch) of the chosen sequences, in order; gathering
    Q/K/V rows with them gives the rank's own packed batch."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    starts = np.concatenate([[0], cu[:-1]])
    if len(seqs) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(starts[s], cu[s], dtype=np.int64) for s in seqs])


def local_cu_seqlens(cu_seqlens: Sequence[int], seqs: Sequence[int]) -> np.ndarray:
    """Cumulative lengths (no leading zero) of the rank's packed batch."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = np.diff(np.concatenate([[0], cu]))
    return np.cumsum(lens[list(seqs)]).astype(np.int32)
