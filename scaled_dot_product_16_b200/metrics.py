"""Algorithmic work of each operation, used to turn measured times into throughput.

attn_fwd:        4 * Nq * D FLOPs per visible (query, key) pair (QK^T and PV, 2 FLOPs per
                 multiply-add); causal masks count the diagonal, so a sequence of length L has
                 L(L+1)/2 pairs per head.
attn_sparse_csr: 4 * D FLOPs per stored entry.
attn_merge:      bytes that must move: read prev/cur outputs and 4 statistic arrays, write the
                 output and 2 statistic arrays.
"""
from __future__ import annotations

import numpy as np

from . import workloads as W


def seq_lengths(inp: W.AttnInputs):
    if inp.layout == W.BHSD:
        return [inp.Sq] * inp.B, [inp.Skv] * inp.B
    return (W.lengths_from_cu_seqlens(inp.cu_q).tolist(), W.lengths_from_cu_seqlens(inp.cu_kv).tolist())


def visible_pairs(inp: W.AttnInputs) -> int:
    tot = 0
    for sq, sk in zip(*seq_lengths(inp)):
        if inp.mask_mode == W.MASK_NONE:
            tot += sq * sk
            continue
        off = 0 if inp.mask_mode == W.MASK_CAUSAL_TOPLEFT else sk - sq
        rows = np.clip(np.arange(sq, dtype=np.int64) + off + 1, 0, sk)
        tot += int(rows.sum())
    return int(tot)


def attn_fwd_flops(inp: W.AttnInputs) -> int:
    return 4 * inp.Nq * inp.D * visible_pairs(inp)


def band_pairs(inp: W.AttnInputs, pre: int, nxt: int) -> int:
    """(query, key) pairs with i - pre <= j <= i + nxt (in-sequence positions), summed over the
    sequences: the visible pairs of the band mode."""
    tot = 0
    for sq, sk in zip(*seq_lengths(inp)):
        i = np.arange(sq, dtype=np.int64)
        lo = np.clip(i - pre, 0, sk)
        hi = np.clip(i + nxt + 1, 0, sk)
        tot += int(np.maximum(hi - lo, 0).sum())
    return int(tot)


def attn_fwd_min_bytes(inp: W.AttnInputs) -> int:
    """Compulsory HBM traffic: read Q, K, V once, write O and the two statistics."""
    e = 2 if inp.dtype == W.BF16 else 4
    q = inp.q.numel() * e
    kv = 2 * inp.k.numel() * e
    return int(q + kv + q + 2 * 4 * (inp.q.numel() // inp.D))


def csr_flops(inp: W.CsrInputs) -> int:
    return 4 * inp.D * int(inp.offset[..., -1].astype(np.int64).sum())


def csr_min_bytes(inp: W.CsrInputs, elem: int = 4) -> int:
    """Compulsory HBM traffic of attn_sparse_csr: q, k, v read and out written once, plus the
    column indices and row pointers."""
    qkvo = 4 * inp.B * inp.H * inp.S * inp.D * elem
    return int(qkvo + inp.columns.size * 4 + inp.offset.size * 4)


def merge_bytes(S: int, B: int, N: int, D: int, elem: int) -> int:
    out = S * B * N * D * elem
    stats = B * N * S * 8 * 4
    return 3 * out + 6 * stats
