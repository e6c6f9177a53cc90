"""Seeded synthetic inputs for the attention forward, the CSR-sparse attention and the merge.

This module only draws numbers and builds index structures (sequence lengths, CSR patterns).
It holds none of the attention arithmetic, so both the CUDA path and the float64 oracle can
consume what it produces without sharing any of the method's code.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)`` as float32
N(0, 1) and, for bf16 workloads, rounded to bf16 with torch's round-to-nearest-even cast.
The same host arrays feed the oracle (widened exactly to float64) and the device copy.

Workload shapes follow the pages:
  * dense BHSD attention ("flash attention的调用", MultiHeadAttention example; the
    ``(batch, heads, seq_len, head_dim)`` shape rule of the torch.nn.attention blog),
  * packed TND varlen attention with cumulative lengths and GQA head ratios
    (aclnnFlashAttentionVarLenScore, constraints section),
  * CSR-sparse attention over [B, H, S, D] fp32 (paddle.nn.functional.sparse_attention),
  * the ring-attention merge in SBH layout with [B, N, S, 8] statistics
    (npu_ring_attention_update, interface and example).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np
import torch

# Layout / mask / dtype codes, matching the values of the C header enums.
BHSD, TND = 0, 1
MASK_NONE, MASK_CAUSAL_TOPLEFT, MASK_CAUSAL_BOTTOMRIGHT = 0, 1, 2
BF16, F32, F16 = 0, 1, 2


def dtype_code(dtype: torch.dtype) -> int:
    return {torch.bfloat16: BF16, torch.float32: F32, torch.float16: F16}[dtype]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn(shape: Sequence[int], seed: int, dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """i.i.d. N(0,1) float32 draws on the CPU, cast (RNE) to ``dtype``."""
    x = torch.randn(tuple(int(s) for s in shape), generator=_gen(seed), dtype=torch.float32)
    return x if dtype == torch.float32 else x.to(dtype)


def mix_seed(config_index: int, seed: int, stream: int = 0) -> int:
    """Distinct seeds per (config, seed, tensor) so that Q, K and V are independent."""
    return (int(config_index) * 1_000_003 + int(seed) * 7919 + int(stream) * 104_729) & 0x7FFFFFFF


def cu_seqlens_from_lengths(lengths: Sequence[int]) -> np.ndarray:
    """Cumulative lengths with B entries and no leading zero.

    aclnnFlashAttentionVarLenScore, constraints on actualSeqQLenOptional: lengths
    [2, 2, 0, 2, 2] are passed as [2, 4, 4, 6, 8].
    """
    return np.cumsum(np.asarray(lengths, dtype=np.int64)).astype(np.int32)


def lengths_from_cu_seqlens(cu: Sequence[int]) -> np.ndarray:
    cu = np.asarray(cu, dtype=np.int64)
    return np.diff(np.concatenate([[0], cu])).astype(np.int64)


def varlen_lengths(n_seq: int, max_len: int, seed: int, zero_index: Optional[int] = 7) -> np.ndarray:
    """Integers uniform on [0, max_len] inclusive; one index forced to 0 (an empty sequence)."""
    g = _gen(seed)
    lens = torch.randint(0, max_len + 1, (n_seq,), generator=g, dtype=torch.int64).numpy()
    if zero_index is not None and 0 <= zero_index < n_seq:
        lens[zero_index] = 0
    return lens


def window_stride_pattern(S: int, half_window: int = 128, stride: int = 64) -> tuple[np.ndarray, np.ndarray]:
    """CSR row pointer and sorted columns of a local window plus a strided global set.

    Row i keeps {j : i - half_window <= j <= i + half_window - 1, 0 <= j < S} united with
    {j : j mod stride == 0}, sorted and without duplicates. For S = 4096, a 256-wide
    window and every 64th column this gives 1,278,208 stored entries.
    """
    rows: List[np.ndarray] = []
    glob = np.arange(0, S, stride, dtype=np.int64)
    for i in range(S):
        lo, hi = max(0, i - half_window), min(S, i + half_window)
        win = np.arange(lo, hi, dtype=np.int64)
        rows.append(np.union1d(win, glob))
    offs = np.zeros(S + 1, dtype=np.int64)
    offs[1:] = np.cumsum([len(r) for r in rows])
    cols = np.concatenate(rows)
    return offs.astype(np.int32), cols.astype(np.int32)


# ----------------------------------------------------------------------------------------------
# Concrete workloads
# ----------------------------------------------------------------------------------------------
@dataclasses.dataclass
class AttnInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    layout: int
    mask_mode: int
    dtype: int
    B: int
    Sq: int          # BHSD: per-sequence length; TND: total query tokens
    Skv: int         # BHSD: per-sequence length; TND: total key tokens
    Nq: int
    Nkv: int
    D: int
    scale: float
    cu_q: Optional[np.ndarray] = None   # TND only: int32 [B], no leading zero
    cu_kv: Optional[np.ndarray] = None


def dense_bhsd(B, H, S, D, *, causal: bool, dtype: torch.dtype, seed: int, cfg: int,
               Hkv: Optional[int] = None, Skv: Optional[int] = None) -> AttnInputs:
    Hkv = H if Hkv is None else Hkv
    Skv = S if Skv is None else Skv
    q = randn((B, H, S, D), mix_seed(cfg, seed, 0), dtype)
    k = randn((B, Hkv, Skv, D), mix_seed(cfg, seed, 1), dtype)
    v = randn((B, Hkv, Skv, D), mix_seed(cfg, seed, 2), dtype)
    return AttnInputs(q, k, v, BHSD, MASK_CAUSAL_TOPLEFT if causal else MASK_NONE,
                      dtype_code(dtype), B, S, Skv, H, Hkv, D,
                      1.0 / float(np.sqrt(D)))


def varlen_tnd(lengths_q, Nq, Nkv, D, *, causal: bool, dtype: torch.dtype, seed: int, cfg: int,
               lengths_kv=None, mask_mode: Optional[int] = None) -> AttnInputs:
    lengths_kv = lengths_q if lengths_kv is None else lengths_kv
    cu_q = cu_seqlens_from_lengths(lengths_q)
    cu_kv = cu_seqlens_from_lengths(lengths_kv)
    Tq, Tk = int(cu_q[-1]) if len(cu_q) else 0, int(cu_kv[-1]) if len(cu_kv) else 0
    q = randn((Tq, Nq, D), mix_seed(cfg, seed, 0), dtype)
    k = randn((Tk, Nkv, D), mix_seed(cfg, seed, 1), dtype)
    v = randn((Tk, Nkv, D), mix_seed(cfg, seed, 2), dtype)
    if mask_mode is None:
        mask_mode = MASK_CAUSAL_TOPLEFT if causal else MASK_NONE
    return AttnInputs(q, k, v, TND, mask_mode, dtype_code(dtype),
                      len(cu_q), Tq, Tk, Nq, Nkv, D, 1.0 / float(np.sqrt(D)), cu_q, cu_kv)


def cfg1_dense_small(dtype: torch.dtype, seed: int = 0) -> AttnInputs:
    """Dense SDPA forward, B=2, H=4, S=256, D=64, non-causal, scale 1/8."""
    return dense_bhsd(2, 4, 256, 64, causal=False, dtype=dtype, seed=seed, cfg=1)


def cfg2_dense_causal(seed: int = 0, B=8, H=16, S=4096, D=128) -> AttnInputs:
    """Dense MHA self-attention forward, bf16, B=8, H=16, S=4096, D=128, causal."""
    return dense_bhsd(B, H, S, D, causal=True, dtype=torch.bfloat16, seed=seed, cfg=2)


def cfg3_lengths(seed: int = 0, n_seq: int = 16, max_len: int = 8192) -> np.ndarray:
    return varlen_lengths(n_seq, max_len, mix_seed(3, seed, 9), zero_index=7)


def cfg3_varlen_gqa(seed: int = 0, n_seq: int = 16, max_len: int = 8192,
                    Nq: int = 32, Nkv: int = 8, D: int = 128) -> AttnInputs:
    """Varlen packed TND, bf16, 16 sequences of length U{0..8192} (index 7 forced to 0),
    Nq=32, Nkv=8 (GQA ratio 4), D=128, causal per sequence; shared cu_seqlens."""
    lens = cfg3_lengths(seed, n_seq, max_len)
    return varlen_tnd(lens, Nq, Nkv, D, causal=True, dtype=torch.bfloat16, seed=seed, cfg=3)


@dataclasses.dataclass
class CsrInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    offset: np.ndarray     # int32 [B, H, S+1]
    columns: np.ndarray    # int32 [B, H, nnz_cap]
    B: int
    H: int
    S: int
    D: int

    @property
    def nnz_cap(self) -> int:
        return int(self.columns.shape[-1])


def cfg4_csr(seed: int = 0, B=2, H=8, S=4096, D=64) -> CsrInputs:
    """CSR-sparse attention forward, fp32, B=2, H=8, S=4096, D=64, window 256 + every 64th."""
    offs, cols = window_stride_pattern(S)
    offset = np.broadcast_to(offs, (B, H, S + 1)).copy()
    columns = np.broadcast_to(cols, (B, H, cols.shape[0])).copy()
    q = randn((B, H, S, D), mix_seed(4, seed, 0))
    k = randn((B, H, S, D), mix_seed(4, seed, 1))
    v = randn((B, H, S, D), mix_seed(4, seed, 2))
    return CsrInputs(q, k, v, offset, columns, B, H, S, D)


def merge_stats_random(B, N, S, seed: int, lanes_equal: bool = True) -> tuple[torch.Tensor, torch.Tensor]:
    """Random [B, N, S, 8] fp32 (max, sum) statistics; sums positive (>= 1), as a real forward gives."""
    m = randn((B, N, S, 1 if lanes_equal else 8), seed)
    s = 1.0 + randn((B, N, S, 1 if lanes_equal else 8), seed + 1).abs() * 50.0
    if lanes_equal:
        m, s = m.expand(B, N, S, 8).contiguous(), s.expand(B, N, S, 8).contiguous()
    return m, s
