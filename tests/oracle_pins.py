"""Pins that tie the float64 oracle to something other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with what the pages
or the mathematics fix. They are plain functions so that ``test_oracle_pins.py`` can run them
on the built oracle and ``test_oracle_mutants.py`` can run them on copies with planted
mistakes (every planted mistake must fail at least one pin).

What pins what:
  * the printed worked example of "paddle.nn.functional.sparse_attention" (CSR semantics),
  * the cumulative-length example of "aclnnFlashAttentionVarLenScore" (varlen decoding),
  * torch's own float64 scaled_dot_product_attention / logsumexp (library routines, an
    independent implementation of the dense definition, with causal, GQA and explicit masks),
  * closed forms and invariants (one visible key, Q = 0, V = 1, key shifts, merge of chunked
    partials equals the full result, merge with itself or with an empty side),
  * torch's float32 -> bfloat16 cast (rounding).
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from scaled_dot_product_16_b200 import workloads as W
from tests.golden.loader import load as load_golden

BHSD, TND = W.BHSD, W.TND
NONE, TL, BR = W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, W.MASK_CAUSAL_BOTTOMRIGHT


def _rng(seed):
    return np.random.default_rng(seed)


def _torch_sdpa(q, k, v, *, causal=False, mask=None, scale=None, gqa=False):
    return F.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale, enable_gqa=gqa).numpy()


def _bhsd(q, k, v, mask_mode, scale=None):
    B, Nq, Sq, D = q.shape
    _, Nkv, Skv, _ = k.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    return oracle.attn_fwd(q, k, v, B=B, Sq=Sq, Skv=Skv, Nq=Nq, Nkv=Nkv, D=D, scale=scale,
                           mask_mode=mask_mode, layout=BHSD)


# ---------------------------------------------------------------------------------------------
# CSR
# ---------------------------------------------------------------------------------------------
def pin_paddle_worked_example():
    g = load_golden("paddle_sparse_attention_example.txt")
    shape = tuple(int(x) for x in g["shape"])
    q = g["query"].astype(np.float32).reshape(shape)
    k = g["key"].astype(np.float32).reshape(shape)
    v = g["value"].astype(np.float32).reshape(shape)
    off = g["offset"].astype(np.int32).reshape(1, 1, -1)
    col = g["columns"].astype(np.int32).reshape(1, 1, -1)
    out = oracle.sparse_csr(q, k, v, off, col, B=1, H=1, S=shape[2], D=shape[3])
    want = g["output"].reshape(shape)
    # the page prints float32 results to 8 decimals
    assert np.max(np.abs(out - want)) <= 1e-6, (out, want)


def pin_csr_full_pattern_is_dense():
    r = _rng(1)
    B, H, S, D = 2, 3, 9, 5
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    cols = np.tile(np.arange(S, dtype=np.int32), S)
    off = np.arange(0, S * S + 1, S, dtype=np.int32)
    out = oracle.sparse_csr(q, k, v, np.broadcast_to(off, (B, H, S + 1)),
                            np.broadcast_to(cols, (B, H, S * S)), B=B, H=H, S=S, D=D)
    assert np.max(np.abs(out - _torch_sdpa(q, k, v))) <= 1e-12


def pin_csr_lower_triangle_is_causal():
    r = _rng(2)
    B, H, S, D = 1, 2, 11, 4
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    rows = [np.arange(i + 1, dtype=np.int32)[::-1] for i in range(S)]  # unsorted on purpose
    off = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    cols = np.concatenate(rows).astype(np.int32)
    out = oracle.sparse_csr(q, k, v, np.broadcast_to(off, (B, H, S + 1)),
                            np.broadcast_to(cols, (B, H, cols.size)), B=B, H=H, S=S, D=D)
    assert np.max(np.abs(out - _torch_sdpa(q, k, v, causal=True))) <= 1e-12


def pin_csr_single_and_empty_rows():
    r = _rng(3)
    B, H, S, D = 1, 1, 4, 3
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    # row 0: column 2 only; row 1: empty; row 2: column 3 twice; row 3: columns 0 and 1
    cols = np.array([2, 3, 3, 0, 1], dtype=np.int32).reshape(1, 1, -1)
    off = np.array([0, 1, 1, 3, 5], dtype=np.int32).reshape(1, 1, -1)
    out = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    assert np.array_equal(out[0, 0, 0], v[0, 0, 2])
    assert np.all(out[0, 0, 1] == 0.0)
    assert np.max(np.abs(out[0, 0, 2] - v[0, 0, 3])) <= 1e-15
    s = np.array([q[0, 0, 3] @ k[0, 0, 0], q[0, 0, 3] @ k[0, 0, 1]]) / math.sqrt(D)
    p = np.exp(s - s.max())
    p /= p.sum()
    assert np.max(np.abs(out[0, 0, 3] - (p[0] * v[0, 0, 0] + p[1] * v[0, 0, 1]))) <= 1e-14


def pin_csr_repeated_columns_weigh_per_entry():
    """A column stored c times in a row weighs c times (the row pointer counts entries): each
    row equals torch's float64 attention of its query over the key/value rows gathered entry
    by entry, repeats included."""
    r = _rng(31)
    B, H, S, D = 1, 1, 6, 4
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    rows = [[1, 4, 1], [2, 2, 2, 5], [0, 3, 0, 3, 3], [5], [], [4, 0, 4, 0, 1, 4]]
    off = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32).reshape(1, 1, -1)
    cols = np.concatenate([np.array(x, np.int32) for x in rows]).reshape(1, 1, -1)
    out = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    for i, row in enumerate(rows):
        if not row:
            assert np.all(out[0, 0, i] == 0.0)
            continue
        kk = torch.from_numpy(k[0, 0, row]).view(1, 1, len(row), D)
        vv = torch.from_numpy(v[0, 0, row]).view(1, 1, len(row), D)
        qq = torch.from_numpy(q[0, 0, i:i + 1]).view(1, 1, 1, D)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv).view(D).numpy()
        assert np.max(np.abs(out[0, 0, i] - ref)) <= 1e-13


def pin_csr_heads_independent():
    """Each (b, h) slice uses its own row pointer and columns."""
    r = _rng(4)
    B, H, S, D = 2, 2, 5, 3
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    off = np.zeros((B, H, S + 1), np.int32)
    cols = np.zeros((B, H, S), np.int32)
    for b in range(B):
        for h in range(H):
            off[b, h] = np.arange(S + 1)
            cols[b, h] = (np.arange(S) + b + 2 * h) % S  # row i keeps one column
    out = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    for b in range(B):
        for h in range(H):
            for i in range(S):
                assert np.array_equal(out[b, h, i], v[b, h, cols[b, h, i]])


def pin_csr_rejects_bad_columns():
    q = np.zeros((1, 1, 2, 2))
    try:
        oracle.sparse_csr(q, q, q, np.array([[[0, 1, 2]]], np.int32), np.array([[[0, 2]]], np.int32),
                          B=1, H=1, S=2, D=2)
    except ValueError:
        return
    raise AssertionError("column 2 of a 2-row slice was accepted")


def _rejected(call) -> bool:
    try:
        call()
    except ValueError:
        return True
    return False


def pin_csr_rejects_bad_row_pointers():
    """The row pointer must start at 0, never decrease and end within nnz_cap (the offset
    argument read as a row pointer); anything else is refused, never computed."""
    q = np.zeros((1, 1, 3, 2))
    cols = np.zeros((1, 1, 4), np.int32)
    for off in ([1, 2, 3, 4], [0, 3, 2, 4], [0, 1, 2, 5]):
        o = np.array(off, np.int32).reshape(1, 1, -1)
        assert _rejected(lambda: oracle.sparse_csr(q, q, q, o, cols, B=1, H=1, S=3, D=2)), off
    o = np.array([0, 1, 3, 4], np.int32).reshape(1, 1, -1)
    oracle.sparse_csr(q, q, q, o, cols, B=1, H=1, S=3, D=2)  # the same shapes, well formed


def pin_cumulative_lengths_rejected_when_bad():
    """Cumulative lengths (B entries, no leading zero) must not decrease and must end at the
    token count; anything else is refused, never computed."""
    x = np.zeros((10, 2, 4))
    args = dict(B=3, Sq=10, Skv=10, Nq=2, Nkv=2, D=4, scale=1.0, mask_mode=W.MASK_NONE, layout=W.TND)
    for cq, ck in (([6, 4, 10], [3, 6, 10]), ([3, 6, 10], [3, 6, 8]), ([3, 6, 9], [3, 6, 10])):
        assert _rejected(lambda: oracle.attn_fwd(x, x, x, cu_q=np.array(cq, np.int32),
                                                 cu_kv=np.array(ck, np.int32), **args)), (cq, ck)
    oracle.attn_fwd(x, x, x, cu_q=np.array([3, 6, 10], np.int32), cu_kv=np.array([2, 2, 10], np.int32),
                    **args)  # well formed, an empty key sequence included


# ---------------------------------------------------------------------------------------------
# Dense / varlen forward
# ---------------------------------------------------------------------------------------------
def pin_dense_matches_torch_sdpa():
    r = _rng(10)
    for (B, H, Sq, Skv, D) in [(1, 1, 1, 1, 1), (2, 3, 7, 7, 5), (1, 2, 5, 13, 8), (2, 1, 17, 4, 3)]:
        q = r.standard_normal((B, H, Sq, D))
        k = r.standard_normal((B, H, Skv, D))
        v = r.standard_normal((B, H, Skv, D))
        out, _, _ = _bhsd(q, k, v, NONE)
        assert np.max(np.abs(out - _torch_sdpa(q, k, v))) <= 1e-12
        # a non-default scale (the forward takes the scale as an argument)
        out, _, _ = _bhsd(q, k, v, NONE, scale=0.37)
        assert np.max(np.abs(out - _torch_sdpa(q, k, v, scale=0.37))) <= 1e-12


def pin_causal_topleft_matches_torch():
    r = _rng(11)
    for (B, H, S, D) in [(1, 1, 6, 2), (2, 2, 9, 4)]:
        q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
        out, _, _ = _bhsd(q, k, v, TL)
        assert np.max(np.abs(out - _torch_sdpa(q, k, v, causal=True))) <= 1e-12
        # with Sq == Skv, bottom-right and top-left coincide
        out2, _, _ = _bhsd(q, k, v, BR)
        assert np.array_equal(out, out2)


def pin_causal_rectangular_masks():
    r = _rng(12)
    B, H, D = 1, 2, 3
    for Sq, Skv in [(4, 9), (9, 4)]:
        q = r.standard_normal((B, H, Sq, D))
        k = r.standard_normal((B, H, Skv, D))
        v = r.standard_normal((B, H, Skv, D))
        i = np.arange(Sq)[:, None]
        j = np.arange(Skv)[None, :]
        for mode, vis in [(TL, j <= i), (BR, j <= i + Skv - Sq)]:
            out, m, l = _bhsd(q, k, v, mode)
            rows = vis.any(axis=1)
            if rows.any():
                ref = _torch_sdpa(q[:, :, rows], k, v, mask=np.broadcast_to(vis[rows], (B, H, rows.sum(), Skv)).copy())
                assert np.max(np.abs(out[:, :, rows] - ref)) <= 1e-12
            # rows with no visible key: out 0, max -inf, sum 0
            assert np.all(out[:, :, ~rows] == 0.0)
            assert np.all(np.isneginf(m[:, :, ~rows])) and np.all(l[:, :, ~rows] == 0.0)


def pin_gqa_mqa_match_torch():
    r = _rng(13)
    for Nq, Nkv in [(4, 2), (6, 1), (8, 4)]:
        B, S, D = 2, 7, 4
        q = r.standard_normal((B, Nq, S, D))
        k = r.standard_normal((B, Nkv, S, D))
        v = r.standard_normal((B, Nkv, S, D))
        for mode, causal in [(NONE, False), (TL, True)]:
            out, _, _ = _bhsd(q, k, v, mode)
            ref = _torch_sdpa(q, k, v, causal=causal, gqa=True)
            assert np.max(np.abs(out - ref)) <= 1e-12


def pin_stats_logsumexp():
    """max + ln(sum) is the log-sum-exp of the scaled, masked scores (torch.logsumexp)."""
    r = _rng(14)
    B, H, S, D = 2, 2, 8, 4
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    for mode in (NONE, TL):
        _, m, l = _bhsd(q, k, v, mode)
        sc = torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / math.sqrt(D)
        if mode == TL:
            sc = sc.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
        lse = torch.logsumexp(sc, dim=-1).numpy()
        mx = sc.max(dim=-1).values.numpy()
        assert np.max(np.abs(m - mx)) <= 1e-13
        assert np.max(np.abs(m + np.log(l) - lse)) <= 1e-12
        assert np.all(l >= 1.0)


def pin_closed_forms():
    r = _rng(15)
    B, H, S, D = 1, 2, 6, 3
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    # causal row 0 sees only key 0: o = v_0, sum = 1, max = scale * q0.k0
    out, m, l = _bhsd(q, k, v, TL)
    assert np.array_equal(out[:, :, 0], v[:, :, 0])
    assert np.all(l[:, :, 0] == 1.0)
    assert np.max(np.abs(m[:, :, 0] - np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]) / math.sqrt(D))) <= 1e-15
    # Q = 0: every score is 0, o = mean of the visible V rows, max 0, sum = #visible
    z = np.zeros_like(q)
    out, m, l = _bhsd(z, k, v, TL)
    for i in range(S):
        assert np.max(np.abs(out[:, :, i] - v[:, :, : i + 1].mean(axis=2))) <= 1e-15
    assert np.all(m == 0.0) and np.array_equal(l[0, 0], np.arange(1, S + 1, dtype=float))
    # V = 1: softmax rows sum to one
    out, _, _ = _bhsd(q, k, np.ones_like(v), NONE)
    assert np.max(np.abs(out - 1.0)) <= 1e-14


def pin_key_shift_invariance():
    """k_j -> k_j + u shifts row i's scores by scale*q_i.u: out and sum unchanged, max shifted."""
    r = _rng(16)
    B, H, S, D = 1, 2, 7, 5
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    u = r.standard_normal(D)
    o1, m1, l1 = _bhsd(q, k, v, NONE)
    o2, m2, l2 = _bhsd(q, k + u, v, NONE)
    assert np.max(np.abs(o1 - o2)) <= 1e-12
    assert np.max(np.abs(l1 - l2)) <= 1e-12
    assert np.max(np.abs(m2 - m1 - (q @ u) / math.sqrt(D))) <= 1e-12


def _slice_bhsd(x_tnd, lo, hi):
    """[T, N, D] rows lo..hi -> [1, N, hi-lo, D]."""
    return np.ascontiguousarray(np.transpose(x_tnd[lo:hi], (1, 0, 2))[None])


def pin_cumulative_lengths_example():
    g = load_golden("ascend_cumulative_seqlen_example.txt")
    lens = g["lengths"].astype(np.int64)
    cu = W.cu_seqlens_from_lengths(lens)
    assert np.array_equal(cu, g["cumulative"].astype(np.int32))
    assert np.array_equal(W.lengths_from_cu_seqlens(cu), lens)
    # the oracle decodes the same array into the same sequences
    r = _rng(20)
    T, Nq, Nkv, D = int(cu[-1]), 2, 1, 3
    q = r.standard_normal((T, Nq, D))
    k = r.standard_normal((T, Nkv, D))
    v = r.standard_normal((T, Nkv, D))
    out, _, _ = oracle.attn_fwd(q, k, v, cu_q=cu, cu_kv=cu, B=len(cu), Sq=T, Skv=T, Nq=Nq, Nkv=Nkv,
                                D=D, scale=0.5, mask_mode=NONE, layout=TND)
    starts = np.concatenate([[0], cu[:-1]])
    for lo, hi in zip(starts, cu):
        if hi == lo:
            continue
        ref = _torch_sdpa(_slice_bhsd(q, lo, hi), _slice_bhsd(k, lo, hi), _slice_bhsd(v, lo, hi),
                          scale=0.5, gqa=True)
        assert np.max(np.abs(np.transpose(ref[0], (1, 0, 2)) - out[lo:hi])) <= 1e-12


def pin_varlen_equals_per_sequence_dense():
    r = _rng(21)
    for lens in ([0, 5, 3], [4, 0, 0, 6], [7, 2, 0], [1, 1, 9]):
        for mode in (NONE, TL, BR):
            lens_q = np.array(lens)
            lens_k = np.array(lens) + (np.array(lens) > 0) * 2 if mode == BR else np.array(lens)
            cq, ck = W.cu_seqlens_from_lengths(lens_q), W.cu_seqlens_from_lengths(lens_k)
            Tq, Tk, Nq, Nkv, D = int(cq[-1]), int(ck[-1]), 4, 2, 3
            q = r.standard_normal((Tq, Nq, D))
            k = r.standard_normal((Tk, Nkv, D))
            v = r.standard_normal((Tk, Nkv, D))
            out, m, l = oracle.attn_fwd(q, k, v, cu_q=cq, cu_kv=ck, B=len(lens), Sq=Tq, Skv=Tk,
                                        Nq=Nq, Nkv=Nkv, D=D, scale=1 / math.sqrt(D), mask_mode=mode,
                                        layout=TND)
            sq0 = np.concatenate([[0], cq[:-1]])
            sk0 = np.concatenate([[0], ck[:-1]])
            for b in range(len(lens)):
                if lens_q[b] == 0:
                    continue
                qs = _slice_bhsd(q, sq0[b], cq[b])
                ks, vs = _slice_bhsd(k, sk0[b], ck[b]), _slice_bhsd(v, sk0[b], ck[b])
                Sq, Skv = qs.shape[2], ks.shape[2]
                i, j = np.arange(Sq)[:, None], np.arange(Skv)[None, :]
                vis = {NONE: np.ones((Sq, Skv), bool), TL: j <= i, BR: j <= i + Skv - Sq}[mode]
                ref = _torch_sdpa(qs, ks, vs, mask=np.broadcast_to(vis, (1, Nq, Sq, Skv)).copy(), gqa=True)
                assert np.max(np.abs(np.transpose(ref[0], (1, 0, 2)) - out[sq0[b]:cq[b]])) <= 1e-12
                # statistics land at [token, head]
                sc = torch.from_numpy(qs) @ torch.from_numpy(np.repeat(ks, Nq // Nkv, axis=1)).transpose(-1, -2) / math.sqrt(D)
                sc = sc.masked_fill(~torch.from_numpy(vis), float("-inf"))
                mx = sc.max(dim=-1).values.numpy()[0].T
                assert np.max(np.abs(m[sq0[b]:cq[b]] - mx)) <= 1e-13


def pin_rows_api_matches_full():
    r = _rng(22)
    lens = np.array([3, 0, 6, 2])
    cu = W.cu_seqlens_from_lengths(lens)
    T, Nq, Nkv, D = int(cu[-1]), 4, 2, 5
    q, k, v = (r.standard_normal((T, n, D)) for n in (Nq, Nkv, Nkv))
    kw = dict(cu_q=cu, cu_kv=cu, B=len(lens), Sq=T, Skv=T, Nq=Nq, Nkv=Nkv, D=D, scale=0.3,
              mask_mode=TL, layout=TND)
    out, m, l = oracle.attn_fwd(q, k, v, **kw)
    rows_t = np.array([0, 2, 3, 8, 10, 9])
    rows_h = np.array([0, 3, 1, 2, 0, 1])
    o2, m2, l2 = oracle.attn_fwd_rows(q, k, v, rows_h, rows_t, **kw)
    assert np.array_equal(o2, out[rows_t, rows_h])
    assert np.array_equal(m2, m[rows_t, rows_h]) and np.array_equal(l2, l[rows_t, rows_h])


# ---------------------------------------------------------------------------------------------
# Masked forward: band limits, explicit mask, value head size
# ---------------------------------------------------------------------------------------------
BAND = oracle.MASK_BAND
BIG = 1 << 40


def _ext_bhsd(q, k, v, mode, pre=0, nxt=0, mask=None, bstride=0, rstride=0, scale=None):
    B, Nq, Sq, D = q.shape
    _, Nkv, Skv, Dv = v.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    return oracle.attn_fwd_ext(q, k, v, B=B, Sq=Sq, Skv=Skv, Nq=Nq, Nkv=Nkv, Dqk=D, Dv=Dv,
                               scale=scale, mask_mode=mode, pre_tokens=pre, next_tokens=nxt,
                               mask=mask, mask_bstride=bstride, mask_rstride=rstride, layout=BHSD)


def _check_against_torch(out, m, l, q, k, v, vis, gqa=False):
    """vis: bool [B, Sq, Skv] (True = attend). Rows with a visible key match torch's float64
    SDPA with that boolean mask; rows without one give out 0, max -inf, sum 0."""
    B, Nq, Sq, _ = q.shape
    for b in range(B):
        rows = vis[b].any(axis=1)
        if rows.any():
            mk = np.broadcast_to(vis[b][rows], (1, Nq, int(rows.sum()), vis.shape[2])).copy()
            ref = _torch_sdpa(q[b:b + 1, :, rows], k[b:b + 1], v[b:b + 1], mask=mk, gqa=gqa)
            assert np.max(np.abs(out[b:b + 1, :, rows] - ref)) <= 1e-12
        assert np.all(out[b, :, ~rows] == 0.0)
        assert np.all(np.isneginf(m[b, :, ~rows])) and np.all(l[b, :, ~rows] == 0.0)


def pin_band_matches_torch_mask():
    """Band reading: key j visible to row i iff i - pre <= j <= i + next."""
    r = _rng(30)
    for (Sq, Skv) in [(9, 9), (6, 11), (11, 6)]:
        B, Nq, Nkv, D = 2, 4, 2, 3
        q = r.standard_normal((B, Nq, Sq, D))
        k = r.standard_normal((B, Nkv, Skv, D))
        v = r.standard_normal((B, Nkv, Skv, D))
        i, j = np.arange(Sq)[:, None], np.arange(Skv)[None, :]
        for pre, nxt in [(2, 1), (0, 0), (3, -1), (-1, 3), (0, 5), (100, 100), (-4, 4)]:
            out, m, l = _ext_bhsd(q, k, v, BAND, pre, nxt)
            vis = np.broadcast_to((j >= i - pre) & (j <= i + nxt), (B, Sq, Skv))
            _check_against_torch(out, m, l, q, k, v, vis, gqa=True)


def pin_band_limits_and_diagonal():
    r = _rng(31)
    B, H, S, D = 2, 2, 8, 3
    q, k, v = (r.standard_normal((B, H, S, D)) for _ in range(3))
    # an unbounded band is the full attention; no look-ahead with unbounded look-back is causal
    o_full, m_full, l_full = _bhsd(q, k, v, NONE)
    o_b, m_b, l_b = _ext_bhsd(q, k, v, BAND, BIG, BIG)
    assert np.max(np.abs(o_b - o_full)) <= 1e-14 and np.max(np.abs(l_b - l_full)) <= 1e-13
    o_c, _, _ = _bhsd(q, k, v, TL)
    o_b, _, _ = _ext_bhsd(q, k, v, BAND, BIG, 0)
    assert np.max(np.abs(o_b - o_c)) <= 1e-14
    # a band of width one: each row sees only its own key, o = v_i, sum = 1, max = scale q_i.k_i
    o, m, l = _ext_bhsd(q, k, v, BAND, 0, 0)
    assert np.array_equal(o, v) and np.all(l == 1.0)
    assert np.max(np.abs(m - np.einsum("bhsd,bhsd->bhs", q, k) / math.sqrt(D))) <= 1e-15


def pin_explicit_mask_matches_torch():
    """uint8 mask, 1 = excluded, element (b, i, j) at b*bstride + i*rstride + j; combined
    with the mode by AND."""
    r = _rng(32)
    B, Nq, Nkv, Sq, Skv, D = 3, 2, 1, 7, 10, 4
    q = r.standard_normal((B, Nq, Sq, D))
    k = r.standard_normal((B, Nkv, Skv, D))
    v = r.standard_normal((B, Nkv, Skv, D))
    rs = Skv + 3                                   # padded rows
    bs = Sq * rs + 5                               # padded batches
    flat = (r.random(B * bs) < 0.35).astype(np.uint8)
    flat[1 * bs + 2 * rs: 1 * bs + 2 * rs + Skv] = 1   # batch 1, row 2 fully excluded
    excl = np.stack([flat[b * bs: b * bs + Sq * rs].reshape(Sq, rs)[:, :Skv] for b in range(B)])
    i, j = np.arange(Sq)[:, None], np.arange(Skv)[None, :]
    for mode, base in [(NONE, np.ones((Sq, Skv), bool)), (TL, j <= i), (BR, j <= i + Skv - Sq),
                       (BAND, (j >= i - 1) & (j <= i + 2))]:
        out, m, l = _ext_bhsd(q, k, v, mode, 1, 2, mask=flat, bstride=bs, rstride=rs)
        _check_against_torch(out, m, l, q, k, v, (excl == 0) & base[None], gqa=True)
    # stride 0 across batches: one mask shared by every batch
    out, m, l = _ext_bhsd(q, k, v, NONE, mask=flat, bstride=0, rstride=rs)
    _check_against_torch(out, m, l, q, k, v, np.broadcast_to(excl[0] == 0, (B, Sq, Skv)), gqa=True)


def pin_value_head_size():
    """qD == kD >= vD: the scores use D = Dqk, the output has Dv columns (torch SDPA allows a
    value head size of its own)."""
    r = _rng(33)
    B, H, Sq, Skv, D = 2, 3, 6, 9, 8
    for Dv in (1, 3, 8):
        q = r.standard_normal((B, H, Sq, D))
        k = r.standard_normal((B, H, Skv, D))
        v = r.standard_normal((B, H, Skv, Dv))
        out, _, _ = _ext_bhsd(q, k, v, NONE)
        assert out.shape == (B, H, Sq, Dv)
        assert np.max(np.abs(out - _torch_sdpa(q, k, v))) <= 1e-12
        i, j = np.arange(Sq)[:, None], np.arange(Skv)[None, :]
        out, m, l = _ext_bhsd(q, k, v, BR)
        _check_against_torch(out, m, l, q, k, v, np.broadcast_to(j <= i + Skv - Sq, (B, Sq, Skv)))


def pin_ext_varlen_per_sequence():
    """TND with a band and a per-sequence mask equals torch on each sequence's slice; the mask
    is indexed by in-sequence positions with one batch stride per sequence."""
    r = _rng(34)
    lens_q = np.array([5, 0, 7, 3])
    lens_k = np.array([6, 4, 7, 0])
    cq, ck = W.cu_seqlens_from_lengths(lens_q), W.cu_seqlens_from_lengths(lens_k)
    Tq, Tk, Nq, Nkv, D, Dv = int(cq[-1]), int(ck[-1]), 4, 2, 3, 2
    q = r.standard_normal((Tq, Nq, D))
    k = r.standard_normal((Tk, Nkv, D))
    v = r.standard_normal((Tk, Nkv, Dv))
    rs, bs = 8, 8 * 8
    flat = (r.random(len(lens_q) * bs) < 0.3).astype(np.uint8)
    pre, nxt = 2, 1
    out, m, l = oracle.attn_fwd_ext(q, k, v, cu_q=cq, cu_kv=ck, B=len(lens_q), Sq=Tq, Skv=Tk,
                                    Nq=Nq, Nkv=Nkv, Dqk=D, Dv=Dv, scale=0.4, mask_mode=BAND,
                                    pre_tokens=pre, next_tokens=nxt, mask=flat, mask_bstride=bs,
                                    mask_rstride=rs, layout=TND)
    sq0 = np.concatenate([[0], cq[:-1]])
    sk0 = np.concatenate([[0], ck[:-1]])
    for b in range(len(lens_q)):
        Sq, Skv = int(lens_q[b]), int(lens_k[b])
        if Sq == 0:
            continue
        i, j = np.arange(Sq)[:, None], np.arange(Skv)[None, :]
        excl = flat[b * bs: b * bs + Sq * rs].reshape(Sq, rs)[:, :Skv]
        vis = ((j >= i - pre) & (j <= i + nxt) & (excl == 0))[None]
        qs = _slice_bhsd(q, sq0[b], cq[b])
        ks, vs = _slice_bhsd(k, sk0[b], ck[b]), _slice_bhsd(v, sk0[b], ck[b])
        o_b = np.transpose(out[sq0[b]:cq[b]], (1, 0, 2))[None]
        m_b = m[sq0[b]:cq[b]].T[None]
        l_b = l[sq0[b]:cq[b]].T[None]
        if Skv == 0:
            assert np.all(o_b == 0.0) and np.all(np.isneginf(m_b)) and np.all(l_b == 0.0)
            continue
        def sd(qq, kk, vv, mask=None, gqa=False):
            return F.scaled_dot_product_attention(
                torch.from_numpy(qq), torch.from_numpy(kk), torch.from_numpy(vv),
                attn_mask=None if mask is None else torch.from_numpy(mask), scale=0.4,
                enable_gqa=gqa).numpy()
        rows = vis[0].any(axis=1)
        if rows.any():
            mk = np.broadcast_to(vis[0][rows], (1, Nq, int(rows.sum()), Skv)).copy()
            ref = sd(qs[:, :, rows], ks, vs, mask=mk, gqa=True)
            assert np.max(np.abs(o_b[:, :, rows] - ref)) <= 1e-12
        assert np.all(o_b[:, :, ~rows] == 0.0) and np.all(l_b[:, :, ~rows] == 0.0)


def pin_ext_rows_and_rejections():
    r = _rng(35)
    B, Nq, Nkv, S, D, Dv = 2, 4, 2, 9, 4, 2
    q = r.standard_normal((B, Nq, S, D))
    k = r.standard_normal((B, Nkv, S, D))
    v = r.standard_normal((B, Nkv, S, Dv))
    mask = (r.random(S * S) < 0.2).astype(np.uint8)
    kw = dict(B=B, Sq=S, Skv=S, Nq=Nq, Nkv=Nkv, Dqk=D, Dv=Dv, scale=0.3, mask_mode=BAND,
              pre_tokens=3, next_tokens=2, mask=mask, mask_bstride=0, mask_rstride=S, layout=BHSD)
    out, m, l = oracle.attn_fwd_ext(q, k, v, **kw)
    rows_t = np.array([0, 5, 9, 17, 12])
    rows_h = np.array([1, 0, 3, 2, 2])
    o2, m2, l2 = oracle.attn_fwd_ext_rows(q, k, v, rows_h, rows_t, **kw)
    b, i = rows_t // S, rows_t % S
    assert np.array_equal(o2, out[b, rows_h, i])
    assert np.array_equal(m2, m[b, rows_h, i]) and np.array_equal(l2, l[b, rows_h, i])
    for bad in (dict(pre_tokens=-3, next_tokens=2), dict(Dv=D + 1), dict(mask_mode=4)):
        try:
            oracle.attn_fwd_ext(q, k, v, **{**kw, **bad})
        except ValueError:
            continue
        raise AssertionError(f"accepted {bad}")


# ---------------------------------------------------------------------------------------------
# Merge (ring-attention update)
# ---------------------------------------------------------------------------------------------
def _to_sbh(o_bnsd):
    """[B, N, S, D] -> [S, B, N*D]."""
    B, N, S, D = o_bnsd.shape
    return np.ascontiguousarray(np.transpose(o_bnsd, (2, 0, 1, 3)).reshape(S, B, N * D))


def _rep8(x_bns):
    return np.ascontiguousarray(np.repeat(x_bns[..., None], 8, axis=-1))


def pin_merge_chunks_equal_full():
    """Attention over 4 key chunks merged one after another equals attention over all keys."""
    r = _rng(30)
    B, N, S, Skv, D = 2, 3, 5, 16, 4
    q = r.standard_normal((B, N, S, D))
    k = r.standard_normal((B, N, Skv, D)) * 2.0
    v = r.standard_normal((B, N, Skv, D))
    full, fm, fl = _bhsd(q, k, v, NONE)
    acc = None
    for c in range(4):
        sl = slice(4 * c, 4 * c + 4)
        o, m, l = _bhsd(q, np.ascontiguousarray(k[:, :, sl]), np.ascontiguousarray(v[:, :, sl]), NONE)
        part = (_to_sbh(o), _rep8(m), _rep8(l))
        if acc is None:
            acc = part
        else:
            acc = oracle.merge(acc[0], acc[1], acc[2], *part, S=S, B=B, N=N, D=D)
    assert np.max(np.abs(acc[0] - _to_sbh(full))) <= 1e-12
    assert np.max(np.abs(acc[1] - _rep8(fm))) <= 1e-13
    assert np.max(np.abs(acc[2] / _rep8(fl) - 1.0)) <= 1e-12


def pin_merge_self_and_empty():
    r = _rng(31)
    S, B, N, D = 4, 2, 3, 5
    o = r.standard_normal((S, B, N * D))
    m = _rep8(r.standard_normal((B, N, S)))
    l = _rep8(1.0 + np.abs(r.standard_normal((B, N, S))))
    out, om, ol = oracle.merge(o, m, l, o, m, l, S=S, B=B, N=N, D=D)
    assert np.max(np.abs(out - o)) <= 1e-15 and np.array_equal(om, m)
    assert np.max(np.abs(ol - 2 * l)) <= 1e-14
    ninf = np.full_like(m, -np.inf)
    zero = np.zeros_like(l)
    for args in [(o, m, l, np.zeros_like(o), ninf, zero), (np.zeros_like(o), ninf, zero, o, m, l)]:
        out, om, ol = oracle.merge(*args, S=S, B=B, N=N, D=D)
        assert np.array_equal(out, o) and np.array_equal(om, m) and np.array_equal(ol, l)
    # both sides empty: out 0, max -inf, sum 0 (no NaN)
    out, om, ol = oracle.merge(o, ninf, zero, o, ninf, zero, S=S, B=B, N=N, D=D)
    assert np.all(out == 0.0) and np.all(np.isneginf(om)) and np.all(ol == 0.0)


def pin_merge_lanes():
    """Statistics merge lane by lane; the output uses lane 0 only."""
    r = _rng(32)
    S, B, N, D = 3, 1, 2, 4
    po, co = r.standard_normal((S, B, N * D)), r.standard_normal((S, B, N * D))
    pm, cm = r.standard_normal((B, N, S, 8)), r.standard_normal((B, N, S, 8))
    ps, cs = 1 + np.abs(r.standard_normal((B, N, S, 8))), 1 + np.abs(r.standard_normal((B, N, S, 8)))
    out, om, ol = oracle.merge(po, pm, ps, co, cm, cs, S=S, B=B, N=N, D=D)
    for lane in range(8):
        sel = lambda x: _rep8(x[..., lane])
        o2, m2, l2 = oracle.merge(po, sel(pm), sel(ps), co, sel(cm), sel(cs), S=S, B=B, N=N, D=D)
        assert np.array_equal(om[..., lane], m2[..., 0]) and np.array_equal(ol[..., lane], l2[..., 0])
        if lane == 0:
            assert np.array_equal(out, o2)


def pin_merge_order_independent():
    r = _rng(33)
    S, B, N, D = 3, 2, 2, 3
    parts = []
    for _ in range(3):
        parts.append((r.standard_normal((S, B, N * D)), _rep8(r.standard_normal((B, N, S)) * 3),
                      _rep8(1 + np.abs(r.standard_normal((B, N, S))))))
    kw = dict(S=S, B=B, N=N, D=D)
    ab = oracle.merge(*parts[0], *parts[1], **kw)
    ba = oracle.merge(*parts[1], *parts[0], **kw)
    assert np.max(np.abs(ab[0] - ba[0])) <= 1e-14
    left = oracle.merge(*ab, *parts[2], **kw)
    right = oracle.merge(*parts[0], *oracle.merge(*parts[1], *parts[2], **kw), **kw)
    for x, y in zip(left, right):
        assert np.max(np.abs(x - y)) <= 1e-12


def pin_merge_tnd_matches_sbh_relayout():
    """The TND merge ([T, N*D] outputs, [T, N, 8] statistics) equals the SBH merge of the same
    rows laid out as B = 1 ([T, 1, N*D] outputs, [1, N, T, 8] statistics)."""
    r = _rng(34)
    T, N, D = 7, 3, 4
    po, co = r.standard_normal((T, N * D)), r.standard_normal((T, N * D))
    pm, cm = r.standard_normal((T, N, 8)), r.standard_normal((T, N, 8))
    ps, cs = 1 + np.abs(r.standard_normal((T, N, 8))), 1 + np.abs(r.standard_normal((T, N, 8)))
    tnd = oracle.merge(po, pm, ps, co, cm, cs, S=T, B=1, N=N, D=D, layout=TND)
    to_sbh = lambda x: np.ascontiguousarray(np.transpose(x, (1, 0, 2))[None])  # [T,N,8] -> [1,N,T,8]
    sbh = oracle.merge(po[:, None], to_sbh(pm), to_sbh(ps), co[:, None], to_sbh(cm), to_sbh(cs),
                       S=T, B=1, N=N, D=D, layout=BHSD)
    assert np.array_equal(tnd[0], sbh[0][:, 0])
    assert np.array_equal(tnd[1], np.transpose(sbh[1][0], (1, 0, 2)))
    assert np.array_equal(tnd[2], np.transpose(sbh[2][0], (1, 0, 2)))


def pin_merge_tnd_chunks_equal_full_varlen():
    """Varlen attention over two key chunks of every sequence, merged in TND layout, equals
    attention over all keys."""
    r = _rng(35)
    lens = np.array([5, 0, 9, 3])
    cu = W.cu_seqlens_from_lengths(lens)
    T, Nq, Nkv, D = int(cu[-1]), 4, 2, 3
    q = r.standard_normal((T, Nq, D))
    k = r.standard_normal((T, Nkv, D)) * 2
    v = r.standard_normal((T, Nkv, D))
    kw = dict(Nq=Nq, Nkv=Nkv, D=D, scale=0.4, mask_mode=NONE, layout=TND)
    full, fm, fl = oracle.attn_fwd(q, k, v, cu_q=cu, cu_kv=cu, B=len(lens), Sq=T, Skv=T, **kw)
    starts = np.concatenate([[0], cu[:-1]])
    parts = []
    for half in range(2):
        idx, lk = [], []
        for s0, L in zip(starts, lens):
            a, b = (0, L // 2) if half == 0 else (L // 2, L)
            idx.extend(range(s0 + a, s0 + b))
            lk.append(b - a)
        idx = np.array(idx, dtype=np.int64)
        ck = W.cu_seqlens_from_lengths(lk)
        o, m, l = oracle.attn_fwd(q, k[idx], v[idx], cu_q=cu, cu_kv=ck, B=len(lens), Sq=T,
                                  Skv=int(ck[-1]), **kw)
        parts.append((o.reshape(T, Nq * D), np.repeat(m[..., None], 8, -1), np.repeat(l[..., None], 8, -1)))
    out, om, ol = oracle.merge(*parts[0], *parts[1], S=T, B=0, N=Nq, D=D, layout=TND)
    assert np.max(np.abs(out - full.reshape(T, Nq * D))) <= 1e-12
    assert np.max(np.abs(om[..., 0] - fm)) <= 1e-13
    assert np.max(np.abs(ol[..., 0] / fl - 1)) <= 1e-12


# ---------------------------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------------------------
def pin_bf16_inputs_read_exactly():
    """bf16 inputs (passed to the oracle as raw 16-bit patterns) give bit-for-bit the results of
    the same values widened to float64 by torch, for the forward, the CSR call and the merge."""
    g = torch.Generator().manual_seed(77)
    B, N, S, D = 2, 3, 9, 8
    q, k, v = (torch.randn((B, N, S, D), generator=g).to(torch.bfloat16) for _ in range(3))
    args = dict(B=B, Sq=S, Skv=S, Nq=N, Nkv=N, D=D, scale=0.3, mask_mode=W.MASK_CAUSAL_TOPLEFT,
                layout=W.BHSD)
    a = oracle.attn_fwd(q, k, v, **args)
    b = oracle.attn_fwd(q.double(), k.double(), v.double(), **args)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    off = np.broadcast_to(np.arange(0, 2 * S + 1, 2, dtype=np.int32), (B, N, S + 1)).copy()
    cols = np.broadcast_to(((np.arange(2 * S) * 5) % S).astype(np.int32), (B, N, 2 * S)).copy()
    a = oracle.sparse_csr(q, k, v, off, cols, B=B, H=N, S=S, D=D)
    b = oracle.sparse_csr(q.double(), k.double(), v.double(), off, cols, B=B, H=N, S=S, D=D)
    assert np.array_equal(a, b)
    po, co = (torch.randn((S, B, N * D), generator=g).to(torch.bfloat16) for _ in range(2))
    m1, m2 = (_rep8(torch.randn((B, N, S), generator=g).double().numpy()) for _ in range(2))
    l1, l2 = (_rep8(1.0 + torch.rand((B, N, S), generator=g).double().numpy()) for _ in range(2))
    a = oracle.merge(po, m1, l1, co, m2, l2, S=S, B=B, N=N, D=D)
    b = oracle.merge(po.double(), m1, l1, co.double(), m2, l2, S=S, B=B, N=N, D=D)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))


def pin_round_bf16_matches_torch():
    r = _rng(40)
    x = np.concatenate([
        r.standard_normal(20000).astype(np.float32),
        (r.standard_normal(2000) * 1e-39).astype(np.float32),        # subnormals
        (r.standard_normal(2000) * 1e37).astype(np.float32),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0, 3.3895314e38, 3.4e38,
                  np.inf, -np.inf], dtype=np.float32),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def pin_round_f16_matches_numpy_and_torch():
    """float64 -> float16 in one rounding: numpy's cast rounds a double directly (torch's goes
    through float32, so it is compared on float32-representable values only)."""
    r = _rng(41)
    tie = 1 + 2 ** -11                                   # halfway between 1 and 1 + 2^-10
    x = np.concatenate([
        r.standard_normal(20000) * 3.0,
        r.standard_normal(2000) * 1e-6,                  # subnormal range (below 2^-14)
        r.standard_normal(2000) * 3e4,                   # near the largest finite value
        np.array([tie, tie + 2 ** -40, tie - 2 ** -40, 1 + 3 * 2 ** -11, -tie, 0.0, -0.0,
                  2 ** -25, 2 ** -25 + 2 ** -60, 3 * 2 ** -25, 2 ** -14 - 2 ** -26, 65504.0,
                  65519.99, 65520.0, -65520.0, 1e9, np.inf, -np.inf]),
    ])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.round_f16(x), want)
    x32 = r.standard_normal(20000).astype(np.float32) * np.float32(100.0)
    want32 = torch.from_numpy(x32).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.round_f16(x32.astype(np.float64)), want32)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
