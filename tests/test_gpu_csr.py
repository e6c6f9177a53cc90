"""attn_sparse_csr on the GPU against the float64 oracle (and the Paddle worked example)."""
import numpy as np
import pytest
import torch

import oracle
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G
from tests.golden.loader import load as load_golden

pytestmark = pytest.mark.gpu


def _run(q, k, v, off, cols, B, H, S, D):
    dq, dk, dv = (torch.as_tensor(x).float().cuda().contiguous() for x in (q, k, v))
    doff = torch.from_numpy(np.ascontiguousarray(off, np.int32)).cuda()
    dcol = torch.from_numpy(np.ascontiguousarray(cols, np.int32)).cuda()
    out = G.guarded_like(dq)  # NaN-filled: every element must be written
    sdpa.attn_sparse_csr(dq, dk, dv, doff, dcol, B=B, H=H, S=S, D=D, nnz_cap=cols.shape[-1], out=out.t)
    st = sdpa.attn_get_last_error()
    out.check("csr out")
    return out.t.cpu(), st


def test_paddle_worked_example():
    g = load_golden("paddle_sparse_attention_example.txt")
    shape = tuple(int(x) for x in g["shape"])
    q = g["query"].astype(np.float32).reshape(shape)
    off = g["offset"].astype(np.int32).reshape(1, 1, -1)
    col = g["columns"].astype(np.int32).reshape(1, 1, -1)
    out, st = _run(q, q, q, off, col, 1, 1, shape[2], shape[3])
    assert st == 0
    # the page prints float32 values to 8 decimals
    assert np.max(np.abs(out.numpy() - g["output"].reshape(shape))) <= 1e-6


def _random_pattern(rng, B, H, S, max_per_row, distinct=False):
    """Random row lengths on [0, max_per_row]; columns unsorted, with repeats unless distinct."""
    offs = np.zeros((B, H, S + 1), np.int32)
    rows = []
    for bh in range(B * H):
        cnt = rng.integers(0, max_per_row + 1, size=S)
        offs.reshape(B * H, S + 1)[bh, 1:] = np.cumsum(cnt)
        if distinct:
            rows.append(np.concatenate([rng.permutation(S)[:c] for c in cnt]))
        else:
            rows.append(rng.integers(0, S, size=int(cnt.sum())))
    cap = max(1, max(len(r) for r in rows))
    cols = np.zeros((B, H, cap), np.int32)
    for bh, r in enumerate(rows):
        cols.reshape(B * H, cap)[bh, :len(r)] = r
    return offs, cols


@pytest.mark.parametrize("D", [64, 1, 13, 40, 128, 256])
def test_random_patterns(D):
    rng = np.random.default_rng(D)
    B, H, S = 2, 3, 97
    q, k, v = (W.randn((B, H, S, D), 100 + i) for i in range(3))
    off, cols = _random_pattern(rng, B, H, S, 40)
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(out.numpy(), ref, W.F32, "csr out")


def test_cfg4_full_size():
    """Configuration 4 at full size: B=2, H=8, S=4096, D=64, window 256 + every 64th column."""
    inp = W.cfg4_csr(seed=0)
    out, st = _run(inp.q, inp.k, inp.v, inp.offset, inp.columns, inp.B, inp.H, inp.S, inp.D)
    assert st == 0
    ref = oracle.sparse_csr(inp.q, inp.k, inp.v, inp.offset, inp.columns, B=inp.B, H=inp.H,
                            S=inp.S, D=inp.D)
    G.check_out(out.numpy(), ref, W.F32, "cfg4 out")


def test_full_pattern_equals_dense_attention():
    B, H, S, D = 1, 2, 150, 64
    q, k, v = (W.randn((B, H, S, D), 200 + i) for i in range(3))
    cols = np.broadcast_to(np.tile(np.arange(S, dtype=np.int32), S), (B, H, S * S)).copy()
    off = np.broadcast_to(np.arange(0, S * S + 1, S, dtype=np.int32), (B, H, S + 1)).copy()
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    inp = W.AttnInputs(q, k, v, W.BHSD, W.MASK_NONE, W.F32, B, S, S, H, H, D, 1.0 / np.sqrt(D))
    dense, _, _ = G.run_fwd(inp)
    assert np.max(np.abs(out.numpy() - dense.numpy())) <= 2e-6


def test_bad_columns_report_data_error():
    B, H, S, D = 1, 1, 8, 64
    q = W.randn((B, H, S, D), 1)
    off = np.arange(S + 1, dtype=np.int32).reshape(1, 1, -1)
    cols = np.arange(S, dtype=np.int32).reshape(1, 1, -1)
    cols[0, 0, 3] = S  # out of range
    out, st = _run(q, q, q, off, cols, B, H, S, D)
    assert st == sdpa.ATTN_ERR_DATA
    assert torch.all(out[0, 0, 3] == 0)  # the offending row is written as zeros
    assert torch.allclose(out[0, 0, 2], q[0, 0, 2])  # single-entry rows are v_j
    off2 = off.copy()
    off2[0, 0, 5] = 2  # decreasing row pointer
    cols[0, 0, 3] = 3
    out, st = _run(q, q, q, off2, cols, B, H, S, D)
    assert st == sdpa.ATTN_ERR_DATA


# ---- the tiled path (D = 64 or 128, 16-byte aligned tensors) and the row-per-warp path ---------
def test_repeated_columns_count_per_entry_tiled():
    """A column stored c times in a row weighs c times (reading of the row pointer), including
    a column stored 300 times; such rows take the tiled kernel's exact row-per-warp pass."""
    B, H, S, D = 1, 2, 200, 64
    q, k, v = (W.randn((B, H, S, D), 400 + i) for i in range(3))
    rng = np.random.default_rng(3)
    rows = []
    for i in range(S):
        base = rng.integers(0, S, size=int(rng.integers(0, 12)))
        if i % 7 == 0:
            base = np.concatenate([base, np.full(3, i)])      # a few repeats
        if i == 100:
            base = np.concatenate([base, np.full(300, 5)])    # 300 copies of one column
        rows.append(base.astype(np.int32))
    cnt = np.array([len(r) for r in rows])
    off1 = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    col1 = np.concatenate(rows).astype(np.int32)
    off = np.broadcast_to(off1, (B, H, S + 1)).copy()
    cols = np.broadcast_to(col1, (B, H, col1.size)).copy()
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(out.numpy(), ref, W.F32, "repeats")


@pytest.mark.parametrize("D", [64, 128])
def test_union_wider_than_one_window_tiled(D):
    """Rows of up to 150 random columns (with repeats) over 2,560 keys: each 128-row block's
    union spans about 2,500 columns, so the per-row marks are rebuilt window after window."""
    rng = np.random.default_rng(D)
    B, H, S = 1, 2, 2560
    q, k, v = (W.randn((B, H, S, D), 500 + i) for i in range(3))
    off, cols = _random_pattern(rng, B, H, S, 150)
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(out.numpy(), ref, W.F32, "wide union")


@pytest.mark.parametrize("D", [64, 128])
def test_distinct_columns_across_windows_tiled(D):
    """Rows of up to 200 distinct unsorted columns over 3,000 keys: no row needs the exact pass,
    every block's union spans six 512-column windows, and the last block and tile are ragged."""
    rng = np.random.default_rng(700 + D)
    B, H, S = 1, 2, 3000
    q, k, v = (W.randn((B, H, S, D), 700 + i) for i in range(3))
    off, cols = _random_pattern(rng, B, H, S, 200, distinct=True)
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(out.numpy(), ref, W.F32, "distinct, six windows")


@pytest.mark.parametrize("U", [511, 512, 513, 544])
def test_union_at_the_window_edge_tiled(U):
    """Every row stores the same U distinct columns (reversed), so each block's union is exactly
    U columns: one window short of, at, and just past 512 union columns."""
    B, H, S, D = 1, 1, 1100, 64
    q, k, v = (W.randn((B, H, S, D), 800 + i) for i in range(3))
    row = (np.arange(U, dtype=np.int64) * 2 + 1)[::-1]  # U distinct odd columns, all below S
    assert np.unique(row).size == U
    off = (np.arange(S + 1, dtype=np.int64) * U).astype(np.int32).reshape(1, 1, -1)
    cols = np.tile(row.astype(np.int32), S).reshape(1, 1, -1)
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(out.numpy(), ref, W.F32, f"union of {U}")


def _sparse_distinct_pattern(rng, S, max_per_row):
    """One (b, h) slice: row lengths on [0, max_per_row], distinct random columns per row
    (drawn with replacement, rows holding a repeat drawn again)."""
    cnt = rng.integers(0, max_per_row + 1, size=S)
    rows = []
    for c in cnt:
        r = rng.integers(0, S, size=c)
        while np.unique(r).size != c:
            r = rng.integers(0, S, size=c)
        rows.append(r)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32).reshape(1, 1, -1)
    cols = np.concatenate(rows).astype(np.int32).reshape(1, 1, -1)
    return off, cols


@pytest.mark.parametrize("S,D", [(32768, 64), (32767, 64), (32768, 128)])
def test_longest_sequence_tiled(S, D):
    """S at the tiled kernel's limit of 32,768 keys: the union's byte per column fills the 32 KB
    it borrows from the K/V buffers and the bitmap holds 1,024 words; rows of up to 12 distinct
    random columns, so each block's union (650 to 870 columns) spans two 512-column windows."""
    rng = np.random.default_rng(S + D)
    B, H = 1, 1
    q, k, v = (W.randn((B, H, S, D), 900 + i) for i in range(3))
    off, cols = _sparse_distinct_pattern(rng, S, 12)
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(out.numpy(), ref, W.F32, f"S={S}")


def test_row_per_warp_path_on_misaligned_tensors():
    """A q view that starts 4 bytes into its buffer is not 16-byte aligned, so the call takes the
    row-per-warp kernel; both paths agree with the oracle on the same data."""
    B, H, S, D = 1, 2, 130, 64
    rng = np.random.default_rng(11)
    q, k, v = (W.randn((B, H, S, D), 600 + i) for i in range(3))
    off, cols = _random_pattern(rng, B, H, S, 30)
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    buf = torch.zeros(B * H * S * D + 1, device="cuda")
    dq = buf[1:].view(B, H, S, D)
    dq.copy_(q.cuda())
    dk, dv = k.cuda(), v.cuda()
    out = G.guarded_like(dk)
    sdpa.attn_sparse_csr(dq, dk, dv, torch.from_numpy(off).cuda(), torch.from_numpy(cols).cuda(),
                         B=B, H=H, S=S, D=D, nnz_cap=cols.shape[-1], out=out.t)
    assert sdpa.attn_get_last_error() == 0
    out.check("row-per-warp out")
    G.check_out(out.t.cpu().numpy(), ref, W.F32, "row-per-warp path")
    out2, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    G.check_out(out2.numpy(), ref, W.F32, "tiled path")
