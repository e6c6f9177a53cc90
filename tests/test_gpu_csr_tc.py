"""attn_sparse_csr_tc (bf16 / fp16 on the tensor cores) on the GPU against the float64 oracle.

The oracle takes the same 16-bit input values, widened exactly; the output is compared with
the bf16/fp16 tolerance of the other parity tests."""
import numpy as np
import pytest
import torch

import oracle
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

BF, F16 = torch.bfloat16, torch.float16


def _run(q, k, v, off, cols, B, H, S, D):
    dq, dk, dv = (torch.as_tensor(x).cuda().contiguous() for x in (q, k, v))
    doff = torch.from_numpy(np.ascontiguousarray(off, np.int32)).cuda()
    dcol = torch.from_numpy(np.ascontiguousarray(cols, np.int32)).cuda()
    out = G.guarded_like(dq)  # NaN-filled: every element must be written
    sdpa.attn_sparse_csr_tc(dq, dk, dv, doff, dcol, B=B, H=H, S=S, D=D, nnz_cap=cols.shape[-1],
                            dtype=W.dtype_code(dq.dtype), out=out.t)
    st = sdpa.attn_get_last_error()
    out.check("csr_tc out")
    return out.t.cpu(), st


def _inputs(B, H, S, D, dtype, seed):
    return [W.randn((B, H, S, D), 300 + 7 * seed + i).to(dtype) for i in range(3)]


def _distinct_pattern(rng, B, H, S, max_per_row, empty_every=0):
    """Random rows of distinct, unsorted columns; every empty_every-th row empty."""
    offs = np.zeros((B * H, S + 1), np.int32)
    rows = []
    for bh in range(B * H):
        cnt = rng.integers(0, max_per_row + 1, size=S)
        if empty_every:
            cnt[::empty_every] = 0
        offs[bh, 1:] = np.cumsum(cnt)
        rows.append(np.concatenate([rng.permutation(S)[:c] for c in cnt]) if cnt.sum() else np.zeros(0, int))
    cap = max(1, max(len(r) for r in rows))
    cols = np.zeros((B * H, cap), np.int32)
    for bh, r in enumerate(rows):
        cols[bh, :len(r)] = r
    return offs.reshape(B, H, S + 1), cols.reshape(B, H, cap)


def _abs_ref(q, k, v, off, cols, B, H, S, D):
    """A = sum_j w_j |v_j| per output element (the oracle on |V|), for the rule where |exact| >= 4."""
    return lambda: oracle.sparse_csr(q, k, v.abs(), off, cols, B=B, H=H, S=S, D=D)


def _check(q, k, v, off, cols, B, H, S, D):
    out, st = _run(q, k, v, off, cols, B, H, S, D)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(G.f64(out), ref, W.dtype_code(q.dtype), "csr_tc out",
                abs_ref=_abs_ref(q, k, v, off, cols, B, H, S, D))


@pytest.mark.parametrize("dtype", [BF, F16], ids=["bf16", "f16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [300, 640])
def test_window_stride_pattern(dtype, D, S):
    offs, c = W.window_stride_pattern(S)
    B, H = 1, 2
    off = np.broadcast_to(offs, (B, H, S + 1)).copy()
    cols = np.broadcast_to(c, (B, H, c.shape[0])).copy()
    _check(*_inputs(B, H, S, D, dtype, S + D), off, cols, B, H, S, D)


@pytest.mark.parametrize("dtype", [BF, F16], ids=["bf16", "f16"])
@pytest.mark.parametrize("D", [64, 128])
def test_random_patterns(dtype, D):
    rng = np.random.default_rng(D)
    B, H, S = 2, 3, 333
    off, cols = _distinct_pattern(rng, B, H, S, 60, empty_every=7)
    _check(*_inputs(B, H, S, D, dtype, D), off, cols, B, H, S, D)


def test_union_wider_than_one_pass():
    """Rows of 150 random columns over 2,560 keys: each 128-row block's union spans about 2,000
    columns, so the per-row masks are rebuilt window after window (256 union columns each)."""
    rng = np.random.default_rng(5)
    B, H, S, D = 1, 2, 2560, 64
    off, cols = _distinct_pattern(rng, B, H, S, 150)
    _check(*_inputs(B, H, S, D, BF, 5), off, cols, B, H, S, D)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("aligned", [True, False], ids=["cols16", "cols_unaligned"])
def test_narrow_union_marked_in_one_pass(D, aligned):
    """A +-24 window plus every 100th column: each block's union (about 180 columns) fits one
    mark window at both head sizes. The union is taken with 16-byte loads of the column array
    or, from an array that starts 4 bytes off a 16-byte boundary, one index at a time. Some
    rows are empty and the last block is ragged."""
    B, H, S = 1, 2, 777
    offs, c = W.window_stride_pattern(S, half_window=24, stride=100)
    cnt = np.diff(offs)
    cnt[::11] = 0                                      # empty every 11th row
    keep = np.concatenate([np.arange(offs[i], offs[i + 1]) for i in range(S) if cnt[i]])
    offs = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    c = c[keep]
    off = np.broadcast_to(offs, (B, H, S + 1)).copy()
    cols = np.broadcast_to(c, (B, H, c.shape[0])).copy()
    q, k, v = _inputs(B, H, S, D, BF, 40 + D)
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    doff = torch.from_numpy(off).cuda()
    buf = torch.zeros(cols.size + 1, dtype=torch.int32, device="cuda")
    dcol = (buf[:-1] if aligned else buf[1:]).view(cols.shape)
    dcol.copy_(torch.from_numpy(cols))
    out = G.guarded_like(dq)
    sdpa.attn_sparse_csr_tc(dq, dk, dv, doff, dcol, B=B, H=H, S=S, D=D, nnz_cap=cols.shape[-1],
                            dtype=sdpa.ATTN_BF16, out=out.t)
    assert sdpa.attn_get_last_error() == 0
    out.check("csr_tc out")
    G.check_out(G.f64(out.t.cpu()), ref, W.BF16, "one-pass marks",
                abs_ref=_abs_ref(q, k, v, off, cols, B, H, S, D))


@pytest.mark.parametrize("S,D", [(32768, 64), (32767, 128)])
def test_longest_sequence(S, D):
    """S at the limit of 32,768 keys (a byte per column in shared memory while the union is
    taken); rows of up to 12 distinct random columns, several mark windows per block."""
    rng = np.random.default_rng(S + D)
    B, H = 1, 1
    cnt = rng.integers(0, 13, size=S)
    rows = []
    for c in cnt:
        r = rng.integers(0, S, size=c)
        while np.unique(r).size != c:
            r = rng.integers(0, S, size=c)
        rows.append(r)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32).reshape(1, 1, -1)
    cols = np.concatenate(rows).astype(np.int32).reshape(1, 1, -1)
    _check(*_inputs(B, H, S, D, BF, 60 + D), off, cols, B, H, S, D)


def test_full_pattern_equals_dense():
    B, H, S, D = 1, 2, 200, 128
    q, k, v = _inputs(B, H, S, D, BF, 9)
    cols = np.broadcast_to(np.tile(np.arange(S, dtype=np.int32), S), (B, H, S * S)).copy()
    off = np.broadcast_to(np.arange(0, S * S + 1, S, dtype=np.int32), (B, H, S + 1)).copy()
    _check(q, k, v, off, cols, B, H, S, D)


def test_cfg4_full_size_bf16():
    """Configuration 4's shape and pattern (B=2, H=8, S=4096, D=64, window 256 + every 64th
    column) with the inputs rounded to bf16; every row against the oracle."""
    inp = W.cfg4_csr(seed=0)
    q, k, v = (x.to(BF) for x in (inp.q, inp.k, inp.v))
    _check(q, k, v, inp.offset, inp.columns, inp.B, inp.H, inp.S, inp.D)


def test_data_errors_zero_only_the_bad_rows():
    B, H, S, D = 1, 1, 300, 64
    q, k, v = _inputs(B, H, S, D, BF, 11)
    offs, c = W.window_stride_pattern(S, half_window=8, stride=100)
    off = offs.reshape(1, 1, -1).copy()
    cols = c.reshape(1, 1, -1).copy()
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    bad = cols.copy()
    bad[0, 0, off[0, 0, 20]] = S                       # row 20: a column out of range
    bad[0, 0, off[0, 0, 150] + 1] = bad[0, 0, off[0, 0, 150]]  # row 150: a column stored twice
    out, st = _run(q, k, v, off, bad, B, H, S, D)
    assert st == sdpa.ATTN_ERR_DATA
    assert torch.all(out[0, 0, 20] == 0) and torch.all(out[0, 0, 150] == 0)
    keep = np.ones(S, bool)
    keep[[20, 150]] = False
    absr = oracle.sparse_csr(q, k, v.abs(), off, cols, B=B, H=H, S=S, D=D)
    G.check_out(G.f64(out)[0, 0, keep], ref[0, 0, keep], W.BF16, "other rows", abs_ref=absr[0, 0, keep])


def test_validation():
    q = torch.zeros((1, 1, 8, 96), dtype=BF, device="cuda")
    off = torch.zeros((1, 1, 9), dtype=torch.int32, device="cuda")
    cols = torch.zeros((1, 1, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(sdpa.AttnError) as e:
        sdpa.attn_sparse_csr_tc(q, q, q, off, cols, B=1, H=1, S=8, D=96, nnz_cap=1, dtype=W.BF16, out=q)
    assert e.value.status == sdpa.ATTN_ERR_UNSUPPORTED
    with pytest.raises(ValueError, match="float32"):  # bf16 tensors declared fp32: the binding refuses
        sdpa.attn_sparse_csr_tc(q, q, q, off, cols, B=1, H=1, S=8, D=96, nnz_cap=1, dtype=W.F32, out=q)
    with pytest.raises(sdpa.AttnError) as e:  # fp32 tensors: the library runs 16-bit types only
        qf = q.float()
        sdpa.attn_sparse_csr_tc(qf, qf, qf, off, cols, B=1, H=1, S=8, D=96, nnz_cap=1, dtype=W.F32, out=qf)
    assert e.value.status == sdpa.ATTN_ERR_INVALID


# ---- plans: the pattern's bookkeeping once, then calls that only gather and multiply ---------
def _plan(off, cols, B, H, S):
    """Build the plan of a pattern on the device (inside a guarded buffer). Returns (plan
    tensor, guard, device status of the plan call)."""
    nbytes = sdpa.attn_csr_plan_size(B=B, H=H, S=S, nnz_cap=cols.shape[-1])
    g = G.Guarded((nbytes,), torch.uint8, fill=False)
    sdpa.attn_csr_plan(torch.from_numpy(np.ascontiguousarray(off, np.int32)).cuda(),
                       torch.from_numpy(np.ascontiguousarray(cols, np.int32)).cuda(),
                       B=B, H=H, S=S, nnz_cap=cols.shape[-1], plan=g.t)
    st = sdpa.attn_get_last_error()
    g.check("plan")
    return g.t, st


def _run_planned(q, k, v, plan, B, H, S, D, nnz_cap):
    dq, dk, dv = (torch.as_tensor(x).cuda().contiguous() for x in (q, k, v))
    out = G.guarded_like(dq)
    sdpa.attn_sparse_csr_tc_planned(dq, dk, dv, plan, B=B, H=H, S=S, D=D, nnz_cap=nnz_cap,
                                    dtype=W.dtype_code(dq.dtype), out=out.t)
    st = sdpa.attn_get_last_error()
    out.check("planned out")
    return out.t.cpu(), st


@pytest.mark.parametrize("dtype", [BF, F16], ids=["bf16", "f16"])
@pytest.mark.parametrize("D", [64, 128])
def test_planned_equals_per_call_union(dtype, D):
    """The planned call gives bit for bit the result of the call that builds the union itself
    (same union order, same marks), and both agree with the oracle; the plan is built once and
    serves two different sets of inputs."""
    rng = np.random.default_rng(70 + D)
    B, H, S = 2, 3, 333
    off, cols = _distinct_pattern(rng, B, H, S, 60, empty_every=7)
    plan, st = _plan(off, cols, B, H, S)
    assert st == 0
    for seed in (D, D + 1):
        q, k, v = _inputs(B, H, S, D, dtype, seed)
        got, st = _run_planned(q, k, v, plan, B, H, S, D, cols.shape[-1])
        assert st == 0
        want, st = _run(q, k, v, off, cols, B, H, S, D)
        assert st == 0
        assert torch.equal(got, want)
        ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
        G.check_out(G.f64(got), ref, W.dtype_code(dtype), "planned out",
                    abs_ref=_abs_ref(q, k, v, off, cols, B, H, S, D))


@pytest.mark.parametrize("D", [64, 128])
def test_planned_union_wider_than_one_window(D):
    """Rows of up to 150 random columns over 2,560 keys: unions of about 2,000 columns, so the
    plan's marks are built over two windows of 2,048 union columns."""
    rng = np.random.default_rng(5 + D)
    B, H, S = 1, 2, 2560
    off, cols = _distinct_pattern(rng, B, H, S, 150)
    plan, st = _plan(off, cols, B, H, S)
    assert st == 0
    q, k, v = _inputs(B, H, S, D, BF, 5)
    got, st = _run_planned(q, k, v, plan, B, H, S, D, cols.shape[-1])
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    G.check_out(G.f64(got), ref, W.BF16, "planned wide union", abs_ref=_abs_ref(q, k, v, off, cols, B, H, S, D))


def test_planned_cfg4_full_size_bf16():
    """Configuration 4's shape and pattern (B=2, H=8, S=4096, D=64, window 256 + every 64th
    column) in bf16 from a plan: every row against the oracle."""
    inp = W.cfg4_csr(seed=0)
    q, k, v = (x.to(BF) for x in (inp.q, inp.k, inp.v))
    plan, st = _plan(inp.offset, inp.columns, inp.B, inp.H, inp.S)
    assert st == 0
    got, st = _run_planned(q, k, v, plan, inp.B, inp.H, inp.S, inp.D, inp.nnz_cap)
    assert st == 0
    ref = oracle.sparse_csr(q, k, v, inp.offset, inp.columns, B=inp.B, H=inp.H, S=inp.S, D=inp.D)
    G.check_out(G.f64(got), ref, W.BF16, "planned cfg4",
                abs_ref=_abs_ref(q, k, v, inp.offset, inp.columns, inp.B, inp.H, inp.S, inp.D))


def test_planned_data_errors_zero_only_the_bad_rows():
    B, H, S, D = 1, 1, 300, 64
    q, k, v = _inputs(B, H, S, D, BF, 12)
    offs, c = W.window_stride_pattern(S, half_window=8, stride=100)
    off = offs.reshape(1, 1, -1).copy()
    cols = c.reshape(1, 1, -1).copy()
    ref = oracle.sparse_csr(q, k, v, off, cols, B=B, H=H, S=S, D=D)
    bad = cols.copy()
    bad[0, 0, off[0, 0, 20]] = S                       # row 20: a column out of range
    bad[0, 0, off[0, 0, 150] + 1] = bad[0, 0, off[0, 0, 150]]  # row 150: a column stored twice
    plan, st = _plan(off, bad, B, H, S)
    assert st == sdpa.ATTN_ERR_DATA
    out, st = _run_planned(q, k, v, plan, B, H, S, D, cols.shape[-1])
    assert st == 0
    assert torch.all(out[0, 0, 20] == 0) and torch.all(out[0, 0, 150] == 0)
    keep = np.ones(S, bool)
    keep[[20, 150]] = False
    absr = oracle.sparse_csr(q, k, v.abs(), off, cols, B=B, H=H, S=S, D=D)
    G.check_out(G.f64(out)[0, 0, keep], ref[0, 0, keep], W.BF16, "other rows", abs_ref=absr[0, 0, keep])


def test_buffer_that_is_not_a_plan_is_refused_on_the_device():
    """A buffer of the right size that no attn_csr_plan call filled (all zeros), or a plan built
    for another key count, is not used: every row is written as zeros and ATTN_ERR_DATA is set."""
    B, H, S, D = 1, 2, 300, 64
    offs, c = W.window_stride_pattern(S)
    off = np.broadcast_to(offs, (B, H, S + 1)).copy()
    cols = np.broadcast_to(c, (B, H, c.shape[0])).copy()
    q, k, v = _inputs(B, H, S, D, BF, 13)
    nbytes = sdpa.attn_csr_plan_size(B=B, H=H, S=S, nnz_cap=cols.shape[-1])
    zero = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    out, st = _run_planned(q, k, v, zero, B, H, S, D, cols.shape[-1])
    assert st == sdpa.ATTN_ERR_DATA and torch.all(out == 0)
    # a plan of the same pattern cut to 290 keys has another S in every record
    S2 = 290
    offs2, c2 = W.window_stride_pattern(S2)
    off2 = np.broadcast_to(offs2, (B, H, S2 + 1)).copy()
    cols2 = np.broadcast_to(c2, (B, H, c2.shape[0])).copy()
    plan2, st = _plan(off2, cols2, B, H, S2)
    assert st == 0
    big = torch.zeros(max(nbytes, plan2.numel()), dtype=torch.uint8, device="cuda")
    big[:plan2.numel()].copy_(plan2)
    out, st = _run_planned(q, k, v, big, B, H, S, D, cols.shape[-1])
    assert st == sdpa.ATTN_ERR_DATA and torch.all(out == 0)


def test_plan_is_deterministic_and_reusable():
    """A plan depends on the pattern only: two builds of the same pattern give the same bytes
    (the marks' atomic ORs land in any order but OR is order-free), and one plan serves any
    number of calls with bit-identical results."""
    rng = np.random.default_rng(91)
    B, H, S, D = 1, 2, 700, 64
    off, cols = _distinct_pattern(rng, B, H, S, 80)
    p1, st1 = _plan(off, cols, B, H, S)
    p2, st2 = _plan(off, cols, B, H, S)
    assert st1 == 0 and st2 == 0
    # both buffers start zeroed, so the whole plans compare, unused tails included
    assert torch.equal(p1, p2)
    q, k, v = _inputs(B, H, S, D, BF, 91)
    a, sa = _run_planned(q, k, v, p1, B, H, S, D, cols.shape[-1])
    b, sb = _run_planned(q, k, v, p1, B, H, S, D, cols.shape[-1])
    c, sc = _run_planned(q, k, v, p2, B, H, S, D, cols.shape[-1])
    assert sa == sb == sc == 0
    assert torch.equal(a, b) and torch.equal(a, c)
