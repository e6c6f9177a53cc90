"""attn_sparse_csr_tc_noalloc against attn_sparse_csr_tc, through the C ABI, on two calls in a row.

Some callers of this library cannot allocate device memory: a plugin running inside a host
application that owns all GPU memory through its own pool and hands out no workspace, or a path
where cudaMalloc's possible device synchronisation or failure is not acceptable. The no-alloc
entry point serves them from a fixed 48 MiB scratch array inside the library, in which it plans
the pattern before running the planned kernel. Its two calls here use different patterns, head
sizes and types, so the second one reuses the scratch that the first one filled; each must agree
with the existing entry point (which builds its union per block and needs no plan) within the
16-bit tolerance the other tests use. A pattern whose plan exceeds the scratch is refused.

This file is collected after every other test file, so a run that stops at its first failure has
already run the rest; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _pattern_cfg4():
    inp = W.cfg4_csr(seed=3)
    return inp.offset, inp.columns, inp.B, inp.H, inp.S, inp.D


def _pattern_random(S=700, D=128):
    rng = np.random.default_rng(11)
    B, H = 1, 3
    offs = np.zeros((B * H, S + 1), np.int32)
    rows = []
    for bh in range(B * H):
        cnt = rng.integers(0, 41, size=S)
        offs[bh, 1:] = np.cumsum(cnt)
        rows.append(np.concatenate([rng.permutation(S)[:c] for c in cnt]))
    cap = max(len(r) for r in rows)
    cols = np.zeros((B * H, cap), np.int32)
    for bh, r in enumerate(rows):
        cols[bh, :len(r)] = r
    return offs.reshape(B, H, S + 1), cols.reshape(B, H, cap), B, H, S, D


def _both(off, cols, B, H, S, D, dtype, seed):
    q, k, v = (W.randn((B, H, S, D), 900 + 3 * seed + i).to(dtype).cuda() for i in range(3))
    doff = torch.from_numpy(np.ascontiguousarray(off)).cuda()
    dcol = torch.from_numpy(np.ascontiguousarray(cols)).cuda()
    code = W.dtype_code(dtype)
    new = G.guarded_like(q)
    sdpa.attn_sparse_csr_tc_noalloc(q, k, v, doff, dcol, B=B, H=H, S=S, D=D, nnz_cap=cols.shape[-1],
                                    dtype=code, out=new.t)
    st_new = sdpa.attn_get_last_error()
    new.check("no-alloc out")
    old = G.guarded_like(q)
    sdpa.attn_sparse_csr_tc(q, k, v, doff, dcol, B=B, H=H, S=S, D=D, nnz_cap=cols.shape[-1], dtype=code,
                            out=old.t)
    st_old = sdpa.attn_get_last_error()
    old.check("existing out")
    return new.t.cpu(), old.t.cpu(), st_new, st_old


def test_noalloc_matches_existing_entry_point_on_two_calls_in_a_row():
    calls = [(_pattern_cfg4(), torch.bfloat16, 1),      # workload 4's pattern: a 42 MB plan
             (_pattern_random(), torch.float16, 2)]     # another pattern, D = 128, fp16
    for (off, cols, B, H, S, D), dtype, seed in calls:
        new, old, st_new, st_old = _both(off, cols, B, H, S, D, dtype, seed)
        assert st_new == 0 and st_old == 0
        assert torch.isfinite(new.float()).all()
        diff = (new.double() - old.double()).abs().max().item()
        assert diff <= G.BF16_ABS, f"no-alloc and existing entry points differ by {diff}"


def test_noalloc_refuses_a_plan_larger_than_its_scratch():
    """S = 32,768 keys with up to 32,768 entries per (b, h): its plan needs 168 MB, more than the
    48 MiB scratch, and the call is refused before anything runs."""
    S, D = 32768, 64
    q = torch.zeros((1, 1, S, D), dtype=torch.bfloat16, device="cuda")
    off = torch.arange(S + 1, dtype=torch.int32, device="cuda")
    cols = torch.arange(S, dtype=torch.int32, device="cuda")
    need = sdpa.attn_csr_plan_size(B=1, H=1, S=S, nnz_cap=S)
    assert need > 48 << 20
    out = torch.zeros_like(q)
    with pytest.raises(sdpa.AttnError) as e:
        sdpa.attn_sparse_csr_tc_noalloc(q, q, q, off, cols, B=1, H=1, S=S, D=D, nnz_cap=S,
                                        dtype=sdpa.ATTN_BF16, out=out)
    assert e.value.status == sdpa.ATTN_ERR_UNSUPPORTED
    assert sdpa.attn_get_last_error() == 0
    assert torch.all(out == 0)
