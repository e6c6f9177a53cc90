"""attn_fwd at the limits the Ascend constraints set (约束说明): 2,048 cumulative-length entries,
Nq = 256 heads (MQA), T = 1M (2^20) packed tokens, and the fp32 path at its largest head size."""
import numpy as np
import pytest
import torch

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

BF, F32 = torch.bfloat16, torch.float32


def _full(inp):
    out, m, l = G.run_fwd(inp)
    ref, rm, rl = G.oracle_fwd(inp)
    G.check_out(G.f64(out), ref, inp.dtype, abs_ref=lambda: G.oracle_abs_fwd(inp))
    G.check_stats(m.numpy(), l.numpy(), rm, rl)


def test_2048_sequences():
    """The most cumulative-length entries the constraints allow, lengths 0..64 (zeros included)."""
    rng = np.random.default_rng(7)
    lens = rng.integers(0, 65, size=2048)
    lens[::97] = 0
    inp = W.varlen_tnd(lens.tolist(), 8, 2, 128, causal=False, dtype=BF, seed=1, cfg=50,
                       mask_mode=W.MASK_CAUSAL_TOPLEFT)
    _full(inp)


def test_256_heads_mqa():
    inp = W.dense_bhsd(1, 256, 300, 64, causal=True, dtype=BF, seed=2, cfg=51, Hkv=1)
    _full(inp)


@pytest.mark.parametrize("S", [33, 200])
def test_f32_largest_head_size(S):
    _full(W.dense_bhsd(1, 2, S, 256, causal=True, dtype=F32, seed=3, cfg=52))


def test_one_million_tokens_sampled():
    """T = 2^20 packed tokens (16 causal sequences of 65,536), Nq = Nkv = 1, D = 64: sampled
    rows, including the first and last rows of every sequence, against the oracle."""
    inp = W.varlen_tnd([65536] * 16, 1, 1, 64, causal=False, dtype=BF, seed=4, cfg=53,
                       mask_mode=W.MASK_CAUSAL_TOPLEFT)
    assert inp.Sq == 1 << 20
    out, m, l = G.run_fwd(inp)
    rows_h, rows_t = G.sample_rows(inp, 9, n_random=256, edge=8, heads=[0])
    og, mg, lg = G.gather_rows(out, m, l, inp, rows_h, rows_t)
    ref, rm, rl = G.oracle_rows(inp, rows_h, rows_t)
    G.check_out(og, ref, inp.dtype, abs_ref=lambda: G.oracle_abs_rows(inp, rows_h, rows_t))
    G.check_stats(mg, lg, rm, rl)
    assert torch.isfinite(out.float()).all()


def test_one_token_past_the_limit_is_rejected():
    q = torch.zeros((1 << 20) + 1, 1, 64, dtype=BF, device="cuda")
    cu = torch.tensor([(1 << 20) + 1], dtype=torch.int32, device="cuda")
    with pytest.raises(sdpa.AttnError) as e:
        sdpa.attn_fwd(q, q, q, cu_seqlens_q=cu, cu_seqlens_kv=cu, B=1, Sq=(1 << 20) + 1,
                      Skv=(1 << 20) + 1, Nq=1, Nkv=1, D=64, scale=0.125, mask_mode=1,
                      dtype=W.BF16, layout=W.TND, out=q)
    assert e.value.status == sdpa.ATTN_ERR_INVALID
