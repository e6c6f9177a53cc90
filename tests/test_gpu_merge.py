"""attn_merge on the GPU against the float64 oracle, and the chunked-attention merge chain."""
import numpy as np
import pytest
import torch

import oracle
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _merge_gpu(po, pm, ps, co, cm, cs, S, B, N, D, dtype, inplace=False):
    """The merge on the device into guarded outputs (for the in-place form, guarded copies of
    the previous side that the call overwrites)."""
    prev = [G.guarded_copy(t.contiguous()) for t in (po, pm, ps)]
    cur = [t.cuda().contiguous() for t in (co, cm, cs)]
    outs = prev if inplace else [G.guarded_like(g.t) for g in prev]
    sdpa.attn_merge(*(g.t for g in prev), *cur, S=S, B=B, N=N, D=D, dtype=dtype, out=outs[0].t,
                    out_max=outs[1].t, out_sum=outs[2].t)
    assert sdpa.attn_get_last_error() == 0
    for g in prev + outs:
        g.check("merge")
    return outs[0].t.cpu(), outs[1].t.cpu(), outs[2].t.cpu()


def rne_eps(po, co) -> np.ndarray:
    """Bound on the fp32 arithmetic's error in an output element before its single rounding:
    both scales lie in [0, 1] (positive sums), and each product carries a few fp32 roundings
    plus expf's, so 2^-18 (|prev| + |cur|) bounds it with room to spare."""
    return 2.0 ** -18 * (np.abs(G.f64(po)) + np.abs(G.f64(co)))


def _check_out_merge(out, ro, po, co, dtype, what):
    if dtype == W.F32:
        G.check_out(G.f64(out), ro, dtype, what)
    else:
        G.check_rne(out, ro, dtype, rne_eps(po, co), what)


def _check_merge(po, pm, ps, co, cm, cs, S, B, N, D, dtype, inplace=False):
    out, om, osum = _merge_gpu(po, pm, ps, co, cm, cs, S, B, N, D, dtype, inplace)
    ro, rm, rs = oracle.merge(po, pm, ps, co, cm, cs, S=S, B=B, N=N, D=D)
    _check_out_merge(out, ro, po, co, dtype, "merge out")
    G.check_stats(om.numpy(), osum.numpy(), rm, rs, "merge stats")


@pytest.mark.parametrize("dtype", [W.BF16, W.F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("S,B,N,D", [(2048, 1, 12, 1), (100, 2, 3, 128), (37, 3, 5, 40), (1, 1, 1, 8)])
@pytest.mark.parametrize("lanes_equal", [True, False])
def test_merge_random(dtype, S, B, N, D, lanes_equal):
    tdt = torch.bfloat16 if dtype == W.BF16 else torch.float32
    po = W.randn((S, B, N * D), 1, tdt)
    co = W.randn((S, B, N * D), 2, tdt)
    pm, ps = W.merge_stats_random(B, N, S, 3, lanes_equal)
    cm, cs = W.merge_stats_random(B, N, S, 5, lanes_equal)
    _check_merge(po, pm, ps, co, cm, cs, S, B, N, D, dtype)


def test_merge_page_example_shapes():
    """The op page's example shapes (out [2048,1,12], stats [1,12,2048,8] of randn values; N=12
    heads of d=1). With randn sums the page's formula is applied literally."""
    S, B, N, D = 2048, 1, 12, 1
    po = W.randn((S, B, N * D), 11, torch.bfloat16)
    co = W.randn((S, B, N * D), 12, torch.bfloat16)
    pm, ps, cm, cs = (W.randn((B, N, S, 8), 13 + i) for i in range(4))
    out, om, osum = _merge_gpu(po, pm, ps, co, cm, cs, S, B, N, D, W.BF16)
    ro, rm, rs = oracle.merge(po, pm, ps, co, cm, cs, S=S, B=B, N=N, D=D)
    # statistics lane by lane; random sums of either sign can cancel, so compare absolutely too
    assert np.allclose(om.numpy(), rm, rtol=1e-6, atol=0)
    assert np.allclose(osum.numpy(), rs, rtol=1e-5, atol=1e-5)
    # outputs on rows where the lane-0 sum does not cancel (|l| >= |ps'| + |cs'| over 10):
    # elsewhere fp32 and float64 legitimately disagree about the near-zero denominator
    m = np.maximum(pm.numpy(), cm.numpy())[..., 0].astype(np.float64)
    a = np.abs(ps.numpy()[..., 0] * np.exp(pm.numpy()[..., 0] - m))
    c = np.abs(cs.numpy()[..., 0] * np.exp(cm.numpy()[..., 0] - m))
    good = (np.abs(rs[..., 0]) * 10 >= a + c)            # [B, N, S]
    good_sbh = np.repeat(np.transpose(good, (2, 0, 1)), D, axis=2)  # [S, B, N*D]
    err = np.abs(G.f64(out) - ro)[good_sbh]
    tol = np.maximum(1e-2, G.bf16_ulp(ro[good_sbh])) * (1.0 + np.abs(ro[good_sbh]))
    assert good.mean() > 0.5 and np.all(err <= tol)


def test_merge_inplace_alias():
    S, B, N, D = 300, 2, 4, 128
    po = W.randn((S, B, N * D), 21, torch.bfloat16)
    co = W.randn((S, B, N * D), 22, torch.bfloat16)
    pm, ps = W.merge_stats_random(B, N, S, 23)
    cm, cs = W.merge_stats_random(B, N, S, 25)
    _check_merge(po, pm, ps, co, cm, cs, S, B, N, D, W.BF16, inplace=True)


def test_merge_empty_sides():
    S, B, N, D = 64, 2, 2, 128
    o = W.randn((S, B, N * D), 31, torch.bfloat16)
    m, l = W.merge_stats_random(B, N, S, 32)
    ninf = torch.full_like(m, float("-inf"))
    zero = torch.zeros_like(l)
    out, om, osum = _merge_gpu(o, m, l, torch.zeros_like(o), ninf, zero, S, B, N, D, W.BF16)
    assert torch.equal(out, o) and torch.equal(om, m) and torch.equal(osum, l)
    out, om, osum = _merge_gpu(o, ninf, zero, o, ninf, zero, S, B, N, D, W.BF16)
    assert torch.all(out == 0) and torch.all(torch.isneginf(om)) and torch.all(osum == 0)


def _chunked_partials(B, N, S, Skv, D, chunks, seed):
    """Partials of a non-causal attention over `chunks` key chunks, from attn_fwd, converted to
    the merge layouts (out [S,B,N*D], statistics [B,N,S,8])."""
    inp = W.dense_bhsd(B, N, S, D, causal=False, dtype=torch.bfloat16, seed=seed, cfg=5, Skv=Skv)
    c = Skv // chunks
    parts = []
    for i in range(chunks):
        sub = W.AttnInputs(inp.q, inp.k[:, :, i * c:(i + 1) * c].contiguous(),
                           inp.v[:, :, i * c:(i + 1) * c].contiguous(), W.BHSD, W.MASK_NONE,
                           W.BF16, B, S, c, N, N, D, inp.scale)
        o, m, l = G.run_fwd(sub)
        parts.append((o.permute(2, 0, 1, 3).reshape(S, B, N * D).contiguous(),
                      m.unsqueeze(-1).expand(B, N, S, 8).contiguous(),
                      l.unsqueeze(-1).expand(B, N, S, 8).contiguous()))
    return inp, parts


def _merge_chain_check(B, N, S, Skv, D, seed, sampled):
    inp, parts = _chunked_partials(B, N, S, Skv, D, 4, seed)
    acc = [t.cuda() for t in parts[0]]
    for p in parts[1:]:
        cur = [t.cuda() for t in p]
        sdpa.attn_merge(acc[0], acc[1], acc[2], *cur, S=S, B=B, N=N, D=D, dtype=W.BF16,
                        out=acc[0], out_max=acc[1], out_sum=acc[2])
    assert sdpa.attn_get_last_error() == 0
    out = acc[0].cpu().reshape(S, B, N, D).permute(1, 2, 0, 3)  # -> [B, N, S, D]
    m = acc[1][..., 0].cpu()
    l = acc[2][..., 0].cpu()
    if sampled:
        rows_h, rows_t = G.sample_rows(inp, seed, n_random=512, edge=8)
        og, mg, lg = G.gather_rows(out, m, l, inp, rows_h, rows_t)
        ref, rm, rl = G.oracle_rows(inp, rows_h, rows_t)
    else:
        og, mg, lg = G.f64(out), m.numpy(), l.numpy()
        ref, rm, rl = G.oracle_fwd(inp)
    # a non-causal attention over 1,024 or more keys: every |exact| is far below 4
    G.check_out(og, ref, W.BF16, "merged out vs full attention")
    G.check_stats(mg, lg, rm, rl, "merged stats vs full attention")


def test_merge_chain_equals_full_attention_small():
    _merge_chain_check(2, 4, 300, 1024, 128, seed=1, sampled=False)


def test_merge_chain_cfg5_full_size():
    """Configuration 5: S=8192, B=4, N=32, D=128; Skv=8192 split into 4 chunks of 2048."""
    _merge_chain_check(4, 32, 8192, 8192, 128, seed=0, sampled=True)


# ---- TND layout and fp16 ---------------------------------------------------------------------
def _merge_tnd_gpu(po, pm, ps, co, cm, cs, T, N, D, dtype, seq_qlen=None, B=0):
    dev = [t.cuda().contiguous() for t in (po, pm, ps, co, cm, cs)]
    outs = [G.guarded_like(t) for t in dev[:3]]
    sq = None if seq_qlen is None else torch.as_tensor(seq_qlen, dtype=torch.int64).cuda()
    sdpa.attn_merge(*dev, S=T, B=B, N=N, D=D, dtype=dtype, out=outs[0].t, out_max=outs[1].t,
                    out_sum=outs[2].t, layout=sdpa.ATTN_TND, actual_seq_qlen=sq)
    st = sdpa.attn_get_last_error()
    for g in outs:
        g.check("TND merge")
    return outs[0].t.cpu(), outs[1].t.cpu(), outs[2].t.cpu(), st


@pytest.mark.parametrize("dtype,tdt", [(W.BF16, torch.bfloat16), (W.F16, torch.float16), (W.F32, torch.float32)],
                         ids=["bf16", "f16", "f32"])
@pytest.mark.parametrize("T,N,D", [(1000, 4, 128), (37, 3, 40), (513, 12, 1)])
def test_merge_tnd(dtype, tdt, T, N, D):
    po = W.randn((T, N * D), 41, tdt)
    co = W.randn((T, N * D), 42, tdt)
    pm, ps = W.merge_stats_random(1, T, N, 43, lanes_equal=False)
    cm, cs = W.merge_stats_random(1, T, N, 45, lanes_equal=False)
    pm, ps, cm, cs = (x[0] for x in (pm, ps, cm, cs))  # [T, N, 8]
    out, om, osum, st = _merge_tnd_gpu(po, pm, ps, co, cm, cs, T, N, D, dtype)
    assert st == 0
    ro, rm, rs = oracle.merge(po, pm, ps, co, cm, cs, S=T, B=0, N=N, D=D, layout=W.TND)
    _check_out_merge(out, ro, po, co, dtype, "tnd merge out")
    G.check_stats(om.numpy(), osum.numpy(), rm, rs, "tnd merge stats")


def test_merge_tnd_seq_qlen_checked():
    T, N, D = 64, 2, 128
    po = W.randn((T, N * D), 51, torch.bfloat16)
    pm, ps = W.merge_stats_random(1, T, N, 52)
    pm, ps = pm[0], ps[0]
    _, _, _, st = _merge_tnd_gpu(po, pm, ps, po, pm, ps, T, N, D, W.BF16, seq_qlen=[10, 10, 64], B=3)
    assert st == 0
    _, _, _, st = _merge_tnd_gpu(po, pm, ps, po, pm, ps, T, N, D, W.BF16, seq_qlen=[10, 5, 64], B=3)
    assert st == sdpa.ATTN_ERR_DATA
    _, _, _, st = _merge_tnd_gpu(po, pm, ps, po, pm, ps, T, N, D, W.BF16, seq_qlen=[10, 20, 63], B=3)
    assert st == sdpa.ATTN_ERR_DATA


@pytest.mark.parametrize("S,B,N,D", [(100, 2, 3, 128), (37, 3, 5, 40)])
def test_merge_f16_sbh(S, B, N, D):
    po = W.randn((S, B, N * D), 61, torch.float16)
    co = W.randn((S, B, N * D), 62, torch.float16)
    pm, ps = W.merge_stats_random(B, N, S, 63)
    cm, cs = W.merge_stats_random(B, N, S, 65)
    _check_merge(po, pm, ps, co, cm, cs, S, B, N, D, W.F16)
