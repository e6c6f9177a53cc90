"""attn_fwd on the GPU against the float64 oracle (element by element), through the C ABI."""
import numpy as np
import pytest
import torch

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

BF, F32 = torch.bfloat16, torch.float32


def _full_check(inp, stats=True):
    out, m, l = G.run_fwd(inp, stats=stats)
    ref, rm, rl = G.oracle_fwd(inp)
    info = G.check_out(G.f64(out), ref, inp.dtype, abs_ref=lambda: G.oracle_abs_fwd(inp))
    if stats:
        G.check_stats(m.numpy(), l.numpy(), rm, rl)
    return info


# ---- configuration 1: dense 2x4x256x64, non-causal, fp32 and bf16 ---------------------------
@pytest.mark.parametrize("dtype", [F32, BF], ids=["f32", "bf16"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_cfg1_dense_small(dtype, seed):
    _full_check(W.cfg1_dense_small(dtype, seed))


# ---- dense BHSD shapes spanning several tiles with ragged tails ------------------------------
@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("S", [1, 100, 256, 300, 640])
def test_dense_shapes(dtype, D, causal, S):
    inp = W.dense_bhsd(2, 3, S, D, causal=causal, dtype=dtype, seed=S + D, cfg=11)
    _full_check(inp)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("Sq,Skv", [(200, 700), (700, 200), (129, 1), (1, 513)])
@pytest.mark.parametrize("mode", [W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, W.MASK_CAUSAL_BOTTOMRIGHT])
def test_rectangular_and_masks(dtype, Sq, Skv, mode):
    inp = W.dense_bhsd(1, 2, Sq, 128, causal=False, dtype=dtype, seed=Sq * 7 + Skv, cfg=12, Skv=Skv)
    inp.mask_mode = mode
    _full_check(inp)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("Nq,Nkv", [(8, 2), (6, 1), (4, 4)])
def test_gqa_mqa(dtype, Nq, Nkv):
    inp = W.dense_bhsd(2, Nq, 333, 128, causal=True, dtype=dtype, seed=Nq + Nkv, cfg=13, Hkv=Nkv)
    _full_check(inp)


# ---- packed varlen (TND) ---------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("lens", [[2, 2, 0, 2, 2], [0, 700, 1, 0, 257, 513, 0], [1000], [0, 0, 5]])
@pytest.mark.parametrize("mode", [W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT])
def test_varlen(dtype, lens, mode):
    inp = W.varlen_tnd(lens, 8, 2, 128, causal=False, dtype=dtype, seed=sum(lens), cfg=14,
                       mask_mode=mode)
    _full_check(inp)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
def test_varlen_different_kv_lengths(dtype):
    lq, lk = [100, 0, 300, 129], [250, 7, 300, 0]
    for mode in (W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, W.MASK_CAUSAL_BOTTOMRIGHT):
        inp = W.varlen_tnd(lq, 4, 1, 64, causal=False, dtype=dtype, seed=5, cfg=15, lengths_kv=lk,
                           mask_mode=mode)
        _full_check(inp)


def test_cfg3_small_varlen_gqa():
    """Configuration 3 in miniature: 16 sequences up to 1024 tokens (index 7 empty), GQA 32/8."""
    inp = W.cfg3_varlen_gqa(seed=0, max_len=1024)
    _full_check(inp)


def test_no_stats_pointer():
    inp = W.dense_bhsd(1, 2, 300, 128, causal=True, dtype=BF, seed=3, cfg=16)
    out, _, _ = G.run_fwd(inp, stats=False)
    ref, _, _ = G.oracle_fwd(inp)
    G.check_out(G.f64(out), ref, inp.dtype, abs_ref=lambda: G.oracle_abs_fwd(inp))


# ---- full-size configurations: sampled rows ----------------------------------------------------
def _sampled_check(inp, seed):
    out, m, l = G.run_fwd(inp)
    rows_h, rows_t = G.sample_rows(inp, seed)
    og, mg, lg = G.gather_rows(out, m, l, inp, rows_h, rows_t)
    ref, rm, rl = G.oracle_rows(inp, rows_h, rows_t)
    G.check_out(og, ref, inp.dtype, abs_ref=lambda: G.oracle_abs_rows(inp, rows_h, rows_t))
    G.check_stats(mg, lg, rm, rl)
    # every output is finite (no NaN from masked or padded rows)
    assert torch.isfinite(out.float()).all()


def test_cfg2_full_size_sampled():
    _sampled_check(W.cfg2_dense_causal(seed=0), seed=2)


def test_cfg3_full_size_sampled():
    _sampled_check(W.cfg3_varlen_gqa(seed=0), seed=3)


# ---- properties -----------------------------------------------------------------------------------
def test_deterministic_bitwise():
    inp = W.cfg3_varlen_gqa(seed=1, max_len=2048)
    a = G.run_fwd(inp)
    b = G.run_fwd(inp)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_varlen_equals_dense_per_sequence():
    lens = [300, 0, 513]
    inp = W.varlen_tnd(lens, 4, 2, 128, causal=True, dtype=BF, seed=9, cfg=17)
    out, m, l = G.run_fwd(inp)
    start = 0
    for L in lens:
        if L == 0:
            continue
        q = inp.q[start:start + L].permute(1, 0, 2).unsqueeze(0).contiguous()
        k = inp.k[start:start + L].permute(1, 0, 2).unsqueeze(0).contiguous()
        v = inp.v[start:start + L].permute(1, 0, 2).unsqueeze(0).contiguous()
        d = W.AttnInputs(q, k, v, W.BHSD, W.MASK_CAUSAL_TOPLEFT, W.BF16, 1, L, L, 4, 2, 128, inp.scale)
        od, md, ld = G.run_fwd(d)
        assert torch.equal(od[0].permute(1, 0, 2), out[start:start + L])
        assert torch.equal(md[0].T, m[start:start + L]) and torch.equal(ld[0].T, l[start:start + L])
        start += L


@pytest.mark.parametrize("masked", [False, True], ids=["attn_fwd", "attn_fwd_masked"])
def test_tnd_rows_past_each_sequence_untouched(masked):
    """Each sequence of a packed batch run as a batch of its own, on views that start at its
    first token: the last row block of a sequence covers rows past its end (the next sequence's
    tokens, pre-filled with the NaN pattern), and none of them may be stored. Afterwards the
    assembled outputs equal the packed call's bit for bit."""
    lens = [300, 129, 1, 513, 0, 256, 77]
    inp = W.varlen_tnd(lens, 4, 2, 128, causal=True, dtype=BF, seed=21, cfg=24)
    q, k, v, _, _ = G.to_dev(inp)
    out = G.Guarded(tuple(q.shape), q.dtype)
    m = G.Guarded((inp.Sq, inp.Nq), torch.float32)
    l = G.Guarded((inp.Sq, inp.Nq), torch.float32)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).tolist()
    for s0, L in zip(starts, lens):
        if L == 0:
            continue
        before = [g.buf.view(torch.int16).clone() for g in (out, m, l)]
        cu = torch.tensor([L], dtype=torch.int32, device="cuda")
        kw = dict(cu_seqlens_q=cu, cu_seqlens_kv=cu, B=1, Sq=L, Skv=L, Nq=4, Nkv=2, scale=inp.scale,
                  dtype=W.BF16, layout=W.TND, out=out.t[s0:s0 + L], softmax_max=m.t[s0:s0 + L],
                  softmax_sum=l.t[s0:s0 + L])
        sl = slice(s0, s0 + L)
        if masked:
            sdpa.attn_fwd_masked(q[sl], k[sl], v[sl], Dqk=128, Dv=128, mask_mode=W.MASK_CAUSAL_TOPLEFT, **kw)
        else:
            sdpa.attn_fwd(q[sl], k[sl], v[sl], D=128, mask_mode=W.MASK_CAUSAL_TOPLEFT, **kw)
        assert sdpa.attn_get_last_error() == 0
        for g, b, per_row in ((out, before[0], inp.Nq * 128), (m, before[1], inp.Nq * 2),
                              (l, before[2], inp.Nq * 2)):
            now = g.buf.view(torch.int16)
            a = g.g * g.buf.element_size() // 2 + s0 * per_row  # first int16 of this sequence's rows
            e = a + L * per_row
            assert torch.equal(now[:a], b[:a]) and torch.equal(now[e:], b[e:]), \
                f"sequence at {s0} (length {L}) stored outside its rows"
        for g in (out, m, l):
            g.check()
    whole = G.run_fwd(inp)
    assert torch.equal(out.t.cpu(), whole[0])
    assert torch.equal(m.t.cpu(), whole[1]) and torch.equal(l.t.cpu(), whole[2])


# ---- boundary errors ------------------------------------------------------------------------------
def test_bad_cu_seqlens_reports_data_error():
    inp = W.varlen_tnd([100, 200], 2, 2, 128, causal=True, dtype=BF, seed=1, cfg=18)
    q, k, v, cq, ck = G.to_dev(inp)
    out = torch.zeros_like(q)
    bad = torch.tensor([200, 100], dtype=torch.int32, device="cuda")  # decreasing
    sdpa.attn_fwd(q, k, v, cu_seqlens_q=bad, cu_seqlens_kv=ck, B=2, Sq=300, Skv=300, Nq=2, Nkv=2,
                  D=128, scale=inp.scale, mask_mode=1, dtype=W.BF16, layout=W.TND, out=out)
    assert sdpa.attn_get_last_error() == sdpa.ATTN_ERR_DATA
    assert sdpa.attn_get_last_error() == 0  # read clears the word


def test_host_validation():
    inp = W.dense_bhsd(1, 2, 64, 128, causal=False, dtype=BF, seed=1, cfg=19)
    q, k, v, _, _ = G.to_dev(inp)
    out = torch.empty_like(q)
    kw = dict(B=1, Sq=64, Skv=64, Nq=2, Nkv=2, D=128, scale=0.1, mask_mode=0, dtype=W.BF16,
              layout=W.BHSD, out=out)
    with pytest.raises(sdpa.AttnError) as e:  # Nq not a multiple of Nkv (tensors large enough)
        sdpa.attn_fwd(q, k, v, **{**kw, "Nq": 3, "Nkv": 2, "Sq": 32, "Skv": 32})
    assert e.value.status == sdpa.ATTN_ERR_INVALID
    with pytest.raises(ValueError, match="holds"):  # k too small for Nkv = 3: refused by the binding
        sdpa.attn_fwd(q, k, v, **{**kw, "Nkv": 3})
    with pytest.raises(sdpa.AttnError) as e:
        sdpa.attn_fwd(q, k, v, **{**kw, "D": 96})
    assert e.value.status == sdpa.ATTN_ERR_UNSUPPORTED
    # a contiguous view that starts 2 bytes into its buffer: the library's alignment check
    buf = torch.empty(q.numel() + 1, dtype=q.dtype, device=q.device)
    qm = buf[1:].view(q.shape)
    qm.copy_(q)
    with pytest.raises(sdpa.AttnError) as e:
        sdpa.attn_fwd(qm, k, v, **kw)
    assert e.value.status == sdpa.ATTN_ERR_INVALID
    # a strided view is refused by the binding before the library is called
    with pytest.raises(ValueError):
        sdpa.attn_fwd(q[..., 1:], k, v, **kw)


# ---- fp16 on the tensor-core path ---------------------------------------------------------------
F16 = torch.float16


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_f16_dense(D, causal):
    _full_check(W.dense_bhsd(2, 3, 300, D, causal=causal, dtype=F16, seed=D, cfg=21))


def test_f16_varlen_gqa():
    _full_check(W.varlen_tnd([0, 700, 1, 257, 0, 513], 8, 2, 128, causal=True, dtype=F16, seed=4, cfg=22))


def test_f16_matches_bf16_path_structure():
    """Same inputs rounded to fp16 and to bf16: both paths agree with the exact result."""
    base = W.dense_bhsd(1, 2, 200, 128, causal=True, dtype=torch.float32, seed=5, cfg=23)
    for dt in (F16, BF):
        inp = W.AttnInputs(base.q.to(dt), base.k.to(dt), base.v.to(dt), W.BHSD, W.MASK_CAUSAL_TOPLEFT,
                           W.dtype_code(dt), 1, 200, 200, 2, 2, 128, base.scale)
        _full_check(inp)
