"""attn_fwd_masked on the GPU against the float64 oracle: band limits (preTokens/nextTokens),
an explicit uint8 mask (1 = excluded) and a value head size Dv < Dqk, through the C ABI.

Readings (the page lists these inputs without the table that defines the sparse modes): key j
is visible to row i iff i - pre <= j <= i + next (in-sequence positions); a mask entry of 1
excludes the key; the two combine by AND. Tolerances are those of the other parity tests."""
import numpy as np
import pytest
import torch

import oracle
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

BF, F16, F32 = torch.bfloat16, torch.float16, torch.float32
BAND = sdpa.ATTN_MASK_BAND


def _run(inp, *, mode, pre=0, nxt=0, mask=None, bs=0, rs=0, Dv=None, stats=True):
    q, k, v, cq, ck = G.to_dev(inp)
    Dv = inp.D if Dv is None else Dv
    shape_o = (inp.B, inp.Nq, inp.Sq, Dv) if inp.layout == W.BHSD else (inp.Sq, inp.Nq, Dv)
    shape_s = (inp.B, inp.Nq, inp.Sq) if inp.layout == W.BHSD else (inp.Sq, inp.Nq)
    out = G.Guarded(shape_o, q.dtype)  # NaN-filled: every element must be written
    m = G.Guarded(shape_s, torch.float32) if stats else None
    l = G.Guarded(shape_s, torch.float32) if stats else None
    md = None if mask is None else torch.from_numpy(mask).cuda()
    sdpa.attn_fwd_masked(q, k, v, cu_seqlens_q=cq, cu_seqlens_kv=ck, B=inp.B, Sq=inp.Sq,
                         Skv=inp.Skv, Nq=inp.Nq, Nkv=inp.Nkv, Dqk=inp.D, Dv=Dv, scale=inp.scale,
                         mask_mode=mode, pre_tokens=pre, next_tokens=nxt, atten_mask=md,
                         mask_batch_stride=bs, mask_row_stride=rs, dtype=inp.dtype,
                         layout=inp.layout, out=out.t, softmax_max=m.t if stats else None,
                         softmax_sum=l.t if stats else None)
    assert sdpa.attn_get_last_error() == 0
    for g in (out, m, l):
        if g is not None:
            g.check()
    return out.t.cpu(), (m.t.cpu() if stats else None), (l.t.cpu() if stats else None)


def _oracle(inp, *, mode, pre=0, nxt=0, mask=None, bs=0, rs=0, Dv=None):
    return oracle.attn_fwd_ext(inp.q, inp.k, inp.v, cu_q=inp.cu_q, cu_kv=inp.cu_kv, B=inp.B,
                               Sq=inp.Sq, Skv=inp.Skv, Nq=inp.Nq, Nkv=inp.Nkv, Dqk=inp.D,
                               Dv=inp.D if Dv is None else Dv, scale=inp.scale, mask_mode=mode,
                               pre_tokens=pre, next_tokens=nxt, mask=mask, mask_bstride=bs,
                               mask_rstride=rs, layout=inp.layout)


def _check(inp, **kw):
    out, m, l = _run(inp, **kw)
    ref, rm, rl = _oracle(inp, **kw)
    G.check_out(G.f64(out), ref, inp.dtype, abs_ref=lambda: _oracle(G.abs_v(inp), **kw)[0])
    G.check_stats(m.numpy(), l.numpy(), rm, rl)
    return out, m, l


BANDS = [(0, 0), (64, 0), (200, 50), (-100, 300), (5, -3), (127, 128), (1 << 40, 1 << 40)]


@pytest.mark.parametrize("dtype", [BF, F16, F32], ids=["bf16", "f16", "f32"])
@pytest.mark.parametrize("pre,nxt", BANDS)
def test_band_dense(dtype, pre, nxt):
    inp = W.dense_bhsd(2, 2, 300, 128, causal=False, dtype=dtype, seed=pre % 97 + nxt % 89, cfg=31)
    _check(inp, mode=BAND, pre=pre, nxt=nxt)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("Sq,Skv", [(640, 200), (200, 640)])
def test_band_rectangular_gqa_d64(dtype, Sq, Skv):
    inp = W.dense_bhsd(1, 4, Sq, 64, causal=False, dtype=dtype, seed=Sq + Skv, cfg=32, Skv=Skv, Hkv=2)
    _check(inp, mode=BAND, pre=150, nxt=20)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
def test_band_varlen(dtype):
    inp = W.varlen_tnd([0, 700, 1, 257, 513, 0], 8, 2, 128, causal=False, dtype=dtype, seed=3, cfg=33)
    _check(inp, mode=BAND, pre=255, nxt=0)     # sliding window with no look-ahead
    _check(inp, mode=BAND, pre=40, nxt=300)


def test_band_unbounded_equals_causal_bitwise():
    inp = W.varlen_tnd([300, 0, 513], 4, 2, 128, causal=False, dtype=BF, seed=4, cfg=34,
                       mask_mode=W.MASK_CAUSAL_TOPLEFT)
    a = G.run_fwd(inp)
    b = _run(inp, mode=BAND, pre=1 << 40, nxt=0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _random_mask(rng, B, Sq, Skv, rs, bs, p=0.3, full_row=None):
    flat = (rng.random(max(B * bs, Sq * rs)) < p).astype(np.uint8)
    if full_row is not None:
        b, i = full_row
        flat[b * bs + i * rs: b * bs + i * rs + Skv] = 1
    return flat


@pytest.mark.parametrize("dtype", [BF, F16, F32], ids=["bf16", "f16", "f32"])
@pytest.mark.parametrize("aligned", [True, False], ids=["vec16", "bytes"])
@pytest.mark.parametrize("mode", [W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, BAND])
def test_explicit_mask_dense(dtype, aligned, mode):
    rng = np.random.default_rng(7)
    B, Sq, Skv = 2, 300, 390
    rs = 400 if aligned else 397
    bs = Sq * rs + (0 if aligned else 3)
    inp = W.dense_bhsd(B, 2, Sq, 128, causal=False, dtype=dtype, seed=11, cfg=35, Skv=Skv)
    mask = _random_mask(rng, B, Sq, Skv, rs, bs, full_row=(1, 17))
    _check(inp, mode=mode, pre=100, nxt=30, mask=mask, bs=bs, rs=rs)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
def test_explicit_mask_shared_and_all_zero(dtype):
    rng = np.random.default_rng(8)
    inp = W.dense_bhsd(3, 2, 257, 64, causal=False, dtype=dtype, seed=12, cfg=36)
    mask = _random_mask(rng, 1, 257, 257, 272, 0, p=0.5)
    _check(inp, mode=W.MASK_NONE, mask=mask, bs=0, rs=272)
    # an all-zero mask changes nothing: same bits as the unmasked call
    zero = np.zeros(257 * 272, np.uint8)
    a = _run(inp, mode=W.MASK_CAUSAL_TOPLEFT, mask=zero, rs=272)
    inp.mask_mode = W.MASK_CAUSAL_TOPLEFT
    b = G.run_fwd(inp)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", [BF, F32], ids=["bf16", "f32"])
def test_explicit_mask_varlen(dtype):
    rng = np.random.default_rng(9)
    lens = [0, 700, 1, 257, 513]
    inp = W.varlen_tnd(lens, 4, 1, 128, causal=False, dtype=dtype, seed=13, cfg=37)
    rs, bs = 704, 704 * 704
    mask = _random_mask(rng, len(lens), 704, 704, rs, bs, p=0.25, full_row=(3, 5))
    _check(inp, mode=W.MASK_CAUSAL_TOPLEFT, mask=mask, bs=bs, rs=rs)


@pytest.mark.parametrize("Dv", [64, 40, 1])
def test_value_head_size_f32(Dv):
    base = W.dense_bhsd(2, 4, 200, 128, causal=False, dtype=F32, seed=Dv, cfg=38, Hkv=2, Skv=333)
    v = base.v[..., :Dv].contiguous()
    inp = W.AttnInputs(base.q, base.k, v, W.BHSD, W.MASK_CAUSAL_BOTTOMRIGHT, W.F32, 2, 200, 333, 4, 2,
                       128, base.scale)
    _check(inp, mode=W.MASK_CAUSAL_BOTTOMRIGHT, Dv=Dv)
    _check(inp, mode=BAND, pre=30, nxt=70, Dv=Dv)


def test_value_head_size_varlen_f32():
    base = W.varlen_tnd([100, 0, 300], 4, 2, 96, causal=False, dtype=F32, seed=5, cfg=39)
    inp = W.AttnInputs(base.q, base.k, base.v[..., :48].contiguous(), W.TND, W.MASK_NONE, W.F32,
                       base.B, base.Sq, base.Skv, 4, 2, 96, base.scale, cu_q=base.cu_q, cu_kv=base.cu_kv)
    _check(inp, mode=W.MASK_NONE, Dv=48)


def test_band_full_size_sampled():
    """Sliding-window attention (1024 keys back, none ahead) on the 75K-token varlen GQA
    workload: sampled rows against the oracle, every output finite."""
    inp = W.cfg3_varlen_gqa(seed=0)
    out, m, l = _run(inp, mode=BAND, pre=1023, nxt=0)
    rows_h, rows_t = G.sample_rows(inp, 5, n_random=128, edge=32)
    og, mg, lg = G.gather_rows(out, m, l, inp, rows_h, rows_t)
    ref, rm, rl = oracle.attn_fwd_ext_rows(inp.q, inp.k, inp.v, rows_h, rows_t, cu_q=inp.cu_q,
                                           cu_kv=inp.cu_kv, B=inp.B, Sq=inp.Sq, Skv=inp.Skv,
                                           Nq=inp.Nq, Nkv=inp.Nkv, Dqk=inp.D, Dv=inp.D,
                                           scale=inp.scale, mask_mode=BAND, pre_tokens=1023,
                                           next_tokens=0, layout=inp.layout)
    absr = lambda: oracle.attn_fwd_ext_rows(inp.q, inp.k, inp.v.abs(), rows_h, rows_t, cu_q=inp.cu_q,  # noqa: E731
                                            cu_kv=inp.cu_kv, B=inp.B, Sq=inp.Sq, Skv=inp.Skv,
                                            Nq=inp.Nq, Nkv=inp.Nkv, Dqk=inp.D, Dv=inp.D,
                                            scale=inp.scale, mask_mode=BAND, pre_tokens=1023,
                                            next_tokens=0, layout=inp.layout)[0]
    G.check_out(og, ref, inp.dtype, abs_ref=absr)
    G.check_stats(mg, lg, rm, rl)
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("dtype", [BF, F16], ids=["bf16", "f16"])
@pytest.mark.parametrize("mode", [W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, BAND])
def test_value_head_size_tensor_cores(dtype, mode):
    """Dqk = 128, Dv = 64 on the tcgen05 path (qD == kD >= vD)."""
    base = W.dense_bhsd(2, 4, 300, 128, causal=False, dtype=dtype, seed=2, cfg=41, Hkv=2, Skv=333)
    inp = W.AttnInputs(base.q, base.k, base.v[..., :64].contiguous(), W.BHSD, mode, W.dtype_code(dtype),
                       2, 300, 333, 4, 2, 128, base.scale)
    _check(inp, mode=mode, pre=90, nxt=40, Dv=64)


def test_value_head_size_tensor_cores_varlen_masked():
    rng = np.random.default_rng(10)
    base = W.varlen_tnd([0, 700, 1, 257], 8, 2, 128, causal=False, dtype=BF, seed=6, cfg=42)
    inp = W.AttnInputs(base.q, base.k, base.v[..., :64].contiguous(), W.TND, W.MASK_CAUSAL_TOPLEFT,
                       W.BF16, base.B, base.Sq, base.Skv, 8, 2, 128, base.scale, cu_q=base.cu_q,
                       cu_kv=base.cu_kv)
    rs, bs = 704, 704 * 704
    mask = _random_mask(rng, 4, 704, 704, rs, bs, p=0.2)
    _check(inp, mode=W.MASK_CAUSAL_TOPLEFT, mask=mask, bs=bs, rs=rs, Dv=64)


def test_tensor_core_path_rejects_other_value_sizes():
    inp = W.dense_bhsd(1, 2, 64, 128, causal=False, dtype=BF, seed=1, cfg=40)
    for Dv in (32, 96):
        with pytest.raises(sdpa.AttnError) as e:
            _run(inp, mode=W.MASK_NONE, Dv=Dv)
        assert e.value.status == sdpa.ATTN_ERR_UNSUPPORTED


def test_causal_attention_from_band_masked_key_chunks():
    """Causal attention over 512 keys assembled from 4 chunks of 128 keys, as a ring of devices
    would: chunk c sees key j' (its own index) iff j' <= i - 128c, a band with unbounded
    look-back and look-ahead -128c. Each chunk's result (with rows that see none of its keys
    giving out 0, max -inf, sum 0) is merged in turn; the end result equals causal attention."""
    B, N, S, D, L = 1, 2, 512, 128, 128
    full = W.dense_bhsd(B, N, S, D, causal=True, dtype=BF, seed=7, cfg=43)
    acc = None
    for c in range(S // L):
        kc = full.k[:, :, c * L:(c + 1) * L].contiguous()
        vc = full.v[:, :, c * L:(c + 1) * L].contiguous()
        chunk = W.AttnInputs(full.q, kc, vc, W.BHSD, W.MASK_NONE, W.BF16, B, S, L, N, N, D, full.scale)
        out, m, l = _run(chunk, mode=BAND, pre=1 << 40, nxt=-c * L)
        part = [out.permute(2, 0, 1, 3).reshape(S, B, N * D).contiguous().cuda(),
                m.unsqueeze(-1).expand(B, N, S, 8).contiguous().cuda(),
                l.unsqueeze(-1).expand(B, N, S, 8).contiguous().cuda()]
        if acc is None:
            acc = part
            continue
        sdpa.attn_merge(acc[0], acc[1], acc[2], *part, S=S, B=B, N=N, D=D, dtype=W.BF16,
                        out=acc[0], out_max=acc[1], out_sum=acc[2])
        assert sdpa.attn_get_last_error() == 0
    got = acc[0].cpu().reshape(S, B, N, D).permute(1, 2, 0, 3)
    ref, rm, rl = G.oracle_fwd(full)
    G.check_out(G.f64(got), ref, W.BF16, "causal from chunks", abs_ref=lambda: G.oracle_abs_fwd(full))
    G.check_stats(acc[1][..., 0].cpu().numpy(), acc[2][..., 0].cpu().numpy(), rm, rl, "causal stats")


# ---- the two forms of a work item of the bf16 kernel, across GQA group sizes --------------------
# With an even number of query heads per KV head an item is the same 128 rows of two query heads
# of one group; otherwise it is 256 consecutive rows of one head. Both forms, on a packed batch
# with ragged and empty sequences, for the plain, causal, band and explicit-mask paths.
GROUPS = [(2, 1), (6, 2), (8, 2), (16, 2), (5, 5)]
GROUP_IDS = ["group2", "group3", "group4", "group8", "mha"]


@pytest.mark.parametrize("Nq,Nkv", GROUPS, ids=GROUP_IDS)
@pytest.mark.parametrize("mode", [W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, BAND], ids=["full", "causal", "band"])
def test_item_forms_across_groups(Nq, Nkv, mode):
    inp = W.varlen_tnd([300, 0, 129, 520], Nq, Nkv, 128, causal=False, dtype=BF, seed=Nq * 10 + Nkv, cfg=41)
    _check(inp, mode=mode, pre=200, nxt=0)


@pytest.mark.parametrize("Nq,Nkv", [(8, 2), (6, 2)], ids=["group4", "group3"])
def test_item_forms_with_explicit_mask(Nq, Nkv):
    inp = W.varlen_tnd([300, 129, 520], Nq, Nkv, 128, causal=False, dtype=BF, seed=Nq + 7 * Nkv, cfg=42)
    rng = np.random.default_rng(Nq * Nkv)
    rs, bs = 528, 528 * 528
    mask = _random_mask(rng, inp.B, 528, 528, rs, bs, p=0.3, full_row=(1, 7))
    _check(inp, mode=W.MASK_CAUSAL_TOPLEFT, mask=mask, bs=bs, rs=rs)
