"""attn_fwd_accumulate: attention over a key range split into chunks, folded chunk by chunk into
one accumulator, equals attention over the whole range (float64 oracle), in both layouts and
all dtypes; and agrees with the two-step path attn_fwd + attn_merge."""
import numpy as np
import pytest
import torch

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _chunks_bhsd(inp, n):
    c = inp.Skv // n
    return [(inp.k[:, :, i * c:(i + 1) * c].contiguous(), inp.v[:, :, i * c:(i + 1) * c].contiguous(), c)
            for i in range(n)]


def _accumulate_bhsd(inp, n_chunks):
    B, N, S, D = inp.B, inp.Nq, inp.Sq, inp.D
    q = inp.q.cuda()
    acc = G.Guarded((S, B, N * D), inp.q.dtype)
    am = G.Guarded((B, N, S, 8), torch.float32)
    al = G.Guarded((B, N, S, 8), torch.float32)
    for idx, (k, v, c) in enumerate(_chunks_bhsd(inp, n_chunks)):
        sdpa.attn_fwd_accumulate(q, k.cuda(), v.cuda(), B=B, Sq=S, Skv=c, Nq=N, Nkv=inp.Nkv, D=D,
                                 scale=inp.scale, mask_mode=W.MASK_NONE, dtype=inp.dtype,
                                 layout=W.BHSD, first=idx == 0, acc_out=acc.t, acc_max=am.t,
                                 acc_sum=al.t)
    assert sdpa.attn_get_last_error() == 0
    for g in (acc, am, al):
        g.check("accumulator")
    return acc.t.cpu(), am.t.cpu(), al.t.cpu()


@pytest.mark.parametrize("tdt", [torch.bfloat16, torch.float16, torch.float32], ids=["bf16", "f16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
def test_bhsd_chunks_equal_full(tdt, D):
    inp = W.dense_bhsd(2, 4, 300, D, causal=False, dtype=tdt, seed=D, cfg=31, Hkv=2, Skv=1024)
    acc, am, al = _accumulate_bhsd(inp, 4)
    ref, rm, rl = G.oracle_fwd(inp)
    out = acc.reshape(inp.Sq, inp.B, inp.Nq, D).permute(1, 2, 0, 3)
    G.check_out(G.f64(out), ref, inp.dtype, "accumulated out", abs_ref=lambda: G.oracle_abs_fwd(inp))
    for lane in (0, 7):
        G.check_stats(am[..., lane].numpy(), al[..., lane].numpy(), rm, rl, "accumulated stats")


def test_first_chunk_equals_plain_forward():
    inp = W.dense_bhsd(1, 2, 200, 128, causal=False, dtype=torch.bfloat16, seed=3, cfg=32)
    acc, am, al = _accumulate_bhsd(inp, 1)
    out, m, l = G.run_fwd(inp)
    assert torch.equal(acc.reshape(200, 1, 2, 128).permute(1, 2, 0, 3), out)
    assert torch.equal(am[..., 3], m) and torch.equal(al[..., 5], l)


def test_fused_agrees_with_two_step_merge():
    inp = W.dense_bhsd(2, 4, 256, 128, causal=False, dtype=torch.bfloat16, seed=4, cfg=33, Skv=512)
    acc, am, al = _accumulate_bhsd(inp, 2)
    # two-step: attn_fwd per chunk (rounded to bf16), permute to SBH, attn_merge
    parts = []
    for k, v, c in _chunks_bhsd(inp, 2):
        sub = W.AttnInputs(inp.q, k, v, W.BHSD, W.MASK_NONE, W.BF16, 2, 256, c, 4, 4, 128, inp.scale)
        o, m, l = G.run_fwd(sub)
        parts.append([o.permute(2, 0, 1, 3).reshape(256, 2, 512).contiguous().cuda(),
                      m.unsqueeze(-1).expand(2, 4, 256, 8).contiguous().cuda(),
                      l.unsqueeze(-1).expand(2, 4, 256, 8).contiguous().cuda()])
    sdpa.attn_merge(*parts[0], *parts[1], S=256, B=2, N=4, D=128, dtype=W.BF16,
                    out=parts[0][0], out_max=parts[0][1], out_sum=parts[0][2])
    two = parts[0][0].cpu().to(torch.float64)
    # both are within the bf16 rule of the exact result; they differ by at most two roundings
    assert torch.max(torch.abs(acc.to(torch.float64) - two)).item() <= 2e-2
    assert torch.allclose(am, parts[0][1].cpu()) and torch.allclose(al, parts[0][2].cpu(), rtol=1e-5)


@pytest.mark.parametrize("tdt", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_tnd_chunks_equal_full(tdt):
    lens = [300, 0, 129, 513]
    inp = W.varlen_tnd(lens, 8, 2, 128, causal=False, dtype=tdt, seed=6, cfg=34)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    T, N, D = inp.Sq, inp.Nq, inp.D
    q = inp.q.cuda()
    cq = torch.from_numpy(inp.cu_q).cuda()
    acc_g = G.Guarded((T, N * D), tdt)
    am_g = G.Guarded((T, N, 8), torch.float32)
    al_g = G.Guarded((T, N, 8), torch.float32)
    acc, am, al = acc_g.t, am_g.t, al_g.t
    for part in range(3):  # every sequence's keys split in three, some chunks empty
        idx, lk = [], []
        for s0, L in zip(starts, lens):
            a, b = part * L // 3, (part + 1) * L // 3
            idx.extend(range(s0 + a, s0 + b))
            lk.append(b - a)
        idx = torch.tensor(idx, dtype=torch.int64)
        ck = torch.from_numpy(W.cu_seqlens_from_lengths(lk)).cuda()
        sdpa.attn_fwd_accumulate(q, inp.k[idx].cuda(), inp.v[idx].cuda(), cu_seqlens_q=cq, cu_seqlens_kv=ck,
                                 B=len(lens), Sq=T, Skv=int(sum(lk)), Nq=N, Nkv=inp.Nkv, D=D, scale=inp.scale,
                                 mask_mode=W.MASK_NONE, dtype=inp.dtype, layout=W.TND, first=part == 0,
                                 acc_out=acc, acc_max=am, acc_sum=al)
    assert sdpa.attn_get_last_error() == 0
    for g in (acc_g, am_g, al_g):
        g.check("TND accumulator")
    ref, rm, rl = G.oracle_fwd(inp)
    G.check_out(G.f64(acc.cpu().reshape(T, N, D)), ref, inp.dtype, "accumulated TND out",
                abs_ref=lambda: G.oracle_abs_fwd(inp))
    G.check_stats(am[..., 0].cpu().numpy(), al[..., 0].cpu().numpy(), rm, rl, "accumulated TND stats")


def test_ring_cfg5_full_size_sampled():
    """The ring-attention configuration (B=4, N=32, S=8192, D=128, keys in 4 chunks of 2048),
    fused: sampled rows against the oracle."""
    inp = W.dense_bhsd(4, 32, 8192, 128, causal=False, dtype=torch.bfloat16, seed=0, cfg=5)
    acc, am, al = _accumulate_bhsd(inp, 4)
    out = acc.reshape(8192, 4, 32, 128).permute(1, 2, 0, 3)
    rows_h, rows_t = G.sample_rows(inp, 5, n_random=512, edge=8)
    og, mg, lg = G.gather_rows(out, am[..., 0], al[..., 0], inp, rows_h, rows_t)
    ref, rm, rl = G.oracle_rows(inp, rows_h, rows_t)
    G.check_out(og, ref, W.BF16, "ring out", abs_ref=lambda: G.oracle_abs_rows(inp, rows_h, rows_t))
    G.check_stats(mg, lg, rm, rl, "ring stats")
