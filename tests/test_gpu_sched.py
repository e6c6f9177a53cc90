"""The persistent attn_fwd grid's item hand-out, through the C ABI.

Each block of the forward kernel takes 256-row items one after another. It draws them from a
counter slot that the library gives each stream, and it divides them statically when there is no
slot, as when the launch is captured into a CUDA graph. Whichever block computes an item, the
item's arithmetic is the same, so every way of handing the items out must give bit-identical
outputs and statistics. These tests run two calls concurrently on two streams (two slots in use
at once), replay a captured graph (static division), and make many launches in a row on one
stream (the slot is reset by each launch's last block). They compare each result with one eager
call on the default stream, and that call once with the float64 oracle.
"""
import pytest
import torch

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


class _Call:
    """One attn_fwd problem with resident inputs; run() writes fresh output tensors."""

    def __init__(self, inp):
        self.inp = inp
        self.q, self.k, self.v = (t.cuda() for t in (inp.q, inp.k, inp.v))
        self.cq = torch.from_numpy(inp.cu_q).cuda() if inp.cu_q is not None else None
        self.ck = torch.from_numpy(inp.cu_kv).cuda() if inp.cu_kv is not None else None
        self.shape = (inp.Sq, inp.Nq) if inp.layout == W.TND else (inp.B, inp.Nq, inp.Sq)

    def outputs(self):
        return (torch.full_like(self.q, float("nan")), torch.full(self.shape, float("nan"), device="cuda"),
                torch.full(self.shape, float("nan"), device="cuda"))

    def run(self, out, m, l, stream=None):
        i = self.inp
        sdpa.attn_fwd(self.q, self.k, self.v, cu_seqlens_q=self.cq, cu_seqlens_kv=self.ck, B=i.B, Sq=i.Sq,
                      Skv=i.Skv, Nq=i.Nq, Nkv=i.Nkv, D=i.D, scale=i.scale, mask_mode=i.mask_mode,
                      dtype=i.dtype, layout=i.layout, out=out, softmax_max=m, softmax_sum=l, stream=stream)


def _same(a, b, what):
    for x, y, name in zip(a, b, ("out", "max", "sum")):
        assert torch.equal(x.view(torch.int16) if x.dtype == BF else x, y.view(torch.int16) if y.dtype == BF else y), \
            f"{what}: {name} differs from the eager call"


@pytest.fixture(scope="module")
def calls():
    a = _Call(W.cfg3_varlen_gqa(seed=1, max_len=1536))
    b = _Call(W.dense_bhsd(2, 8, 700, 128, causal=True, dtype=BF, seed=5, cfg=12))
    refs = []
    for c in (a, b):
        o = c.outputs()
        c.run(*o)
        torch.cuda.synchronize()
        assert sdpa.attn_get_last_error() == 0
        refs.append(o)
    # the eager result of the dense call is itself checked against the oracle
    out, m, l = refs[1]
    ref, rm, rl = G.oracle_fwd(b.inp)
    G.check_out(G.f64(out.cpu()), ref, b.inp.dtype, "eager dense call", abs_ref=lambda: G.oracle_abs_fwd(b.inp))
    G.check_stats(m.cpu().numpy(), l.cpu().numpy(), rm, rl)
    return (a, b), refs


def test_two_streams_at_once_match_the_eager_calls(calls):
    (a, b), (ra, rb) = calls
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(4):
        oa, ob = a.outputs(), b.outputs()
        torch.cuda.synchronize()
        a.run(*oa, stream=s1)
        b.run(*ob, stream=s2)
        outs.append((oa, ob))
    torch.cuda.synchronize()
    assert sdpa.attn_get_last_error() == 0
    for oa, ob in outs:
        _same(oa, ra, "varlen call on stream 1")
        _same(ob, rb, "dense call on stream 2")


def test_graph_replay_matches_the_eager_call(calls):
    (a, _), (ra, _) = calls
    o = a.outputs()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        a.run(*o)  # first call of the instantiation outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    for t in o:
        t.fill_(float("nan"))
    with torch.cuda.graph(g):
        a.run(*o)
    for _ in range(3):
        for t in o:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert sdpa.attn_get_last_error() == 0
        _same(o, ra, "graph replay")
    del g


def test_many_launches_in_a_row_on_one_stream(calls):
    (_, b), (_, rb) = calls
    outs = [b.outputs() for _ in range(40)]
    for o in outs:
        b.run(*o)
    torch.cuda.synchronize()
    assert sdpa.attn_get_last_error() == 0
    for o in outs:
        _same(o, rb, "launch in a row")
