"""Helpers for the GPU parity tests: run the C-ABI calls on seeded inputs and compare with the
float64 oracle under the stated tolerances, with guard regions around every output.

Tolerances (written here, used by every parity test):
  * bf16 and fp16 outputs: |gpu - exact| <= max(1e-2, ulp(exact) / 2 + c * A), where ulp(exact)/2
    is the output's own rounding and c * A bounds what the kernel's arithmetic adds before it:
    A = sum_j w_j |v_j| (the softmax-weighted mean of |v| in that element's column, which the
    oracle gives when it is handed |V|) and c = u_P + 2^-13 + 2^-12, with u_P (2^-8 for bf16,
    2^-11 for fp16) the relative rounding of the probabilities P the tensor cores multiply with V
    (a 16-bit operand), 2^-13 the relative error of the kernel's exp2 (its polynomial's is
    7.5e-5), and 2^-12 the fp32 accumulation over at most 65,536 keys (a rounding of 2^-24 per
    16-key product step); each bounds |sum_j w_j e_j v_j| <= e * A. The bound exceeds 1e-2 only
    in rows dominated by a few large |v| (few visible keys, or |exact| >= 4 where bf16's own
    spacing is 2^-5); A is computed only for elements whose error is above 1e-2, and every such
    element is counted in the report.
  * fp32 outputs: |gpu - exact| <= 1e-5.
  * softmax max: |gpu - exact| <= 1e-3 * max(1, |exact|); softmax sum: relative 1e-3. Rows that
    see no key must give max = -inf and sum = 0 on both sides.
  * merge outputs in bf16/fp16 are checked against the single rounding of the exact value
    (check_rne): bit for bit, or the neighbouring value only where the exact value lies within
    the fp32 arithmetic's error of a rounding midpoint.

Every check records its largest error and the count of elements above 1e-2 (REPORT); the
session summary prints them and, with ATTN_PARITY_REPORT=<path>, writes them as JSON.

Guard regions: outputs are allocated inside a larger buffer with GUARD_BYTES before and after
and the whole buffer is filled with a NaN bit pattern (0xFFC1 per 16 bits); after the call the
guards must still hold it bit for bit, so a store past either end of an output is caught, and
an element the call should have written but did not fails the comparison as NaN.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W

BF16_ABS = 1e-2
F32_ABS = 1e-5
STAT_REL = 1e-3
BIG = 4.0                                   # |exact| from which bf16's own rounding can pass 1e-2
UNIT_P = {W.BF16: 2.0 ** -8, W.F16: 2.0 ** -11}
EXP2_REL = 2.0 ** -13
ACC_REL = 2.0 ** -12
GUARD_BYTES = 4096
SENTINEL16 = -63                            # 0xFFC1: NaN as bf16, fp16 and (twice) fp32

REPORT: list = []


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.exp2(e - 7)


def f16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -14)))
    return np.exp2(e - 10)


def _record(what: str, dtype: int, err: np.ndarray, ref: np.ndarray, extra: dict) -> dict:
    small = np.abs(ref) < BIG
    info = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "what": what,
            "dtype": {W.BF16: "bf16", W.F16: "f16", W.F32: "f32"}.get(dtype, str(dtype)),
            "n": int(err.size), "max_abs": float(np.nanmax(err)) if err.size else 0.0,
            "max_abs_below_4": float(np.nanmax(err[small])) if small.any() else 0.0,
            "n_over_1e-2": int((err > 1e-2).sum()), "n_at_or_above_4": int((~small).sum())}
    info.update(extra)
    REPORT.append(info)
    return info


def check_out(gpu: np.ndarray, ref: np.ndarray, dtype: int, what: str = "out", abs_ref=None) -> dict:
    """Element by element against the exact (float64) result under the rule above. `abs_ref`
    is A (same shape as ref), or a callable returning it; it is needed only where |exact| >= 4."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    extra = {}
    if dtype in (W.BF16, W.F16):
        tol = np.full(ref.shape, BF16_ABS)
        over = err > BF16_ABS
        if over.any():
            A = abs_ref() if callable(abs_ref) else abs_ref
            assert A is not None, f"{what}: {int(over.sum())} elements above 1e-2 and no A to bound them"
            A = np.asarray(A, np.float64)
            half = (bf16_ulp(ref[over]) if dtype == W.BF16 else f16_ulp(ref[over])) / 2
            bound = half + (UNIT_P[dtype] + EXP2_REL + ACC_REL) * A[over]
            tol[over] = np.maximum(BF16_ABS, bound)
            extra["max_err_over_bound_above_1e-2"] = float(np.max(err[over] / bound))
    else:
        tol = np.full(ref.shape, F32_ABS)
    bad = ~(err <= tol)
    info = _record(what, dtype, err, ref, extra)
    info["n_bad"] = int(bad.sum())
    assert not bad.any(), f"{what}: {info}; first bad at {np.argwhere(bad)[:5].tolist()}"
    return info


def check_rne(gpu: torch.Tensor, ref: np.ndarray, dtype: int, eps: np.ndarray, what: str = "out") -> dict:
    """A 16-bit result computed in fp32 and rounded once: its value must be the rounding of a
    value within eps of the exact one (eps bounding the fp32 arithmetic's error), that is, lie
    between the roundings of exact - eps and exact + eps. Where no rounding boundary falls in
    that window the two are the same value and the result must be bit for bit the rounding of
    the exact value."""
    rnd = oracle.round_bf16 if dtype == W.BF16 else oracle.round_f16
    tdt = torch.bfloat16 if dtype == W.BF16 else torch.float16
    ref = np.asarray(ref, np.float64)

    def value(bits):
        return torch.from_numpy(bits.view(np.int16)).view(tdt).to(torch.float64).numpy()

    got_bits = gpu.contiguous().view(torch.int16).numpy().view(np.uint16)
    want, lo, hi = rnd(ref), rnd(ref - eps), rnd(ref + eps)
    got, lo_v, hi_v = value(got_bits), value(lo), value(hi)
    ok = (got_bits == want) | ((got >= lo_v) & (got <= hi_v))
    info = _record(what, dtype, np.abs(got - ref), ref, {
        "n_not_bit_equal_to_rne": int((got_bits != want).sum()),
        "n_window_holds_a_boundary": int((lo != hi).sum())})
    assert ok.all(), f"{what}: {int((~ok).sum())} elements are not the rounding of a value within eps"
    return info


def check_stats(m_gpu, l_gpu, m_ref, l_ref, what: str = "stats") -> None:
    m_gpu = np.asarray(m_gpu, np.float64)
    l_gpu = np.asarray(l_gpu, np.float64)
    empty = np.isneginf(m_ref)
    assert np.array_equal(np.isneginf(m_gpu), empty), f"{what}: -inf pattern differs"
    assert np.all(l_gpu[empty] == 0.0), f"{what}: empty rows need sum 0"
    full = ~empty
    dm = np.abs(m_gpu[full] - m_ref[full])
    assert np.all(dm <= STAT_REL * np.maximum(1.0, np.abs(m_ref[full]))), f"{what}: max err {dm.max()}"
    dl = np.abs(l_gpu[full] - l_ref[full]) / l_ref[full]
    assert np.all(dl <= STAT_REL), f"{what}: sum rel err {dl.max()}"


# ---- guarded outputs ---------------------------------------------------------------------------
class Guarded:
    """An output tensor inside a buffer with GUARD_BYTES of guard on each side, all filled with
    the NaN pattern; check() asserts that both guards are untouched."""

    def __init__(self, shape, dtype, device="cuda", fill=True):
        n = int(np.prod(shape)) if len(shape) else 1
        es = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // es
        self.buf = torch.empty(self.g + n + self.g, dtype=dtype, device=device)
        self.buf.view(torch.int16).fill_(SENTINEL16)
        self.t = self.buf[self.g:self.g + n].view(tuple(shape))
        if not fill:
            self.t.zero_()

    def check(self, what: str = "output") -> None:
        raw = self.buf.view(torch.int16)
        gb = GUARD_BYTES // 2
        head, tail = raw[:gb], raw[raw.numel() - gb:]
        assert bool(torch.all(head == SENTINEL16)) and bool(torch.all(tail == SENTINEL16)), \
            f"{what}: a store landed in the guard region outside the output"


def guarded_like(t: torch.Tensor) -> "Guarded":
    return Guarded(tuple(t.shape), t.dtype, t.device)


def guarded_copy(t: torch.Tensor, device="cuda") -> "Guarded":
    """A guarded device copy of t (for outputs that also start as inputs: in-place merges,
    accumulators)."""
    g = Guarded(tuple(t.shape), t.dtype, device)
    g.t.copy_(t.to(device))
    return g


def to_dev(inp: W.AttnInputs, device="cuda"):
    q, k, v = (t.to(device).contiguous() for t in (inp.q, inp.k, inp.v))
    cq = ck = None
    if inp.layout == W.TND:
        cq = torch.from_numpy(np.asarray(inp.cu_q, np.int32)).to(device)
        ck = torch.from_numpy(np.asarray(inp.cu_kv, np.int32)).to(device)
    return q, k, v, cq, ck


def run_fwd(inp: W.AttnInputs, stats: bool = True, device="cuda"):
    """Run attn_fwd on the device into guarded outputs. Returns (out, softmax_max, softmax_sum)
    as CPU tensors."""
    q, k, v, cq, ck = to_dev(inp, device)
    out = Guarded(tuple(q.shape), q.dtype, device)
    shape = (inp.B, inp.Nq, inp.Sq) if inp.layout == W.BHSD else (inp.Sq, inp.Nq)
    m = Guarded(shape, torch.float32, device) if stats else None
    l = Guarded(shape, torch.float32, device) if stats else None
    sdpa.attn_fwd(q, k, v, cu_seqlens_q=cq, cu_seqlens_kv=ck, B=inp.B, Sq=inp.Sq, Skv=inp.Skv,
                  Nq=inp.Nq, Nkv=inp.Nkv, D=inp.D, scale=inp.scale, mask_mode=inp.mask_mode,
                  dtype=inp.dtype, layout=inp.layout, out=out.t,
                  softmax_max=m.t if stats else None, softmax_sum=l.t if stats else None)
    st = sdpa.attn_get_last_error()
    assert st == 0, f"device status {st}"
    for g, name in ((out, "out"), (m, "softmax_max"), (l, "softmax_sum")):
        if g is not None:
            g.check(name)
    return out.t.cpu(), (m.t.cpu() if stats else None), (l.t.cpu() if stats else None)


def abs_v(inp: W.AttnInputs) -> W.AttnInputs:
    """The same inputs with V replaced by |V| (exact in every input type): the oracle then gives
    A = sum_j w_j |v_j| for each output element, which the rule above needs where |exact| >= 4."""
    import dataclasses
    return dataclasses.replace(inp, v=inp.v.abs())


def oracle_fwd(inp: W.AttnInputs):
    return oracle.attn_fwd(inp.q, inp.k, inp.v, cu_q=inp.cu_q, cu_kv=inp.cu_kv, B=inp.B, Sq=inp.Sq,
                           Skv=inp.Skv, Nq=inp.Nq, Nkv=inp.Nkv, D=inp.D, scale=inp.scale,
                           mask_mode=inp.mask_mode, layout=inp.layout)


def oracle_abs_fwd(inp: W.AttnInputs) -> np.ndarray:
    return oracle_fwd(abs_v(inp))[0]


def f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def sample_rows(inp: W.AttnInputs, seed: int, n_random: int = 512, edge: int = 32, heads=None):
    """Row sample for checks at full sizes, over every query head (or the listed heads): for
    each head, the first and last `edge` rows of every sequence, plus `n_random` random
    (head, token) rows spread over the heads."""
    rng = np.random.default_rng(seed)
    heads = list(range(inp.Nq)) if heads is None else list(heads)
    if inp.layout == W.BHSD:
        starts = [b * inp.Sq for b in range(inp.B)]
        lens = [inp.Sq] * inp.B
        total = inp.B * inp.Sq
    else:
        lens = W.lengths_from_cu_seqlens(inp.cu_q).tolist()
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).tolist()
        total = inp.Sq
    toks = set()
    for s0, ln in zip(starts, lens):
        for i in list(range(min(edge, ln))) + list(range(max(0, ln - edge), ln)):
            toks.add(s0 + i)
    pairs = {(h, t) for h in heads for t in toks}
    if total > 0:
        hs = rng.choice(np.asarray(heads), size=n_random)
        ts = rng.integers(0, total, size=n_random)
        pairs.update(zip(hs.tolist(), ts.tolist()))
    pairs = sorted(pairs)
    rows_h = np.array([h for h, _ in pairs], dtype=np.int32)
    rows_t = np.array([t for _, t in pairs], dtype=np.int64)
    return rows_h, rows_t


def gather_rows(out: torch.Tensor, m, l, inp: W.AttnInputs, rows_h, rows_t):
    """Pick sampled rows out of full GPU outputs (layout-aware)."""
    o = f64(out)
    if inp.layout == W.BHSD:
        b, i = rows_t // inp.Sq, rows_t % inp.Sq
        og = o[b, rows_h, i]
        mg = None if m is None else m.numpy()[b, rows_h, i]
        lg = None if l is None else l.numpy()[b, rows_h, i]
    else:
        og = o[rows_t, rows_h]
        mg = None if m is None else m.numpy()[rows_t, rows_h]
        lg = None if l is None else l.numpy()[rows_t, rows_h]
    return og, mg, lg


def oracle_rows(inp: W.AttnInputs, rows_h, rows_t):
    return oracle.attn_fwd_rows(inp.q, inp.k, inp.v, rows_h, rows_t, cu_q=inp.cu_q, cu_kv=inp.cu_kv,
                                B=inp.B, Sq=inp.Sq, Skv=inp.Skv, Nq=inp.Nq, Nkv=inp.Nkv, D=inp.D,
                                scale=inp.scale, mask_mode=inp.mask_mode, layout=inp.layout)


def oracle_abs_rows(inp: W.AttnInputs, rows_h, rows_t) -> np.ndarray:
    """A = sum_j w_j |v_j| for the sampled rows (the oracle on |V|)."""
    return oracle_rows(abs_v(inp), rows_h, rows_t)[0]
