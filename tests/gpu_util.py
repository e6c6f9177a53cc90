"""Helpers for the GPU parity tests: run the C-ABI calls on seeded inputs and compare with the
float64 oracle under the stated tolerances.

Tolerances (written here, used by every parity test):
  * bf16 (and fp16) outputs: |gpu - exact| <= max(1e-2, one ulp of the exact value). The exact
    (float64) value is compared directly; a correctly rounded bf16 result is within half an
    ulp of it, and for |o| >= 4 half an ulp is already 1.6e-2, above 1e-2.
  * fp32 outputs: |gpu - exact| <= 1e-5.
  * softmax max: |gpu - exact| <= 1e-3 * max(1, |exact|); softmax sum: relative 1e-3. Rows that
    see no key must give max = -inf and sum = 0 on both sides.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W

BF16_ABS = 1e-2
F32_ABS = 1e-5
STAT_REL = 1e-3


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.exp2(e - 7)


def f16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -14)))
    return np.exp2(e - 10)


def check_out(gpu: np.ndarray, ref: np.ndarray, dtype: int, what: str = "out") -> dict:
    gpu = gpu.astype(np.float64)
    err = np.abs(gpu - ref)
    if dtype == W.BF16:
        tol = np.maximum(BF16_ABS, bf16_ulp(ref))
    elif dtype == W.F16:
        tol = np.maximum(BF16_ABS, f16_ulp(ref))
    else:
        tol = np.full_like(ref, F32_ABS)
    bad = ~(err <= tol)
    info = {"max_abs": float(err.max()) if err.size else 0.0,
            "n_over_1e-2": int((err > 1e-2).sum()), "n_bad": int(bad.sum()), "n": int(err.size)}
    assert not bad.any(), f"{what}: {info}; first bad at {np.argwhere(bad)[:5].tolist()}"
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


def to_dev(inp: W.AttnInputs, device="cuda"):
    q, k, v = (t.to(device).contiguous() for t in (inp.q, inp.k, inp.v))
    cq = ck = None
    if inp.layout == W.TND:
        cq = torch.from_numpy(np.asarray(inp.cu_q, np.int32)).to(device)
        ck = torch.from_numpy(np.asarray(inp.cu_kv, np.int32)).to(device)
    return q, k, v, cq, ck


def run_fwd(inp: W.AttnInputs, stats: bool = True, device="cuda"):
    """Run attn_fwd on the device. Returns (out, softmax_max, softmax_sum) as CPU tensors."""
    q, k, v, cq, ck = to_dev(inp, device)
    out = torch.empty_like(q)
    shape = (inp.B, inp.Nq, inp.Sq) if inp.layout == W.BHSD else (inp.Sq, inp.Nq)
    m = torch.empty(shape, dtype=torch.float32, device=device) if stats else None
    l = torch.empty(shape, dtype=torch.float32, device=device) if stats else None
    sdpa.attn_fwd(q, k, v, cu_seqlens_q=cq, cu_seqlens_kv=ck, B=inp.B, Sq=inp.Sq, Skv=inp.Skv,
                  Nq=inp.Nq, Nkv=inp.Nkv, D=inp.D, scale=inp.scale, mask_mode=inp.mask_mode,
                  dtype=inp.dtype, layout=inp.layout, out=out, softmax_max=m, softmax_sum=l)
    st = sdpa.attn_get_last_error()
    assert st == 0, f"device status {st}"
    return out.cpu(), (m.cpu() if stats else None), (l.cpu() if stats else None)


def oracle_fwd(inp: W.AttnInputs):
    return oracle.attn_fwd(inp.q, inp.k, inp.v, cu_q=inp.cu_q, cu_kv=inp.cu_kv, B=inp.B, Sq=inp.Sq,
                           Skv=inp.Skv, Nq=inp.Nq, Nkv=inp.Nkv, D=inp.D, scale=inp.scale,
                           mask_mode=inp.mask_mode, layout=inp.layout)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def sample_rows(inp: W.AttnInputs, seed: int, n_random: int = 256, edge: int = 64, heads=None):
    """Row sample for checks at full sizes: first and last `edge` rows of every sequence and
    `n_random` random rows, for the listed heads (default: first, middle, last)."""
    rng = np.random.default_rng(seed)
    heads = heads if heads is not None else sorted({0, inp.Nq // 2, inp.Nq - 1})
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
    if total > 0:
        toks.update(rng.integers(0, total, size=n_random).tolist())
    toks = sorted(toks)
    rows_t = np.array([t for h in heads for t in toks], dtype=np.int64)
    rows_h = np.array([h for h in heads for _ in toks], dtype=np.int32)
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
