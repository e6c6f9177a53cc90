"""float64 CPU oracle for attention forward, CSR-sparse attention and the partial-result merge.

TEST INFRASTRUCTURE, NOT THE PRODUCT. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code with the CUDA
path (``scaled_dot_product_16_b200``) and never imports it; inputs come from the seeded
generators, which hold none of the method's arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain C, float64, OpenMP over independent rows),
compiled here with gcc into ``_liboracle.so``. Each C function states the passage it follows.
This module only marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None

F64, F32, BF16 = 0, 1, 2
BHSD, TND = 0, 1


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into _liboracle.so (gcc, -O2, OpenMP). Returns the path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_attn_fwd.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, D, I, I, P, P, P]
    lib.oracle_attn_fwd.restype = I
    lib.oracle_attn_fwd_rows.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, D, I, I,
                                         P, P, I64, P, P, P]
    lib.oracle_attn_fwd_rows.restype = I
    lib.oracle_attn_fwd_ext.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, I, D, I, I64, I64,
                                        P, I64, I64, I, P, P, P]
    lib.oracle_attn_fwd_ext.restype = I
    lib.oracle_attn_fwd_ext_rows.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, I, D, I, I64, I64,
                                             P, I64, I64, I, P, P, I64, P, P, P]
    lib.oracle_attn_fwd_ext_rows.restype = I
    lib.oracle_sparse_csr.argtypes = [P, P, P, I, P, P, I, I, I, I, I64, P]
    lib.oracle_sparse_csr.restype = I
    lib.oracle_merge.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.oracle_merge.restype = I
    lib.oracle_round_bf16_array.argtypes = [P, I64, P]
    lib.oracle_round_bf16_array.restype = None
    lib.oracle_round_f16_array.argtypes = [P, I64, P]
    lib.oracle_round_f16_array.restype = None
    return lib


_active = threading.local()


def _load():
    """The library the wrappers call: the built oracle, or a variant bound by ``using``."""
    global _lib
    alt = getattr(_active, "lib", None)
    if alt is not None:
        return alt
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


class using:
    """Context manager that routes this thread's wrapper calls to another compiled copy of
    the oracle (the pin tests use it to check that planted mistakes are caught)."""

    def __init__(self, so_path: str):
        self._lib = _bind(so_path)

    def __enter__(self):
        self._prev = getattr(_active, "lib", None)
        _active.lib = self._lib
        return self

    def __exit__(self, *exc):
        _active.lib = self._prev
        return False


def _elem(x) -> Tuple[np.ndarray, int]:
    """Accept numpy or torch CPU arrays; bf16 torch tensors are passed as raw 16-bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float16:
                return x.numpy().astype(np.float64), F64  # exact widening
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    return np.ascontiguousarray(x, dtype=np.float64), F64


def _same_type(*arrs):
    out = [_elem(a) for a in arrs]
    ets = {e for _, e in out}
    if len(ets) != 1:
        out = [(np.ascontiguousarray(_widen(a, e)), F64) for a, e in out]
    return [a for a, _ in out], out[0][1]


def _widen(a: np.ndarray, et: int) -> np.ndarray:
    if et == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _cu(cu) -> Optional[np.ndarray]:
    return None if cu is None else np.ascontiguousarray(np.asarray(cu), dtype=np.int32)


def attn_fwd(q, k, v, *, cu_q=None, cu_kv=None, B: int, Sq: int, Skv: int, Nq: int, Nkv: int,
             D: int, scale: float, mask_mode: int, layout: int):
    """All rows. Returns (out float64 shaped like q, softmax_max, softmax_sum)."""
    lib = _load()
    (qa, ka, va), et = _same_type(q, k, v)
    cq, ck = _cu(cu_q), _cu(cu_kv)
    if layout == BHSD:
        out = np.zeros((B, Nq, Sq, D))
        m = np.zeros((B, Nq, Sq))
    else:
        out = np.zeros((Sq, Nq, D))
        m = np.zeros((Sq, Nq))
    l = np.zeros_like(m)
    rc = lib.oracle_attn_fwd(_ptr(qa), _ptr(ka), _ptr(va), et, _ptr(cq), _ptr(ck), B, Sq, Skv,
                             Nq, Nkv, D, float(scale), int(mask_mode), int(layout),
                             _ptr(out), _ptr(m), _ptr(l))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd rejected its arguments (code {rc})")
    return out, m, l


def attn_fwd_rows(q, k, v, rows_h, rows_t, *, cu_q=None, cu_kv=None, B: int, Sq: int, Skv: int,
                  Nq: int, Nkv: int, D: int, scale: float, mask_mode: int, layout: int):
    """Selected rows (head rows_h[r], query token rows_t[r]). Returns (out [n,D], max [n], sum [n])."""
    lib = _load()
    (qa, ka, va), et = _same_type(q, k, v)
    cq, ck = _cu(cu_q), _cu(cu_kv)
    rh = np.ascontiguousarray(rows_h, dtype=np.int32)
    rt = np.ascontiguousarray(rows_t, dtype=np.int64)
    n = int(rh.shape[0])
    out = np.zeros((n, D))
    m = np.zeros(n)
    l = np.zeros(n)
    rc = lib.oracle_attn_fwd_rows(_ptr(qa), _ptr(ka), _ptr(va), et, _ptr(cq), _ptr(ck), B, Sq,
                                  Skv, Nq, Nkv, D, float(scale), int(mask_mode), int(layout),
                                  _ptr(rh), _ptr(rt), n, _ptr(out), _ptr(m), _ptr(l))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_rows rejected its arguments (code {rc})")
    return out, m, l


MASK_BAND = 3


def _mask(mask):
    if mask is None:
        return None
    try:
        import torch
        if isinstance(mask, torch.Tensor):
            mask = mask.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(mask, dtype=np.uint8)


def attn_fwd_ext(q, k, v, *, cu_q=None, cu_kv=None, B: int, Sq: int, Skv: int, Nq: int, Nkv: int,
                 Dqk: int, Dv: int, scale: float, mask_mode: int, pre_tokens: int = 0,
                 next_tokens: int = 0, mask=None, mask_bstride: int = 0, mask_rstride: int = 0,
                 layout: int):
    """Masked forward (band limits, explicit uint8 mask with 1 = excluded, value head size Dv).
    Returns (out float64 [.., Nq, Dv] in q's layout, softmax_max, softmax_sum)."""
    lib = _load()
    (qa, ka, va), et = _same_type(q, k, v)
    cq, ck = _cu(cu_q), _cu(cu_kv)
    mk = _mask(mask)
    if layout == BHSD:
        out = np.zeros((B, Nq, Sq, Dv))
        m = np.zeros((B, Nq, Sq))
    else:
        out = np.zeros((Sq, Nq, Dv))
        m = np.zeros((Sq, Nq))
    l = np.zeros_like(m)
    rc = lib.oracle_attn_fwd_ext(_ptr(qa), _ptr(ka), _ptr(va), et, _ptr(cq), _ptr(ck), B, Sq, Skv,
                                 Nq, Nkv, Dqk, Dv, float(scale), int(mask_mode), int(pre_tokens),
                                 int(next_tokens), _ptr(mk), int(mask_bstride), int(mask_rstride),
                                 int(layout), _ptr(out), _ptr(m), _ptr(l))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_ext rejected its arguments (code {rc})")
    return out, m, l


def attn_fwd_ext_rows(q, k, v, rows_h, rows_t, *, cu_q=None, cu_kv=None, B: int, Sq: int,
                      Skv: int, Nq: int, Nkv: int, Dqk: int, Dv: int, scale: float,
                      mask_mode: int, pre_tokens: int = 0, next_tokens: int = 0, mask=None,
                      mask_bstride: int = 0, mask_rstride: int = 0, layout: int):
    """Selected rows of attn_fwd_ext. Returns (out [n, Dv], max [n], sum [n])."""
    lib = _load()
    (qa, ka, va), et = _same_type(q, k, v)
    cq, ck = _cu(cu_q), _cu(cu_kv)
    mk = _mask(mask)
    rh = np.ascontiguousarray(rows_h, dtype=np.int32)
    rt = np.ascontiguousarray(rows_t, dtype=np.int64)
    n = int(rh.shape[0])
    out = np.zeros((n, Dv))
    m = np.zeros(n)
    l = np.zeros(n)
    rc = lib.oracle_attn_fwd_ext_rows(_ptr(qa), _ptr(ka), _ptr(va), et, _ptr(cq), _ptr(ck), B, Sq,
                                      Skv, Nq, Nkv, Dqk, Dv, float(scale), int(mask_mode),
                                      int(pre_tokens), int(next_tokens), _ptr(mk),
                                      int(mask_bstride), int(mask_rstride), int(layout), _ptr(rh),
                                      _ptr(rt), n, _ptr(out), _ptr(m), _ptr(l))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_ext_rows rejected its arguments (code {rc})")
    return out, m, l


def sparse_csr(q, k, v, offset, columns, *, B: int, H: int, S: int, D: int):
    """CSR-sparse attention, scale 1/sqrt(D). Returns out float64 [B,H,S,D]."""
    lib = _load()
    (qa, ka, va), et = _same_type(q, k, v)
    off = np.ascontiguousarray(offset, dtype=np.int32)
    col = np.ascontiguousarray(columns, dtype=np.int32)
    nnz_cap = int(col.shape[-1]) if col.ndim else 0
    out = np.zeros((B, H, S, D))
    rc = lib.oracle_sparse_csr(_ptr(qa), _ptr(ka), _ptr(va), et, _ptr(off), _ptr(col), B, H, S, D,
                               nnz_cap, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_sparse_csr rejected its arguments (code {rc})")
    return out


def merge(prev_out, prev_max, prev_sum, cur_out, cur_max, cur_sum, *, S: int, B: int, N: int, D: int,
          layout: int = BHSD):
    """Ring-attention update. layout BHSD (the page's SBH): out [S,B,N*D], stats [B,N,S,8];
    layout TND: out [T,N*D] with T = S, stats [T,N,8]. Returns (out float64, max, sum)."""
    lib = _load()
    (po, co), et = _same_type(prev_out, cur_out)
    stats = [np.ascontiguousarray(_widen(*_elem(x)), dtype=np.float64)
             for x in (prev_max, prev_sum, cur_max, cur_sum)]
    if layout == BHSD:
        out = np.zeros((S, B, N * D))
        om = np.zeros((B, N, S, 8))
    else:
        out = np.zeros((S, N * D))
        om = np.zeros((S, N, 8))
    osum = np.zeros_like(om)
    rc = lib.oracle_merge(_ptr(po), _ptr(stats[0]), _ptr(stats[1]), _ptr(co), _ptr(stats[2]),
                          _ptr(stats[3]), et, S, B, N, D, int(layout), _ptr(out), _ptr(om),
                          _ptr(osum))
    if rc != 0:
        raise ValueError(f"oracle_merge rejected its arguments (code {rc})")
    return out, om, osum


def round_bf16(x) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); returns raw uint16 patterns."""
    lib = _load()
    xa = np.ascontiguousarray(x, dtype=np.float64)
    out = np.zeros(xa.shape, dtype=np.uint16)
    lib.oracle_round_bf16_array(_ptr(xa), int(xa.size), _ptr(out))
    return out


def round_f16(x) -> np.ndarray:
    """Round float64 values to IEEE float16 (nearest, ties to even); returns raw uint16 patterns."""
    lib = _load()
    xa = np.ascontiguousarray(x, dtype=np.float64)
    out = np.zeros(xa.shape, dtype=np.uint16)
    lib.oracle_round_f16_array(_ptr(xa), int(xa.size), _ptr(out))
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return _widen(np.asarray(bits, dtype=np.uint16), BF16)
