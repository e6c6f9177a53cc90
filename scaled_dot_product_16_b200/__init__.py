"""Python binding of libattn.so: scaled-dot-product attention forward on B200 (sm_100a).

The operations (attn_fwd, attn_fwd_masked, attn_fwd_accumulate, attn_sparse_csr,
attn_sparse_csr_tc, attn_csr_plan_size, attn_csr_plan, attn_sparse_csr_tc_planned, attn_merge,
attn_get_last_error) are the C-ABI calls declared in
``include/attn.h``; the functions here carry the same names and only marshal arguments (tensor
data pointers, sizes, the current CUDA stream) into them. Every step of the computation runs in the library's CUDA kernels.
There is no CPU path: if ``libattn.so`` is missing the first call raises.

PyTorch is used for device memory and streams only: pass CUDA tensors (contiguous, in the
layouts the header states) and preallocated outputs.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

__all__ = [
    "attn_fwd", "attn_fwd_accumulate", "attn_sparse_csr", "attn_merge", "attn_get_last_error", "AttnError",
    "ATTN_BF16", "ATTN_F32", "ATTN_F16", "ATTN_BHSD", "ATTN_TND", "ATTN_MASK_NONE",
    "ATTN_MASK_CAUSAL_TOPLEFT", "ATTN_MASK_CAUSAL_BOTTOMRIGHT", "ATTN_MASK_BAND", "lib_path",
    "load_library", "attn_fwd_masked", "attn_sparse_csr_tc", "attn_csr_plan_size", "attn_csr_plan",
    "attn_sparse_csr_tc_planned", "attn_sparse_csr_tc_noalloc",
]

ATTN_OK, ATTN_ERR_INVALID, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_DATA, ATTN_ERR_TIMEOUT = range(6)
ATTN_BF16, ATTN_F32, ATTN_F16 = 0, 1, 2
ATTN_BHSD, ATTN_TND = 0, 1
ATTN_MASK_NONE, ATTN_MASK_CAUSAL_TOPLEFT, ATTN_MASK_CAUSAL_BOTTOMRIGHT, ATTN_MASK_BAND = 0, 1, 2, 3

_HERE = os.path.dirname(os.path.abspath(__file__))
_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_status_string(status)} (status {status})")


def lib_path() -> str:
    return os.path.join(_HERE, "libattn.so")


def load_library():
    """Load libattn.so (once). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m scaled_dot_product_16_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, I64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, I, P, P, P, P]
        lib.attn_fwd.restype = I
        lib.attn_fwd_accumulate.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, I, I, P, P, P, P]
        lib.attn_fwd_accumulate.restype = I
        lib.attn_fwd_masked.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, I, I64, I64, P, I64,
                                        I64, I, I, P, P, P, P]
        lib.attn_fwd_masked.restype = I
        lib.attn_sparse_csr.argtypes = [P, P, P, P, P, I, I, I, I, I64, P, P]
        lib.attn_sparse_csr_tc.argtypes = [P, P, P, P, P, I, I, I, I, I64, I, P, P]
        lib.attn_sparse_csr_tc.restype = I
        lib.attn_sparse_csr.restype = I
        lib.attn_csr_plan_size.argtypes = [I, I, I, I64, ctypes.POINTER(I64)]
        lib.attn_csr_plan_size.restype = I
        lib.attn_csr_plan.argtypes = [P, P, I, I, I, I64, P, I64, P]
        lib.attn_csr_plan.restype = I
        lib.attn_sparse_csr_tc_planned.argtypes = [P, P, P, P, I64, I, I, I, I, I64, I, P, P]
        lib.attn_sparse_csr_tc_planned.restype = I
        lib.attn_sparse_csr_tc_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I64, I, P, P]
        lib.attn_sparse_csr_tc_noalloc.restype = I
        lib.attn_merge.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, P]
        lib.attn_merge.restype = I
        lib.attn_get_last_error.argtypes = [P, ctypes.POINTER(I)]
        lib.attn_get_last_error.restype = I
        lib.attn_status_string.argtypes = [I]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_abi_version.argtypes = []
        lib.attn_abi_version.restype = I
        _lib = lib
        return lib


def _status_string(status: int) -> str:
    try:
        return load_library().attn_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - only for messages
        return "unknown"


_ELEM = {ATTN_BF16: "bfloat16", ATTN_F32: "float32", ATTN_F16: "float16"}


def _dtype_name(x) -> str:
    return str(getattr(x, "dtype", "")).replace("torch.", "")


def _ptr(x, name: str = "tensor", numel: int = 0, dtype: Optional[str] = None) -> Optional[int]:
    """Device data pointer of a tensor argument (an int is passed through as a raw address and
    None as a null pointer). A tensor must be a dense CUDA tensor on the current device, of
    element type `dtype` (a torch dtype name) when given, holding at least `numel` elements:
    the library reads exactly the sizes it is given, so a smaller or differently typed tensor,
    or one on another GPU, would be read or written out of bounds."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if getattr(x, "is_cuda", True) is False:
        raise ValueError(f"{name} must be on a CUDA device")
    if hasattr(x, "is_contiguous") and not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and _dtype_name(x) != dtype:
        raise ValueError(f"{name} must be {dtype}, got {_dtype_name(x)}")
    if numel > 0 and x.numel() < numel:
        raise ValueError(f"{name} holds {x.numel()} elements; the sizes given need {numel}")
    dev = getattr(x, "device", None)
    if dev is not None and getattr(dev, "index", None) is not None:
        import torch
        cur = torch.cuda.current_device()
        if dev.index != cur:
            raise ValueError(f"{name} is on cuda:{dev.index} but the current device is cuda:{cur}")
    return int(x.data_ptr())


def _elem(dtype: int) -> Optional[str]:
    return _ELEM.get(int(dtype))


def _n(*xs) -> int:
    """Product of sizes, 0 if any is negative (the library then rejects the sizes itself)."""
    r = 1
    for x in xs:
        if int(x) < 0:
            return 0
        r *= int(x)
    return r


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(status: int, what: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, what)


def _fwd_sizes(B, Sq, Skv, Nq, Nkv, D, Dv, layout):
    """Element counts of q, k, v, out and one statistic array in attn_fwd's layouts."""
    if int(layout) == ATTN_TND:
        return _n(Sq, Nq, D), _n(Skv, Nkv, D), _n(Skv, Nkv, Dv), _n(Sq, Nq, Dv), _n(Sq, Nq)
    return (_n(B, Nq, Sq, D), _n(B, Nkv, Skv, D), _n(B, Nkv, Skv, Dv), _n(B, Nq, Sq, Dv),
            _n(B, Nq, Sq))


def _cu_ptr(cu, name: str, B: int):
    return _ptr(cu, name, _n(B), "int32")


def attn_fwd(q, k, v, *, cu_seqlens_q=None, cu_seqlens_kv=None, B: int, Sq: int, Skv: int,
             Nq: int, Nkv: int, D: int, scale: float, mask_mode: int, dtype: int, layout: int,
             out, softmax_max=None, softmax_sum=None, stream=None) -> None:
    """Fused attention forward (see ``attn_fwd`` in include/attn.h for layouts and limits)."""
    lib = load_library()
    nq, nk, nv, no, ns = _fwd_sizes(B, Sq, Skv, Nq, Nkv, D, D, layout)
    et = _elem(dtype)
    _check(lib.attn_fwd(_ptr(q, "q", nq, et), _ptr(k, "k", nk, et), _ptr(v, "v", nv, et),
                        _cu_ptr(cu_seqlens_q, "cu_seqlens_q", B), _cu_ptr(cu_seqlens_kv, "cu_seqlens_kv", B),
                        int(B), int(Sq), int(Skv), int(Nq), int(Nkv), int(D), float(scale),
                        int(mask_mode), int(dtype), int(layout), _ptr(out, "out", no, et),
                        _ptr(softmax_max, "softmax_max", ns, "float32"),
                        _ptr(softmax_sum, "softmax_sum", ns, "float32"), _stream(stream)), "attn_fwd")


def attn_fwd_accumulate(q, k, v, *, cu_seqlens_q=None, cu_seqlens_kv=None, B: int, Sq: int, Skv: int,
                        Nq: int, Nkv: int, D: int, scale: float, mask_mode: int, dtype: int,
                        layout: int, first: bool, acc_out, acc_max, acc_sum, stream=None) -> None:
    """attn_fwd over one chunk of keys, folded into a running accumulator in attn_merge's
    layouts (see ``attn_fwd_accumulate`` in include/attn.h)."""
    lib = load_library()
    nq, nk, nv, no, ns = _fwd_sizes(B, Sq, Skv, Nq, Nkv, D, D, layout)
    et = _elem(dtype)
    _check(lib.attn_fwd_accumulate(_ptr(q, "q", nq, et), _ptr(k, "k", nk, et), _ptr(v, "v", nv, et),
                                   _cu_ptr(cu_seqlens_q, "cu_seqlens_q", B),
                                   _cu_ptr(cu_seqlens_kv, "cu_seqlens_kv", B), int(B), int(Sq),
                                   int(Skv), int(Nq), int(Nkv), int(D), float(scale), int(mask_mode),
                                   int(dtype), int(layout), 1 if first else 0,
                                   _ptr(acc_out, "acc_out", no, et),
                                   _ptr(acc_max, "acc_max", 8 * ns, "float32"),
                                   _ptr(acc_sum, "acc_sum", 8 * ns, "float32"),
                                   _stream(stream)), "attn_fwd_accumulate")


def attn_fwd_masked(q, k, v, *, cu_seqlens_q=None, cu_seqlens_kv=None, B: int, Sq: int, Skv: int,
                    Nq: int, Nkv: int, Dqk: int, Dv: int, scale: float, mask_mode: int,
                    pre_tokens: int = 0, next_tokens: int = 0, atten_mask=None,
                    mask_batch_stride: int = 0, mask_row_stride: int = 0, dtype: int, layout: int,
                    out, softmax_max=None, softmax_sum=None, stream=None) -> None:
    """attn_fwd with a band, an optional uint8 mask (1 = excluded) and a value head size Dv
    (see ``attn_fwd_masked`` in include/attn.h)."""
    lib = load_library()
    nq, nk, nv, no, ns = _fwd_sizes(B, Sq, Skv, Nq, Nkv, Dqk, Dv, layout)
    et = _elem(dtype)
    nm = 0
    if int(layout) == ATTN_BHSD and _n(B, Sq, Skv) > 0:  # the last entry the mask is read at
        nm = max(0, (int(B) - 1) * int(mask_batch_stride) + (int(Sq) - 1) * int(mask_row_stride) + int(Skv))
    _check(lib.attn_fwd_masked(_ptr(q, "q", nq, et), _ptr(k, "k", nk, et), _ptr(v, "v", nv, et),
                               _cu_ptr(cu_seqlens_q, "cu_seqlens_q", B),
                               _cu_ptr(cu_seqlens_kv, "cu_seqlens_kv", B),
                               int(B), int(Sq), int(Skv), int(Nq), int(Nkv), int(Dqk), int(Dv),
                               float(scale), int(mask_mode), int(pre_tokens), int(next_tokens),
                               _ptr(atten_mask, "atten_mask", nm, "uint8"), int(mask_batch_stride),
                               int(mask_row_stride), int(dtype), int(layout), _ptr(out, "out", no, et),
                               _ptr(softmax_max, "softmax_max", ns, "float32"),
                               _ptr(softmax_sum, "softmax_sum", ns, "float32"), _stream(stream)),
           "attn_fwd_masked")


def attn_sparse_csr(q, k, v, csr_offset, csr_columns, *, B: int, H: int, S: int, D: int,
                    nnz_cap: int, out, stream=None) -> None:
    """CSR-sparse attention forward in float32 (see ``attn_sparse_csr`` in include/attn.h)."""
    lib = load_library()
    n = _n(B, H, S, D)
    _check(lib.attn_sparse_csr(_ptr(q, "q", n, "float32"), _ptr(k, "k", n, "float32"),
                               _ptr(v, "v", n, "float32"),
                               _ptr(csr_offset, "csr_offset", _n(B, H, int(S) + 1), "int32"),
                               _ptr(csr_columns, "csr_columns", _n(B, H, nnz_cap), "int32"),
                               int(B), int(H), int(S), int(D), int(nnz_cap), _ptr(out, "out", n, "float32"),
                               _stream(stream)), "attn_sparse_csr")


def attn_sparse_csr_tc(q, k, v, csr_offset, csr_columns, *, B: int, H: int, S: int, D: int,
                       nnz_cap: int, dtype: int, out, stream=None) -> None:
    """CSR-sparse attention forward in bf16/fp16 on the tensor cores (see
    ``attn_sparse_csr_tc`` in include/attn.h)."""
    lib = load_library()
    n = _n(B, H, S, D)
    et = _elem(dtype)
    _check(lib.attn_sparse_csr_tc(_ptr(q, "q", n, et), _ptr(k, "k", n, et), _ptr(v, "v", n, et),
                                  _ptr(csr_offset, "csr_offset", _n(B, H, int(S) + 1), "int32"),
                                  _ptr(csr_columns, "csr_columns", _n(B, H, nnz_cap), "int32"),
                                  int(B), int(H), int(S), int(D), int(nnz_cap), int(dtype),
                                  _ptr(out, "out", n, et), _stream(stream)), "attn_sparse_csr_tc")


def attn_csr_plan_size(*, B: int, H: int, S: int, nnz_cap: int) -> int:
    """Bytes of the plan of a CSR pattern of this shape (``attn_csr_plan_size`` in
    include/attn.h); allocate that many bytes (uint8, on the device) for attn_csr_plan."""
    lib = load_library()
    n = ctypes.c_int64(0)
    _check(lib.attn_csr_plan_size(int(B), int(H), int(S), int(nnz_cap), ctypes.byref(n)),
           "attn_csr_plan_size")
    return int(n.value)


def attn_csr_plan(csr_offset, csr_columns, *, B: int, H: int, S: int, nnz_cap: int, plan,
                  stream=None) -> None:
    """Build the plan of a CSR pattern into `plan` (a uint8 device tensor of at least
    attn_csr_plan_size bytes); see ``attn_csr_plan`` in include/attn.h."""
    lib = load_library()
    nb = attn_csr_plan_size(B=B, H=H, S=S, nnz_cap=nnz_cap)
    _check(lib.attn_csr_plan(_ptr(csr_offset, "csr_offset", _n(B, H, int(S) + 1), "int32"),
                             _ptr(csr_columns, "csr_columns", _n(B, H, nnz_cap), "int32"), int(B),
                             int(H), int(S), int(nnz_cap), _ptr(plan, "plan", nb, "uint8"),
                             int(plan.numel()) if plan is not None and not isinstance(plan, int) else nb,
                             _stream(stream)), "attn_csr_plan")


def attn_sparse_csr_tc_planned(q, k, v, plan, *, B: int, H: int, S: int, D: int, nnz_cap: int,
                               dtype: int, out, stream=None) -> None:
    """attn_sparse_csr_tc from a plan of the pattern (see ``attn_sparse_csr_tc_planned`` in
    include/attn.h)."""
    lib = load_library()
    n = _n(B, H, S, D)
    et = _elem(dtype)
    nb = attn_csr_plan_size(B=B, H=H, S=S, nnz_cap=nnz_cap)
    _check(lib.attn_sparse_csr_tc_planned(_ptr(q, "q", n, et), _ptr(k, "k", n, et), _ptr(v, "v", n, et),
                                          _ptr(plan, "plan", nb, "uint8"),
                                          int(plan.numel()) if plan is not None and not isinstance(plan, int) else nb,
                                          int(B), int(H), int(S), int(D), int(nnz_cap), int(dtype),
                                          _ptr(out, "out", n, et), _stream(stream)),
           "attn_sparse_csr_tc_planned")


def attn_sparse_csr_tc_noalloc(q, k, v, csr_offset, csr_columns, *, B: int, H: int, S: int, D: int,
                               nnz_cap: int, dtype: int, out, stream=None) -> None:
    """attn_sparse_csr_tc for callers that cannot allocate device memory: the library plans the
    pattern into its own fixed 48 MiB scratch array and runs the planned kernel (see
    ``attn_sparse_csr_tc_noalloc`` in include/attn.h; calls that overlap on the GPU race)."""
    lib = load_library()
    n = _n(B, H, S, D)
    et = _elem(dtype)
    _check(lib.attn_sparse_csr_tc_noalloc(_ptr(q, "q", n, et), _ptr(k, "k", n, et), _ptr(v, "v", n, et),
                                          _ptr(csr_offset, "csr_offset", _n(B, H, int(S) + 1), "int32"),
                                          _ptr(csr_columns, "csr_columns", _n(B, H, nnz_cap), "int32"),
                                          int(B), int(H), int(S), int(D), int(nnz_cap), int(dtype),
                                          _ptr(out, "out", n, et), _stream(stream)),
           "attn_sparse_csr_tc_noalloc")


def attn_merge(prev_out, prev_max, prev_sum, cur_out, cur_max, cur_sum, *, S: int, B: int, N: int,
               D: int, dtype: int, out, out_max, out_sum, layout: int = ATTN_BHSD,
               actual_seq_qlen=None, stream=None) -> None:
    """Merge two partial attention results (see ``attn_merge`` in include/attn.h)."""
    lib = load_library()
    et = _elem(dtype)
    if int(layout) == ATTN_TND:
        no, ns = _n(S, N, D), _n(S, N, 8)
    else:
        no, ns = _n(S, B, N, D), _n(B, N, S, 8)
    f = "float32"
    _check(lib.attn_merge(_ptr(prev_out, "prev_out", no, et), _ptr(prev_max, "prev_max", ns, f),
                          _ptr(prev_sum, "prev_sum", ns, f), _ptr(cur_out, "cur_out", no, et),
                          _ptr(cur_max, "cur_max", ns, f), _ptr(cur_sum, "cur_sum", ns, f), int(S),
                          int(B), int(N), int(D), int(dtype), int(layout),
                          _ptr(actual_seq_qlen, "actual_seq_qlen", _n(B), "int64"),
                          _ptr(out, "out", no, et), _ptr(out_max, "out_max", ns, f),
                          _ptr(out_sum, "out_sum", ns, f), _stream(stream)), "attn_merge")


def attn_get_last_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    lib = load_library()
    st = ctypes.c_int(0)
    _check(lib.attn_get_last_error(_stream(stream), ctypes.byref(st)), "attn_get_last_error")
    return int(st.value)
