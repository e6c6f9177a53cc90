"""The C-ABI library builds, loads and exports every function include/attn.h declares; host-side
argument checks answer without a GPU (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import build as sdpa_build
from scaled_dot_product_16_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    sdpa_build.build()
    return sdpa.load_library()


def _declared():
    text = open(HEADER).read()
    return re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)


def _enums():
    text = open(HEADER).read()
    return {k: int(v) for k, v in re.findall(r"\b(ATTN_[A-Z0-9_]+)\s*=\s*(\d+)", text)}


def test_header_declares_the_three_operations():
    names = set(_declared())
    assert {"attn_fwd", "attn_sparse_csr", "attn_merge", "attn_get_last_error"} <= names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sdpa.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (attn_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_enum_values_match_binding():
    e = _enums()
    for k, v in e.items():
        if hasattr(sdpa, k):
            assert getattr(sdpa, k) == v, k
    assert (W.BF16, W.F32) == (e["ATTN_BF16"], e["ATTN_F32"])
    assert (W.BHSD, W.TND) == (e["ATTN_BHSD"], e["ATTN_TND"])
    assert (W.MASK_NONE, W.MASK_CAUSAL_TOPLEFT, W.MASK_CAUSAL_BOTTOMRIGHT) == (
        e["ATTN_MASK_NONE"], e["ATTN_MASK_CAUSAL_TOPLEFT"], e["ATTN_MASK_CAUSAL_BOTTOMRIGHT"])


def test_version_and_strings(lib):
    assert lib.attn_abi_version() >> 16 == 1
    for s in range(6):
        assert lib.attn_status_string(s)


def _fwd(lib, **kw):
    a = dict(q=16, k=16, v=16, cq=None, ck=None, B=1, Sq=8, Skv=8, Nq=2, Nkv=1, D=64, scale=0.125,
             mask=0, dtype=0, layout=0, out=16, m=None, l=None, stream=None)
    a.update(kw)
    return lib.attn_fwd(a["q"], a["k"], a["v"], a["cq"], a["ck"], a["B"], a["Sq"], a["Skv"],
                        a["Nq"], a["Nkv"], a["D"], a["scale"], a["mask"], a["dtype"], a["layout"],
                        a["out"], a["m"], a["l"], a["stream"])


def test_host_validation_without_gpu(lib):
    INVALID, UNSUP, OK = sdpa.ATTN_ERR_INVALID, sdpa.ATTN_ERR_UNSUPPORTED, sdpa.ATTN_OK
    assert _fwd(lib, layout=7) == INVALID
    assert _fwd(lib, dtype=5) == INVALID
    assert _fwd(lib, mask=3) == INVALID
    assert _fwd(lib, Nq=3, Nkv=2) == INVALID         # Nq/Nkv must be an integer
    assert _fwd(lib, Nq=257, Nkv=1) == INVALID       # Nq in 1..256
    assert _fwd(lib, D=769) == INVALID               # D in 1..768
    assert _fwd(lib, scale=0.0) == INVALID
    assert _fwd(lib, scale=float("nan")) == INVALID
    assert _fwd(lib, m=16) == INVALID                # max without sum
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, D=96) == UNSUP                  # bf16 runs D = 64 or 128
    assert _fwd(lib, D=96, dtype=2) == UNSUP         # fp16 too
    assert _fwd(lib, dtype=3) == INVALID
    assert _fwd(lib, q=18) == INVALID                # bf16 pointers must be 16-byte aligned
    assert _fwd(lib, layout=1, B=3) == INVALID       # TND needs cumulative lengths
    assert _fwd(lib, layout=1, B=2049, cq=16, ck=16) == INVALID
    assert _fwd(lib, layout=1, B=1, Sq=(1 << 20) + 1, cq=16, ck=16) == INVALID
    assert _fwd(lib, layout=0, cq=16) == INVALID     # BHSD takes no lengths
    # empty problems succeed without a launch
    assert _fwd(lib, B=0) == OK
    assert _fwd(lib, Sq=0) == OK
    assert _fwd(lib, layout=1, B=0) == OK


def _masked(lib, **kw):
    a = dict(q=16, k=16, v=16, cq=None, ck=None, B=1, Sq=8, Skv=8, Nq=2, Nkv=1, Dqk=64, Dv=64,
             scale=0.125, mask=3, pre=4, nxt=0, am=None, bs=0, rs=0, dtype=1, layout=0, out=16,
             m=None, l=None, stream=None)
    a.update(kw)
    return lib.attn_fwd_masked(a["q"], a["k"], a["v"], a["cq"], a["ck"], a["B"], a["Sq"], a["Skv"],
                               a["Nq"], a["Nkv"], a["Dqk"], a["Dv"], a["scale"], a["mask"], a["pre"],
                               a["nxt"], a["am"], a["bs"], a["rs"], a["dtype"], a["layout"],
                               a["out"], a["m"], a["l"], a["stream"])


def test_masked_validation_without_gpu(lib):
    INVALID, UNSUP, OK = sdpa.ATTN_ERR_INVALID, sdpa.ATTN_ERR_UNSUPPORTED, sdpa.ATTN_OK
    assert _fwd(lib, mask=3) == INVALID                 # the band needs attn_fwd_masked
    assert _masked(lib, mask=4) == INVALID
    assert _masked(lib, pre=-5, nxt=4) == INVALID       # empty band
    assert _masked(lib, pre=-(1 << 62), nxt=-(1 << 62)) == INVALID
    assert _masked(lib, Dv=65) == INVALID               # Dv <= Dqk
    assert _masked(lib, Dv=0) == INVALID
    assert _masked(lib, am=16, rs=7) == INVALID         # BHSD rows shorter than Skv
    assert _masked(lib, am=16, rs=8, bs=-1) == INVALID
    assert _masked(lib, dtype=0, Dv=32) == UNSUP        # tensor-core path: Dv == Dqk
    assert _masked(lib, B=0) == OK                      # empty problem, no launch
    assert _masked(lib, layout=1, B=0, Sq=0, Skv=0) == OK


def test_merge_and_csr_validation_without_gpu(lib):
    P = 16
    args = [P] * 6
    assert lib.attn_merge(*args, 8, 1, 2, 64, 3, 0, None, P, P, P, None) == sdpa.ATTN_ERR_INVALID  # dtype
    assert lib.attn_merge(*args, 8, 1, 2, 64, 0, 0, P, P, P, P, None) == sdpa.ATTN_ERR_INVALID  # SBH + lengths
    assert lib.attn_merge(*args, 8, 0, 2, 64, 0, 1, P, P, P, P, None) == sdpa.ATTN_ERR_INVALID  # TND, B = 0
    assert lib.attn_merge(*args, 0, 0, 2, 64, 0, 1, None, P, P, P, None) == sdpa.ATTN_OK        # T = 0
    assert lib.attn_merge(*args, 8, 1, 0, 64, 0, 0, None, P, P, P, None) == sdpa.ATTN_ERR_INVALID
    assert lib.attn_merge(*args, 0, 1, 2, 64, 0, 0, None, P, P, P, None) == sdpa.ATTN_OK
    assert lib.attn_sparse_csr(P, P, P, P, P, 1, 1, 4, 0, 4, P, None) == sdpa.ATTN_ERR_INVALID
    assert lib.attn_sparse_csr(P, P, P, P, P, 1, 1, 4, 300, 4, P, None) == sdpa.ATTN_ERR_UNSUPPORTED
    assert lib.attn_sparse_csr(P, P, P, P, P, 0, 1, 4, 64, 4, P, None) == sdpa.ATTN_OK
    tc = lib.attn_sparse_csr_tc
    assert tc(P, P, P, P, P, 1, 1, 4, 64, 4, sdpa.ATTN_F32, P, None) == sdpa.ATTN_ERR_INVALID
    assert tc(P, P, P, P, P, 1, 1, 4, 96, 4, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_ERR_UNSUPPORTED
    assert tc(P, P, P, P, P, 1, 1, 32769, 64, 4, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_ERR_UNSUPPORTED
    assert tc(18, P, P, P, P, 1, 1, 4, 64, 4, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_ERR_INVALID
    assert tc(P, P, P, P, P, 0, 1, 4, 64, 4, sdpa.ATTN_F16, P, None) == sdpa.ATTN_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(sdpa, "_lib", None)
    monkeypatch.setattr(sdpa, "lib_path", lambda: str(tmp_path / "libattn.so"))
    with pytest.raises(RuntimeError):
        sdpa.attn_merge(None, None, None, None, None, None, S=1, B=1, N=1, D=1, dtype=0,
                        out=None, out_max=None, out_sum=None, stream=0)


def test_binding_rejects_host_and_strided_tensors(lib):
    """The C ABI reads device arrays; the binding refuses host tensors (whose addresses a kernel
    cannot read) and non-contiguous views before anything is called."""
    import torch
    host = torch.zeros(4, 8)
    with pytest.raises(ValueError, match="CUDA device"):
        sdpa.attn_merge(host, host, host, host, host, host, S=1, B=1, N=1, D=8, dtype=sdpa.ATTN_F32,
                        out=host, out_max=host, out_sum=host, stream=0)

    class Strided:  # stands in for a strided CUDA tensor on a machine without a GPU
        is_cuda = True

        def is_contiguous(self):
            return False

        def data_ptr(self):
            return 16

    with pytest.raises(ValueError, match="contiguous"):
        sdpa._ptr(Strided())


def test_product_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "scaled_dot_product_16_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "attn_oracle" not in text, f


class FakeCuda:
    """Stands in for a CUDA tensor on a machine without a GPU (the binding reads only these
    attributes before it calls the library)."""

    def __init__(self, numel, dtype, index=0):
        import torch
        self._n, self.dtype, self.device, self.is_cuda = numel, dtype, torch.device("cuda", index), True

    def numel(self):
        return self._n

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return 256


@pytest.fixture
def on_cuda0(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(sdpa, "_stream", lambda s: 0)


def _fwd_kwargs(**kw):
    import torch
    bf = torch.bfloat16
    a = dict(q=FakeCuda(2 * 4 * 64, bf), k=FakeCuda(1 * 4 * 64, bf), v=FakeCuda(1 * 4 * 64, bf),
             B=1, Sq=4, Skv=4, Nq=2, Nkv=1, D=64, scale=0.125, mask_mode=0, dtype=sdpa.ATTN_BF16,
             layout=sdpa.ATTN_BHSD, out=FakeCuda(2 * 4 * 64, bf), softmax_max=FakeCuda(8, torch.float32),
             softmax_sum=FakeCuda(8, torch.float32))
    a.update(kw)
    return a


def test_binding_refuses_undersized_mistyped_and_foreign_tensors(lib, on_cuda0):
    """Each refusal comes from the binding, before the library is called: a tensor smaller than
    the sizes given, a tensor whose element type is not the declared one, integer arrays of the
    wrong width, and a tensor on another device than the current one."""
    import torch
    bf, f32 = torch.bfloat16, torch.float32
    refused = [
        (dict(q=FakeCuda(2 * 4 * 64 - 1, bf)), "holds"),                 # q one element short
        (dict(out=FakeCuda(100, bf)), "holds"),                            # out too small
        (dict(softmax_max=FakeCuda(7, f32)), "holds"),                     # statistics too small
        (dict(q=FakeCuda(2 * 4 * 64, torch.float16)), "bfloat16"),         # fp16 data, bf16 declared
        (dict(q=FakeCuda(2 * 4 * 64, f32), k=FakeCuda(256, f32), v=FakeCuda(256, f32),
              out=FakeCuda(512, f32), dtype=sdpa.ATTN_BF16), "bfloat16"),  # fp32 data, bf16 declared
        (dict(softmax_sum=FakeCuda(8, bf)), "float32"),                    # statistics must be fp32
        (dict(k=FakeCuda(256, bf, index=1)), "current device"),            # k on another GPU
    ]
    for kw, msg in refused:
        with pytest.raises(ValueError, match=msg):
            sdpa.attn_fwd(**_fwd_kwargs(**kw))
    # TND: cumulative lengths must be int32 with B entries
    tnd = dict(layout=sdpa.ATTN_TND, B=2, Sq=4, Skv=4, q=FakeCuda(4 * 2 * 64, bf), k=FakeCuda(4 * 64, bf),
               v=FakeCuda(4 * 64, bf), out=FakeCuda(4 * 2 * 64, bf))
    with pytest.raises(ValueError, match="int32"):
        sdpa.attn_fwd(**_fwd_kwargs(**tnd, cu_seqlens_q=FakeCuda(2, torch.int64), cu_seqlens_kv=FakeCuda(2, torch.int32)))
    with pytest.raises(ValueError, match="holds"):
        sdpa.attn_fwd(**_fwd_kwargs(**tnd, cu_seqlens_q=FakeCuda(1, torch.int32), cu_seqlens_kv=FakeCuda(2, torch.int32)))
    # CSR: fp32 tensors, int32 row pointers and columns of the stated sizes
    n = 1 * 2 * 8 * 64
    csr = dict(B=1, H=2, S=8, D=64, nnz_cap=10)
    good = [FakeCuda(n, f32) for _ in range(3)] + [FakeCuda(2 * 9, torch.int32), FakeCuda(20, torch.int32)]
    with pytest.raises(ValueError, match="csr_columns"):
        sdpa.attn_sparse_csr(*good[:4], FakeCuda(19, torch.int32), out=FakeCuda(n, f32), **csr)
    with pytest.raises(ValueError, match="csr_offset"):
        sdpa.attn_sparse_csr(*good[:3], FakeCuda(2 * 9, torch.int64), good[4], out=FakeCuda(n, f32), **csr)
    with pytest.raises(ValueError, match="float32"):
        sdpa.attn_sparse_csr(FakeCuda(n, bf), *good[1:], out=FakeCuda(n, f32), **csr)
    # merge: TND lengths are int64; statistics fp32 with 8 lanes per row
    S, N, D = 16, 2, 64
    po = FakeCuda(S * N * D, bf)
    st = FakeCuda(S * N * 8, f32)
    with pytest.raises(ValueError, match="int64"):
        sdpa.attn_merge(po, st, st, po, st, st, S=S, B=2, N=N, D=D, dtype=sdpa.ATTN_BF16, out=po,
                        out_max=st, out_sum=st, layout=sdpa.ATTN_TND,
                        actual_seq_qlen=FakeCuda(2, torch.int32))
    with pytest.raises(ValueError, match="holds"):
        sdpa.attn_merge(po, FakeCuda(S * N, f32), st, po, st, st, S=S, B=2, N=N, D=D,
                        dtype=sdpa.ATTN_BF16, out=po, out_max=st, out_sum=st, layout=sdpa.ATTN_TND)
    # accumulator statistics carry 8 lanes per row
    with pytest.raises(ValueError, match="acc_max"):
        a = _fwd_kwargs()
        sdpa.attn_fwd_accumulate(a["q"], a["k"], a["v"], B=1, Sq=4, Skv=4, Nq=2, Nkv=1, D=64, scale=0.125,
                                 mask_mode=0, dtype=sdpa.ATTN_BF16, layout=sdpa.ATTN_BHSD, first=True,
                                 acc_out=FakeCuda(512, bf), acc_max=FakeCuda(8, f32), acc_sum=FakeCuda(64, f32))


def test_accumulate_refuses_unaligned_statistics(lib):
    """The tensor-core epilogue moves a row's 8 statistic lanes as 16-byte vectors, so for 16-bit
    types a 4-byte-aligned accumulator (a sliced view, say) is refused on the host."""
    def call(am, al, dtype):
        return lib.attn_fwd_accumulate(16, 16, 16, None, None, 1, 8, 8, 2, 1, 64, 0.125, 0, dtype,
                                       sdpa.ATTN_BHSD, 1, 16, am, al, None)
    assert call(20, 16, sdpa.ATTN_BF16) == sdpa.ATTN_ERR_INVALID
    assert call(16, 36, sdpa.ATTN_F16) == sdpa.ATTN_ERR_INVALID
    assert call(24, 40, sdpa.ATTN_BF16) == sdpa.ATTN_ERR_INVALID


def test_plan_size_and_validation_without_gpu(lib):
    import ctypes
    n = ctypes.c_int64(0)
    assert lib.attn_csr_plan_size(2, 8, 4096, 1278208, ctypes.byref(n)) == sdpa.ATTN_OK
    # 2*8 slices x 32 row blocks x (64 + 20 * 4096) bytes
    assert n.value == 2 * 8 * 32 * (64 + 20 * 4096)
    assert lib.attn_csr_plan_size(1, 1, 300, 10, ctypes.byref(n)) == sdpa.ATTN_OK
    assert n.value == 3 * (64 + 20 * 128)             # ucap = 10 rounded up to 128
    assert lib.attn_csr_plan_size(1, 1, 32769, 10, ctypes.byref(n)) == sdpa.ATTN_ERR_UNSUPPORTED
    assert lib.attn_csr_plan_size(-1, 1, 8, 10, ctypes.byref(n)) == sdpa.ATTN_ERR_INVALID
    assert lib.attn_csr_plan_size(1, 1, 8, 10, None) == sdpa.ATTN_ERR_INVALID
    need = 64 + 20 * 128
    P = 16
    assert lib.attn_csr_plan(P, P, 1, 1, 8, 10, P, need - 1, None) == sdpa.ATTN_ERR_INVALID  # too small
    assert lib.attn_csr_plan(P, P, 1, 1, 8, 10, 24, need, None) == sdpa.ATTN_ERR_INVALID     # unaligned
    assert lib.attn_csr_plan(None, P, 1, 1, 8, 10, P, need, None) == sdpa.ATTN_ERR_INVALID
    assert lib.attn_csr_plan(P, P, 0, 1, 8, 10, P, 0, None) == sdpa.ATTN_OK                  # empty
    tcp = lib.attn_sparse_csr_tc_planned
    assert tcp(P, P, P, P, need, 1, 1, 8, 64, 10, sdpa.ATTN_F32, P, None) == sdpa.ATTN_ERR_INVALID
    assert tcp(P, P, P, P, need, 1, 1, 8, 96, 10, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_ERR_UNSUPPORTED
    assert tcp(P, P, P, P, need - 16, 1, 1, 8, 64, 10, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_ERR_INVALID
    assert tcp(P, P, P, None, need, 1, 1, 8, 64, 10, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_ERR_INVALID
    assert tcp(P, P, P, P, need, 0, 1, 8, 64, 10, sdpa.ATTN_BF16, P, None) == sdpa.ATTN_OK
