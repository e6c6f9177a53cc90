#!/usr/bin/env python
"""Benchmark of the attention hot path on B200.

One step runs every operation of the path once, on inputs already resident in HBM:
  1. attn_fwd on the packed varlen batch: 16 sequences of U{0..8192} tokens (index 7 empty),
     Nq=32, Nkv=8, D=128, bf16, causal per sequence (the tcgen05 kernel);
  2. attn_sparse_csr on B=2, H=8, S=4096, D=64 fp32 with a 256-wide window plus every 64th column;
  3. three attn_merge calls folding 4 partial results of S=8192, B=4, N=32, D=128 (bf16, SBH,
     statistics [B,N,S,8]) into one, as a 4-chunk ring-attention step would.
Each operation is timed with CUDA events on the stream it is launched on. The headline `value`
is attn_fwd TFLOP/s over all ranks (4*Nq*D FLOPs per visible pair, divided by the max over
ranks of the time); the merge's HBM GB/s is reported beside it (the second half of the metric).

  python bench.py [--gpus N --steps K --warmup W]          # this library
  python bench.py --impl reference ...                       # the float64 CPU oracle, sampled
Multi-GPU: launched by torchrun, one process per GPU; every rank runs its own batch (seeded by
rank, weak scaling) and no data-path collective exists (the path partitions by sequence and
head); NCCL carries only the barrier and the max-over-ranks of the times.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import scaled_dot_product_16_b200 as sdpa  # noqa: E402
from scaled_dot_product_16_b200 import metrics as M  # noqa: E402
from scaled_dot_product_16_b200 import workloads as W  # noqa: E402

METRIC = "attn fwd TFLOP/s & % of BF16 tensor peak; attn_merge HBM GB/s & % of peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attn_fwd launch on the
# default varlen batch (75,336 tokens), from a one-pass ncu capture of that launch. It is
# reported only for that workload and while the kernel source still has the hash it was
# measured on.
TRAFFIC = {"kernel_sha": "bef5e0c1c677025e", "tokens": 75_336, "bytes_per_launch": 938_526_208 + 602_562_816}


KERNEL_SOURCES = ("fwd_bf16_sm100.cu", "sm100.cuh", "common.cuh", "launch.h")


def kernel_sha() -> str:
    """Hash of every source the attn_fwd kernel is built from (its .cu and the headers it
    includes), so a stored DRAM-traffic figure is dropped when any of them changes."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "scaled_dot_product_16_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


# Nominal clock and FP32 FMA width of B200, for the ALU roofline of the fp32 CSR kernel:
# 148 SMs x 128 fp32 FMA lanes x 2 FLOPs per FMA x 1.965 GHz (the maximum SM clock).
B200_SMS, FMA_PER_SM, MAX_SM_GHZ = 148, 128, 1.965
FP32_FMA_TFLOPS = B200_SMS * FMA_PER_SM * 2 * MAX_SM_GHZ / 1e3


def tensor_peak(peaks: dict) -> float:
    """The dense bf16 peak a kernel's fraction is taken against: the burst cuBLAS figure,
    measured like the timed loops here, at full clock over a short region (the sustained
    figure was measured over seconds of back-to-back GEMMs held near 1.35 GHz by the power cap)."""
    return float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------------------------
def dist_setup(use_gpu: bool = True):
    """Rank, world size and local rank from the launcher's environment. The GPU arm binds a
    device and, for N > 1, an NCCL process group; the reference arm (CPU oracle, rank 0 only,
    no collective) touches neither."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not use_gpu:
        return rank, world, local
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce(x: float, world: int, op: str) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        t0 = time.time()  # the first sample marks the sampler as running
        while time.time() - t0 < 15 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = [l.split(", ") for l in open(self.path).read().strip().splitlines() if l.strip()]
        os.unlink(self.path)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# workloads on the device
# ---------------------------------------------------------------------------------------------
class FwdCase:
    def __init__(self, inp: W.AttnInputs):
        self.inp = inp
        self.q, self.k, self.v = (t.cuda() for t in (inp.q, inp.k, inp.v))
        self.cq = torch.from_numpy(inp.cu_q).cuda() if inp.cu_q is not None else None
        self.ck = torch.from_numpy(inp.cu_kv).cuda() if inp.cu_kv is not None else None
        self.out = torch.empty_like(self.q)
        shape = (inp.Sq, inp.Nq) if inp.layout == W.TND else (inp.B, inp.Nq, inp.Sq)
        self.m = torch.empty(shape, device="cuda")
        self.l = torch.empty(shape, device="cuda")
        self.flops = M.attn_fwd_flops(inp)

    def run(self, q=None, k=None, v=None, cq=None, ck=None, out=None, m=None, l=None):
        i = self.inp
        sdpa.attn_fwd(q if q is not None else self.q, k if k is not None else self.k,
                      v if v is not None else self.v, cu_seqlens_q=cq if cq is not None else self.cq,
                      cu_seqlens_kv=ck if ck is not None else self.ck, B=i.B, Sq=i.Sq, Skv=i.Skv,
                      Nq=i.Nq, Nkv=i.Nkv, D=i.D, scale=i.scale, mask_mode=i.mask_mode, dtype=i.dtype,
                      layout=i.layout, out=out if out is not None else self.out,
                      softmax_max=m if m is not None else self.m,
                      softmax_sum=l if l is not None else self.l)


class CsrCase:
    def __init__(self, inp: W.CsrInputs):
        self.inp = inp
        self.q, self.k, self.v = (t.cuda() for t in (inp.q, inp.k, inp.v))
        self.off = torch.from_numpy(inp.offset).cuda()
        self.col = torch.from_numpy(inp.columns).cuda()
        self.out = torch.empty_like(self.q)
        self.flops = M.csr_flops(inp)
        self.bytes = M.csr_min_bytes(inp)

    def run(self):
        i = self.inp
        sdpa.attn_sparse_csr(self.q, self.k, self.v, self.off, self.col, B=i.B, H=i.H, S=i.S, D=i.D,
                             nnz_cap=i.nnz_cap, out=self.out)


class MergeCase:
    """Four partial results (outputs + statistics) folded by three merges into the first."""

    def __init__(self, seed: int, S=8192, B=4, N=32, D=128):
        self.S, self.B, self.N, self.D = S, B, N, D
        self.parts = []
        for c in range(4):
            o = W.randn((S, B, N * D), W.mix_seed(5, seed, 10 + c), torch.bfloat16).cuda()
            m, l = W.merge_stats_random(B, N, S, W.mix_seed(5, seed, 20 + c))
            self.parts.append((o, m.cuda(), l.cuda()))
        self.acc = [t.clone() for t in self.parts[0]]
        self.bytes = M.merge_bytes(S, B, N, D, 2)

    def run_one(self, c: int):
        a, p = self.acc, self.parts[c]
        sdpa.attn_merge(a[0], a[1], a[2], p[0], p[1], p[2], S=self.S, B=self.B, N=self.N, D=self.D,
                        dtype=W.BF16, out=a[0], out_max=a[1], out_sum=a[2])


def _device_ms(fn, iters: int, stream) -> float:
    """Mean device time of fn() over iters calls (CUDA events on the launching stream)."""
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    if sdpa.attn_get_last_error() != 0:
        raise RuntimeError("device status set while timing a later-row operation")
    return a.elapsed_time(b) / iters


def next_rows(fwd: "FwdCase", csr: "CsrCase", rank: int, stream, peaks: dict) -> dict:
    """The operations built beyond the step's own rows, each timed on its own: the fused
    ring fold, the band (sliding window) and the tensor-core CSR variant."""
    res = {}
    # ring attention, B=4, N=32, S=8192, D=128, keys in 4 chunks of 2048 folded by
    # attn_fwd_accumulate into one accumulator (SBH output, [B,N,S,8] statistics)
    inp = W.dense_bhsd(4, 32, 8192, 128, causal=False, dtype=torch.bfloat16, seed=rank, cfg=5)
    q = inp.q.cuda()
    kc = [inp.k[:, :, c * 2048:(c + 1) * 2048].contiguous().cuda() for c in range(4)]
    vc = [inp.v[:, :, c * 2048:(c + 1) * 2048].contiguous().cuda() for c in range(4)]
    acc = torch.empty((8192, 4, 32 * 128), dtype=torch.bfloat16, device="cuda")
    am = torch.empty((4, 32, 8192, 8), device="cuda")
    al = torch.empty_like(am)

    def ring():
        for c in range(4):
            sdpa.attn_fwd_accumulate(q, kc[c], vc[c], B=4, Sq=8192, Skv=2048, Nq=32, Nkv=32, D=128,
                                     scale=inp.scale, mask_mode=W.MASK_NONE, dtype=W.BF16,
                                     layout=W.BHSD, first=c == 0, acc_out=acc, acc_max=am, acc_sum=al)

    ms = _device_ms(ring, 5, stream)
    fl = M.attn_fwd_flops(inp)
    tensor = tensor_peak(peaks)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    res["attn_fwd_accumulate"] = {"workload": "ring: dense 4x32x8192x128 bf16, 4 key chunks of 2048",
                                  "ms_per_ring": ms, "tflops": fl / (ms / 1e3) / 1e12, "launches": 4,
                                  "frac_of_bf16_peak": fl / (ms / 1e3) / 1e12 / tensor}
    del q, kc, vc, acc, am, al
    # sliding window: 1024 keys back, none ahead, on the step's varlen workload
    i = fwd.inp
    ob = torch.empty_like(fwd.out)
    mb, lb = torch.empty_like(fwd.m), torch.empty_like(fwd.l)

    def band():
        sdpa.attn_fwd_masked(fwd.q, fwd.k, fwd.v, cu_seqlens_q=fwd.cq, cu_seqlens_kv=fwd.ck, B=i.B,
                             Sq=i.Sq, Skv=i.Skv, Nq=i.Nq, Nkv=i.Nkv, Dqk=i.D, Dv=i.D, scale=i.scale,
                             mask_mode=sdpa.ATTN_MASK_BAND, pre_tokens=1023, next_tokens=0,
                             dtype=i.dtype, layout=i.layout, out=ob, softmax_max=mb, softmax_sum=lb)

    ms = _device_ms(band, 20, stream)
    fl = 4 * i.Nq * i.D * M.band_pairs(i, 1023, 0)
    res["attn_fwd_masked"] = {"workload": "band pre=1023 next=0 (sliding window) on the varlen GQA "
                                          "batch of the step (Nq=32 Nkv=8 D=128 bf16)",
                              "ms": ms, "tflops": fl / (ms / 1e3) / 1e12, "flops_per_call": fl,
                              "frac_of_bf16_peak": fl / (ms / 1e3) / 1e12 / tensor}
    # CSR on the tensor cores: the fp32 CSR workload's pattern with bf16 inputs
    c = csr if csr is not None else CsrCase(W.cfg4_csr(seed=rank))
    qb, kb, vb = (t.to(torch.bfloat16) for t in (c.q, c.k, c.v))
    outb = torch.empty_like(qb)
    ci = c.inp

    def csr_tc():
        sdpa.attn_sparse_csr_tc(qb, kb, vb, c.off, c.col, B=ci.B, H=ci.H, S=ci.S, D=ci.D,
                                nnz_cap=ci.nnz_cap, dtype=W.BF16, out=outb)

    ms = _device_ms(csr_tc, 20, stream)
    ms32 = _device_ms(c.run, 20, stream)
    res["attn_sparse_csr_tc"] = {"workload": "2x8x4096x64 bf16, window 256 + every 64th column",
                                 "ms": ms, "tflops": c.flops / (ms / 1e3) / 1e12,
                                 "frac_of_bf16_peak": c.flops / (ms / 1e3) / 1e12 / tensor,
                                 "fp32_kernel_ms": ms32, "speedup_vs_fp32": ms32 / ms}
    # the same call from a plan of the pattern: the plan is built once (timed on its own) and
    # each call then only gathers the union's key/value rows and multiplies
    nb = sdpa.attn_csr_plan_size(B=ci.B, H=ci.H, S=ci.S, nnz_cap=ci.nnz_cap)
    plan = torch.empty(nb, dtype=torch.uint8, device="cuda")

    def mkplan():
        sdpa.attn_csr_plan(c.off, c.col, B=ci.B, H=ci.H, S=ci.S, nnz_cap=ci.nnz_cap, plan=plan)

    def planned():
        sdpa.attn_sparse_csr_tc_planned(qb, kb, vb, plan, B=ci.B, H=ci.H, S=ci.S, D=ci.D,
                                        nnz_cap=ci.nnz_cap, dtype=W.BF16, out=outb)

    ms_plan = _device_ms(mkplan, 20, stream)
    ms_exec = _device_ms(planned, 20, stream)
    res["attn_sparse_csr_tc_planned"] = {
        "workload": "2x8x4096x64 bf16, window 256 + every 64th column, from a plan",
        "ms": ms_exec, "tflops": c.flops / (ms_exec / 1e3) / 1e12, "plan_ms": ms_plan,
        "plan_bytes": nb, "speedup_vs_per_call_union": ms / ms_exec,
        "plan_plus_call_ms": ms_plan + ms_exec}
    del qb, kb, vb, outb, plan
    # merge in the TND layout (ring-attention update of a packed batch): T = 65,536 tokens,
    # N = 32, D = 128, bf16 outputs, [T, N, 8] statistics, with actual_seq_qlen checked
    T, N, D = 65536, 32, 128
    po = W.randn((T, N * D), W.mix_seed(6, rank, 1), torch.bfloat16).cuda()
    co = W.randn((T, N * D), W.mix_seed(6, rank, 2), torch.bfloat16).cuda()
    pm, ps = (x.reshape(1, N, T, 8).permute(0, 2, 1, 3).reshape(T, N, 8).contiguous().cuda()
              for x in W.merge_stats_random(1, N, T, W.mix_seed(6, rank, 3)))
    cm, cs = (x.reshape(1, N, T, 8).permute(0, 2, 1, 3).reshape(T, N, 8).contiguous().cuda()
              for x in W.merge_stats_random(1, N, T, W.mix_seed(6, rank, 4)))
    seq = torch.tensor([T // 4, T // 2, 3 * T // 4, T], dtype=torch.int64, device="cuda")
    mo, mm, ml = torch.empty_like(po), torch.empty_like(pm), torch.empty_like(ps)

    def merge_tnd():
        sdpa.attn_merge(po, pm, ps, co, cm, cs, S=T, B=4, N=N, D=D, dtype=W.BF16, layout=W.TND,
                        actual_seq_qlen=seq, out=mo, out_max=mm, out_sum=ml)

    ms = _device_ms(merge_tnd, 20, stream)
    by = M.merge_bytes(T, 1, N, D, 2)
    res["attn_merge_tnd"] = {"workload": "TND T=65536 N=32 D=128 bf16, [T,N,8] statistics, 4 sequences",
                             "ms": ms, "gbs": by / (ms / 1e3) / 1e9,
                             "frac_of_hbm": by / (ms / 1e3) / 1e9 / hbm, "bytes_per_call": by}
    return res


# ---------------------------------------------------------------------------------------------
# CPU oracle (the reported baseline and the reference arm)
# ---------------------------------------------------------------------------------------------
def oracle_sample(inp: W.AttnInputs, n_rows: int, seed: int):
    """Random (head, token) rows of the workload and their algorithmic FLOPs."""
    rng = np.random.default_rng(seed)
    rows_t = rng.integers(0, inp.Sq, size=n_rows).astype(np.int64)
    rows_h = rng.integers(0, inp.Nq, size=n_rows).astype(np.int32)
    lens = W.lengths_from_cu_seqlens(inp.cu_q)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    seq = np.searchsorted(np.cumsum(lens), rows_t, side="right")
    i = rows_t - starts[seq]
    klens = W.lengths_from_cu_seqlens(inp.cu_kv)[seq]
    vis = np.minimum(i + 1, klens) if inp.mask_mode != W.MASK_NONE else klens
    return rows_h, rows_t, int(4 * inp.D * vis.sum())


def time_oracle(inp: W.AttnInputs, n_rows: int, seed: int):
    import oracle  # the CPU baseline leg is one of the two places bench.py runs the oracle
    rows_h, rows_t, flops = oracle_sample(inp, n_rows, seed)
    t0 = time.perf_counter()
    oracle.attn_fwd_rows(inp.q, inp.k, inp.v, rows_h, rows_t, cu_q=inp.cu_q, cu_kv=inp.cu_kv, B=inp.B,
                         Sq=inp.Sq, Skv=inp.Skv, Nq=inp.Nq, Nkv=inp.Nkv, D=inp.D, scale=inp.scale,
                         mask_mode=inp.mask_mode, layout=inp.layout)
    return flops, time.perf_counter() - t0


def oracle_threads() -> int:
    """Gives the oracle every core this process may run on and returns that count. Only rank 0
    runs the oracle (the other ranks do no CPU work), while a launcher such as torchrun sets
    OMP_NUM_THREADS=1 for every rank; the oracle's OpenMP loops run in torch's OpenMP runtime,
    so torch.set_num_threads sets their width."""
    torch.set_num_threads(len(os.sched_getaffinity(0)))
    return torch.get_num_threads()


def cpu_baseline(inp: W.AttnInputs, budget_s: float = 20.0) -> dict:
    """The oracle as it stands on this host's cores, on a bounded row sample of the workload."""
    cores = oracle_threads()
    n = 64
    flops, dt = time_oracle(inp, n, 1234)
    while dt < 1.0 and n < 1 << 20:  # calibrate on growing samples
        n *= 4
        flops, dt = time_oracle(inp, n, 1234)
    n = max(n, int(n * budget_s / dt))  # then one sample sized to about the budget
    flops, dt = time_oracle(inp, n, 4321)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} random (head, query-token) rows of the varlen batch, all their visible keys; "
                      f"{flops / 1e9:.1f} GFLOP in {dt:.1f} s"}


# ---------------------------------------------------------------------------------------------
def config_dict(i: W.AttnInputs, world: int) -> dict:
    return {"workload": "varlen TND causal GQA bf16: 16 seqs U{0..8192} (idx 7 empty), Nq=32 Nkv=8 D=128; "
                        "plus CSR fp32 2x8x4096x64 (window 256 + every 64th) and 3 SBH merges 8192x4x32x128 bf16",
            "tokens_per_rank": int(i.Sq), "n_seq": int(i.B), "Nq": i.Nq, "Nkv": i.Nkv, "D": i.D,
            "causal": True, "parallelism": f"replicas x{world} (sequence partition, no collective)",
            "l2": "inputs larger than L2 (attn_fwd 0.9 GB, merge 1.0 GB per step), no flush"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    inp = W.cfg3_varlen_gqa(seed=0, max_len=args.max_len)
    rows = args.ref_rows
    cores = oracle_threads()
    for s in range(args.warmup):
        time_oracle(inp, max(8, rows // 8), 100 + s)
    fl, dt = 0, 0.0
    for s in range(args.steps):
        f, d = time_oracle(inp, rows, 1000 + s)
        fl += f
        dt += d
    val = fl / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(inp, world),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} random (head, query-token) rows of the varlen batch per step, all their visible keys"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank: int, world: int, local: int):
    sdpa.load_library()
    peaks, peak_src = load_peaks()
    fwd = FwdCase(W.cfg3_varlen_gqa(seed=rank, max_len=args.max_len))
    parts = args.parts.split(",")
    csr = CsrCase(W.cfg4_csr(seed=rank)) if "csr" in parts else None
    mrg = MergeCase(seed=rank) if "merge" in parts else None
    stream = torch.cuda.current_stream()
    launches_per_step = 1 + (1 if csr else 0) + (3 if mrg else 0)

    def step(ev):
        ev[0].record(stream)
        fwd.run()
        ev[1].record(stream)
        if csr:
            csr.run()
        ev[2].record(stream)
        if mrg:
            for c in (1, 2, 3):
                mrg.run_one(c)
        ev[3].record(stream)

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    torch.cuda.synchronize()
    assert sdpa.attn_get_last_error() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    status = sdpa.attn_get_last_error()
    if status != 0:
        raise RuntimeError(f"device status {status} during the timed region")

    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    csr_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    mrg_ms = sum(e[2].elapsed_time(e[3]) for e in evs)
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms_max = reduce(fwd_ms, world, "max")
    total_ms_max = reduce(total_ms, world, "max")
    flops_all = reduce(float(fwd.flops) * args.steps, world, "sum")
    value = flops_all / (fwd_ms_max / 1e3) / 1e12

    # dominant kernel roofline (attn_fwd) against the burst bf16 peak; beside it the same
    # fraction with the peak scaled by the sampled median SM clock (a note, not the headline)
    achieved = fwd.flops / (fwd_ms / args.steps / 1e3) / 1e12
    peak = tensor_peak(peaks)
    clk_scale = (clk["sm_mhz"] / clk["sm_max_mhz"]) if clk.get("sm_mhz") and clk.get("sm_max_mhz") else None
    traffic = (TRAFFIC["bytes_per_launch"]
               if TRAFFIC["kernel_sha"] == kernel_sha() and int(fwd.inp.Sq) == TRAFFIC["tokens"] else None)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(fwd.inp, world),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "attn_fwd bf16 (tcgen05)",
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "frac_at_sampled_clock": (achieved / (peak * clk_scale)) if clk_scale else None,
                         "frac_of_sustained": achieved / float(peaks.get(
                             "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))},
            "parts": {"attn_fwd": {"ms": fwd_ms / args.steps, "tflops": achieved,
                                   "flops_per_call": fwd.flops, "frac_of_bf16_peak": achieved / peak}},
            "gpu_launches": launches_per_step * args.steps, "clocks": clk}
    if csr:
        c_s = csr_ms / args.steps / 1e3
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        c_tf = csr.flops / c_s / 1e12
        c_gbs = csr.bytes / c_s / 1e9
        line["parts"]["attn_sparse_csr"] = {
            "ms": csr_ms / args.steps, "gflops": c_tf * 1e3, "flops_per_call": csr.flops,
            "roofline": {"bound": "alu", "achieved": c_tf, "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s",
                         "frac": c_tf / FP32_FMA_TFLOPS,
                         "peak_source": "148 SMs x 128 FP32 FMA/clk x 2 FLOP x 1.965 GHz (nominal)"},
            "effective_gbs": c_gbs, "frac_of_hbm": c_gbs / hbm, "bytes_per_call": csr.bytes,
            "bytes_what": "q, k, v, out (fp32) + column indices + row pointers, each once"}
    if mrg:
        gbs = mrg.bytes * 3 / (mrg_ms / args.steps / 1e3) / 1e9
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        line["parts"]["attn_merge"] = {"ms_per_call": mrg_ms / args.steps / 3, "gbs": gbs,
                                       "frac_of_hbm": gbs / hbm, "bytes_per_call": mrg.bytes,
                                       "peak_source": f"{peak_src} hbm_gbs"}

    # end to end through the public API: pinned host inputs -> device -> attn_fwd -> host.
    # Steps are pipelined over two device buffer sets and three streams (copy in, compute,
    # copy out), so one step's upload, the previous step's kernel and the one before's
    # download overlap; every byte of every step still crosses inside the timed region.
    if args.e2e_steps > 0:
        i = fwd.inp
        hq, hk, hv = (t.pin_memory() for t in (i.q, i.k, i.v))
        hcq = torch.from_numpy(i.cu_q).pin_memory()
        nb = 2
        ho = [torch.empty(fwd.out.shape, dtype=fwd.out.dtype).pin_memory() for _ in range(nb)]
        hm = [torch.empty(fwd.m.shape).pin_memory() for _ in range(nb)]
        hl = [torch.empty(fwd.l.shape).pin_memory() for _ in range(nb)]
        dev = [dict(q=torch.empty_like(fwd.q), k=torch.empty_like(fwd.k), v=torch.empty_like(fwd.v),
                    cq=torch.empty_like(fwd.cq), o=torch.empty_like(fwd.out), m=torch.empty_like(fwd.m),
                    l=torch.empty_like(fwd.l)) for _ in range(nb)]
        s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_run = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]

        def e2e_step(st: int):
            b, d = st % nb, dev[st % nb]
            with torch.cuda.stream(s_in):
                if st >= nb:
                    s_in.wait_event(ev_run[b])  # the kernel of step st-2 has read these inputs
                d["q"].copy_(hq, non_blocking=True)
                d["k"].copy_(hk, non_blocking=True)
                d["v"].copy_(hv, non_blocking=True)
                d["cq"].copy_(hcq, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(ev_in[b])
                if st >= nb:
                    s_run.wait_event(ev_out[b])  # step st-2's outputs are on the host
                fwd.run(d["q"], d["k"], d["v"], d["cq"], d["cq"], d["o"], d["m"], d["l"])
                ev_run[b].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run[b])
                ho[b].copy_(d["o"], non_blocking=True)
                hm[b].copy_(d["m"], non_blocking=True)
                hl[b].copy_(d["l"], non_blocking=True)
                ev_out[b].record(s_out)

        # the binding launches on torch's current stream, which the `with` blocks set
        for st in range(nb):
            e2e_step(st)
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        s_run.wait_event(a)
        s_out.wait_event(a)
        for st in range(args.e2e_steps):
            e2e_step(nb + st)
        s_in.wait_stream(s_out)
        b.record(s_in)
        torch.cuda.synchronize()
        if sdpa.attn_get_last_error() != 0:
            raise RuntimeError("device status set during the end-to-end steps")
        e_ms = reduce(a.elapsed_time(b), world, "max")
        e_flops = reduce(float(fwd.flops) * args.e2e_steps, world, "sum")
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcq))
        d2h = sum(t.numel() * t.element_size() for t in (ho[0], hm[0], hl[0]))
        line["e2e"] = {"value": e_flops / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "steps": args.e2e_steps, "what": "attn_fwd with pinned-host inputs copied in "
                       "and outputs + statistics copied back, every step; steps pipelined over two "
                       "buffer sets and three streams (copy in, compute, copy out)"}
    if not args.no_next_rows:
        line["next_rows"] = next_rows(fwd, csr, rank, stream, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(fwd.inp, args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_op(args):
    """One operation alone, `--warmup` + `--steps` times, for profiling it (no timing printed)."""
    sdpa.load_library()
    if args.op == "band":
        fwd = FwdCase(W.cfg3_varlen_gqa(seed=0, max_len=args.max_len))
        i = fwd.inp

        def fn():
            sdpa.attn_fwd_masked(fwd.q, fwd.k, fwd.v, cu_seqlens_q=fwd.cq, cu_seqlens_kv=fwd.ck, B=i.B,
                                 Sq=i.Sq, Skv=i.Skv, Nq=i.Nq, Nkv=i.Nkv, Dqk=i.D, Dv=i.D, scale=i.scale,
                                 mask_mode=sdpa.ATTN_MASK_BAND, pre_tokens=1023, next_tokens=0,
                                 dtype=i.dtype, layout=i.layout, out=fwd.out, softmax_max=fwd.m,
                                 softmax_sum=fwd.l)
    else:  # the tensor-core CSR from a plan: each step builds the plan and runs the call
        c = CsrCase(W.cfg4_csr(seed=0))
        ci = c.inp
        qb, kb, vb = (t.to(torch.bfloat16) for t in (c.q, c.k, c.v))
        outb = torch.empty_like(qb)
        plan = torch.empty(sdpa.attn_csr_plan_size(B=ci.B, H=ci.H, S=ci.S, nnz_cap=ci.nnz_cap),
                           dtype=torch.uint8, device="cuda")

        def fn():
            sdpa.attn_csr_plan(c.off, c.col, B=ci.B, H=ci.H, S=ci.S, nnz_cap=ci.nnz_cap, plan=plan)
            sdpa.attn_sparse_csr_tc_planned(qb, kb, vb, plan, B=ci.B, H=ci.H, S=ci.S, D=ci.D,
                                            nnz_cap=ci.nnz_cap, dtype=W.BF16, out=outb)
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    if sdpa.attn_get_last_error() != 0:
        raise RuntimeError("device status set")
    print(json.dumps({"op": args.op, "launches": args.warmup + args.steps}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--max-len", type=int, default=8192, help="max sequence length of the varlen batch")
    ap.add_argument("--parts", default="fwd,csr,merge", help="operations in a step (fwd always runs)")
    ap.add_argument("--e2e-steps", type=int, default=24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip timing the ring fold, the band and the tensor-core CSR")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=2048, help="oracle rows per reference step")
    ap.add_argument("--op", choices=["band", "csr_tc_planned"], default=None,
                    help="run only this operation (for profiling it), no timing line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.op is not None:
        torch.cuda.set_device(0)
        run_op(args)
        return
    rank, world, local = dist_setup(use_gpu=args.impl != "reference")
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1 and args.impl != "reference":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
