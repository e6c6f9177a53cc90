"""A pipeline wait that runs out is reported as ATTN_ERR_TIMEOUT, and the device stays usable.

The test build of the library (libattn_stalltest.so: the same sources with the attention
kernel's pipeline waits bounded at 1 ms, and its MMA warp first waiting on a barrier that
nothing ever arrives on) is loaded in a child process. There the wait runs out: the block
records the timeout in the status word, stops issuing, waits (bounded at 200 ms) for the TMA
loads it already issued, frees its tensor memory and exits. Nothing faults or hangs. The child
then reads the status, reads it again (cleared), and runs an ordinary torch kernel on the same
context. Back in this process, the normal library still passes parity.
"""
import os
import subprocess
import sys

import pytest
import torch

import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import build as sdpa_build
from scaled_dot_product_16_b200 import workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
import torch
sys.path.insert(0, sys.argv[1])
import scaled_dot_product_16_b200 as sdpa
from scaled_dot_product_16_b200 import workloads as W
sdpa.lib_path = lambda: sys.argv[2]          # the test build instead of libattn.so
inp = W.varlen_tnd([300, 0, 129], 4, 2, 128, causal=True, dtype=torch.bfloat16, seed=0, cfg=97)
q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
cu = torch.from_numpy(inp.cu_q).cuda()
out = torch.zeros_like(q)
sdpa.attn_fwd(q, k, v, cu_seqlens_q=cu, cu_seqlens_kv=cu, B=inp.B, Sq=inp.Sq, Skv=inp.Skv, Nq=4,
              Nkv=2, D=128, scale=inp.scale, mask_mode=1, dtype=W.BF16, layout=W.TND, out=out)
first = sdpa.attn_get_last_error()
second = sdpa.attn_get_last_error()
after = int((torch.arange(10, device="cuda") * 2).sum().item())
print("STATUS", first, second, after, flush=True)
"""


def _inputs():
    return W.varlen_tnd([300, 0, 129], 4, 2, 128, causal=True, dtype=torch.bfloat16, seed=0, cfg=97)


def test_pipeline_wait_runs_out_and_is_reported():
    lib = sdpa_build.build_stall_test()
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, lib], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("STATUS")][-1]
    _, first, second, after = line.split()
    assert int(first) == sdpa.ATTN_ERR_TIMEOUT
    assert int(second) == sdpa.ATTN_OK      # the read cleared the word
    assert int(after) == 90                 # the child's context still runs kernels
    # the normal library, in this process, on the same problem
    inp = _inputs()
    out, m, l = G.run_fwd(inp)
    ref, rm, rl = G.oracle_fwd(inp)
    G.check_out(G.f64(out), ref, inp.dtype, abs_ref=lambda: G.oracle_abs_fwd(inp))
    G.check_stats(m.numpy(), l.numpy(), rm, rl)
