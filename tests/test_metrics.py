"""Host-side FLOP and byte counting used by bench.py, against brute force on small cases."""
import numpy as np
import torch

from scaled_dot_product_16_b200 import metrics as M
from scaled_dot_product_16_b200 import workloads as W


def _brute(lens_q, lens_k, vis):
    return sum(1 for lq, lk in zip(lens_q, lens_k) for i in range(lq) for j in range(lk) if vis(i, j, lq, lk))


def test_visible_pairs_and_band_pairs_brute_force():
    lq, lk = [5, 0, 9, 4], [7, 3, 9, 0]
    for mode, vis in [(W.MASK_NONE, lambda i, j, a, b: True),
                      (W.MASK_CAUSAL_TOPLEFT, lambda i, j, a, b: j <= i),
                      (W.MASK_CAUSAL_BOTTOMRIGHT, lambda i, j, a, b: j <= i + b - a)]:
        inp = W.varlen_tnd(lq, 2, 1, 8, causal=False, dtype=torch.float32, seed=1, cfg=1,
                           lengths_kv=lk, mask_mode=mode)
        assert M.visible_pairs(inp) == _brute(lq, lk, vis)
        assert M.attn_fwd_flops(inp) == 4 * 2 * 8 * _brute(lq, lk, vis)
    inp = W.varlen_tnd(lq, 2, 1, 8, causal=False, dtype=torch.float32, seed=1, cfg=1, lengths_kv=lk)
    for pre, nxt in [(0, 0), (3, 1), (-2, 4), (100, 100), (2, -1)]:
        assert M.band_pairs(inp, pre, nxt) == _brute(lq, lk, lambda i, j, a, b: i - pre <= j <= i + nxt)


def test_csr_flops_and_merge_bytes():
    offs, cols = W.window_stride_pattern(300, half_window=8, stride=100)
    inp = W.CsrInputs(*(torch.zeros(1) for _ in range(3)), np.broadcast_to(offs, (2, 3, 301)).copy(),
                      np.broadcast_to(cols, (2, 3, cols.shape[0])).copy(), 2, 3, 300, 16)
    assert M.csr_flops(inp) == 4 * 16 * 6 * int(offs[-1])
    assert M.merge_bytes(8192, 4, 32, 128, 2) == 1_006_632_960
