"""Ring attention over a process group: one long sequence's keys split across GPUs.

"npu_ring_attention_update" (MindSpeed op doc, 功能说明) describes the update as the step that
folds one chunk's partial attention into a running result when the key/value sequence is split
across devices in a ring. Here every rank keeps its own query shard and one chunk of keys and
values. The chunks travel around the ring: at each step a rank sends the chunk it holds to rank
r + 1 and receives the next one from rank r - 1 (torch.distributed point-to-point operations; on
GPUs, NCCL over NVLink / NVSwitch). Meanwhile the rank folds the chunk it holds into its
accumulator with attn_fwd_accumulate, the fused forward + merge. After `world` steps every rank
has attention of its queries over all keys.

The transfer of step s+1's chunk runs while step s's chunk is multiplied: the receive buffer is
the one the previous step's kernel read, and the process group orders the transfer after that
kernel (the communication stream waits for the current stream when the operation is posted),
and the next kernel after the transfer (waiting on its request makes the current stream wait).

Only the non-causal form is provided: a causal ring needs per-chunk mask offsets that the fused
accumulate call does not take, and the pages' ring configuration (workload 5) is non-causal.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import attn_fwd_accumulate, ATTN_BHSD, ATTN_MASK_NONE


def _fold_on_gpu(q, k, v, *, first, B, Sq, Skv, Nq, Nkv, D, scale, dtype, layout, cu_q, cu_kv,
                 acc_out, acc_max, acc_sum):
    attn_fwd_accumulate(q, k, v, cu_seqlens_q=cu_q, cu_seqlens_kv=cu_kv, B=B, Sq=Sq, Skv=Skv, Nq=Nq,
                        Nkv=Nkv, D=D, scale=scale, mask_mode=ATTN_MASK_NONE, dtype=dtype,
                        layout=layout, first=first, acc_out=acc_out, acc_max=acc_max,
                        acc_sum=acc_sum)


def ring_attention(q, k, v, *, B: int, Sq: int, Skv: int, Nq: int, Nkv: int, D: int, scale: float,
                   dtype: int, acc_out, acc_max, acc_sum, layout: int = ATTN_BHSD, cu_seqlens_q=None,
                   cu_seqlens_kv=None, group: Optional[dist.ProcessGroup] = None,
                   fold: Optional[Callable] = None) -> None:
    """Attention of this rank's queries over the keys of every rank in `group`.

    q [B, Nq, Sq, D] (or TND) is this rank's query shard; k, v [B, Nkv, Skv, D] are this rank's
    chunk of keys and values (every rank's chunk has the same shape; for TND, the same cumulative
    lengths cu_seqlens_kv). The result goes to the accumulator in attn_merge's layouts (acc_out
    [Sq, B, Nq*D], acc_max / acc_sum [B, Nq, Sq, 8] for BHSD). `fold` replaces the fused GPU
    step (attn_fwd_accumulate) with any function of the same keyword arguments; the ring's
    schedule is the same for both.
    """
    fold = _fold_on_gpu if fold is None else fold
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    send_to = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    recv_from = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    kbuf = [k.contiguous(), torch.empty_like(k)]
    vbuf = [v.contiguous(), torch.empty_like(v)]
    for step in range(world):
        cur = step & 1
        reqs = []
        if step + 1 < world:
            ops = [dist.P2POp(dist.isend, kbuf[cur], send_to, group),
                   dist.P2POp(dist.irecv, kbuf[cur ^ 1], recv_from, group),
                   dist.P2POp(dist.isend, vbuf[cur], send_to, group),
                   dist.P2POp(dist.irecv, vbuf[cur ^ 1], recv_from, group)]
            reqs = dist.batch_isend_irecv(ops)
        fold(q, kbuf[cur], vbuf[cur], first=step == 0, B=B, Sq=Sq, Skv=Skv, Nq=Nq, Nkv=Nkv, D=D,
             scale=scale, dtype=dtype, layout=layout, cu_q=cu_seqlens_q, cu_kv=cu_seqlens_kv,
             acc_out=acc_out, acc_max=acc_max, acc_sum=acc_sum)
        for r in reqs:
            r.wait()
