"""The multi-process host logic on CPU with gloo, world size 2: the timing reductions bench.py
uses (max / sum over ranks) and the sequence partition of a packed varlen batch, whose per-rank
results (here from the float64 oracle) reassemble into the single-process result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from scaled_dot_product_16_b200 import sharding
        from scaled_dot_product_16_b200 import workloads as W

        out = {}
        out["max"] = bench.reduce(float(rank + 1) * 10.0, world, "max")
        out["sum"] = bench.reduce(float(rank + 1), world, "sum")
        bench.barrier(world)

        # a packed varlen batch, split across ranks by causal work
        lens = [300, 0, 17, 129, 64, 1, 200]
        inp = W.varlen_tnd(lens, 4, 2, 16, causal=True, dtype=torch.float32, seed=3, cfg=77)
        parts = sharding.balanced_partition(lens, world)
        mine = parts[rank]
        idx = sharding.local_token_index(inp.cu_q, mine)
        cu = sharding.local_cu_seqlens(inp.cu_q, mine)
        T = int(cu[-1]) if len(cu) else 0
        q, k, v = (t[torch.from_numpy(idx)] for t in (inp.q, inp.k, inp.v))
        if T:
            o, m, l = oracle.attn_fwd(q, k, v, cu_q=cu, cu_kv=cu, B=len(cu), Sq=T, Skv=T, Nq=4, Nkv=2,
                                      D=16, scale=inp.scale, mask_mode=inp.mask_mode, layout=W.TND)
        else:
            o, m, l = np.zeros((0, 4, 16)), np.zeros((0, 4)), np.zeros((0, 4))
        gathered = [None] * world
        dist.all_gather_object(gathered, (idx, o, m, l))
        if rank == 0:
            T_all = inp.Sq
            O = np.full((T_all, 4, 16), np.nan)
            Mx = np.full((T_all, 4), np.nan)
            for gi, go, gm, gl in gathered:
                O[gi], Mx[gi] = go, gm
            ref, rm, _ = oracle.attn_fwd(inp.q, inp.k, inp.v, cu_q=inp.cu_q, cu_kv=inp.cu_kv, B=inp.B,
                                         Sq=inp.Sq, Skv=inp.Skv, Nq=4, Nkv=2, D=16, scale=inp.scale,
                                         mask_mode=inp.mask_mode, layout=W.TND)
            out["reassembled_max_err"] = float(np.max(np.abs(O - ref)))
            out["stat_err"] = float(np.max(np.abs(Mx - rm)))
            out["parts"] = parts
        results[rank] = out
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, port, results), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(results)
    for r in range(world):
        assert res[r]["max"] == 20.0
        assert res[r]["sum"] == 3.0
    assert res[0]["reassembled_max_err"] == 0.0
    assert res[0]["stat_err"] == 0.0
    parts = res[0]["parts"]
    assert sorted(i for p in parts for i in p) == list(range(7))


def test_balanced_partition_properties():
    from scaled_dot_product_16_b200 import sharding
    lens = [5327, 1493, 4105, 3052, 6658, 7735, 2093, 0, 6792, 4774, 7769, 5862, 6553, 7164, 5944, 15]
    for world in (1, 2, 4, 8):
        parts = sharding.balanced_partition(lens, world)
        assert sorted(i for p in parts for i in p) == list(range(len(lens)))
        loads = [sum(sharding.sequence_work(lens[i], lens[i], True) for i in p) for p in parts]
        heaviest = max(sharding.sequence_work(l, l, True) for l in lens)
        assert max(loads) - min(loads) <= heaviest  # LPT bound
    assert sharding.sequence_work(4, 4, True) == 10
    assert sharding.sequence_work(4, 6, False) == 24
    cu = np.array([2, 4, 4, 6, 8])
    assert sharding.local_token_index(cu, [1, 3]).tolist() == [2, 3, 4, 5]
    assert sharding.local_cu_seqlens(cu, [1, 2, 3]).tolist() == [2, 2, 4]


def _ring_worker(rank, world, port, results):
    """Ring attention's schedule with a float64 CPU fold in place of the GPU one: each rank holds
    its query shard and one chunk of keys; after the ring, every rank's accumulator must equal
    attention of its queries over all ranks' keys."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from scaled_dot_product_16_b200 import ring
        from scaled_dot_product_16_b200 import workloads as W

        B, N, Sq, C, D = 2, 3, 20, 7, 16          # C keys per rank
        full = W.dense_bhsd(B, N, Sq * world, D, causal=False, dtype=torch.float32, seed=5, cfg=78,
                            Skv=C * world)
        q = full.q[:, :, rank * Sq:(rank + 1) * Sq].contiguous()
        k = full.k[:, :, rank * C:(rank + 1) * C].contiguous()
        v = full.v[:, :, rank * C:(rank + 1) * C].contiguous()
        acc = {}
        seen = []

        def cpu_fold(q, k, v, *, first, B, Sq, Skv, Nq, Nkv, D, scale, dtype, layout, cu_q, cu_kv,
                     acc_out, acc_max, acc_sum):
            seen.append(float(k[0, 0, 0, 0]))
            o, m, l = oracle.attn_fwd(q, k, v, B=B, Sq=Sq, Skv=Skv, Nq=Nq, Nkv=Nkv, D=D, scale=scale,
                                      mask_mode=0, layout=W.BHSD)
            o_sbh = o.transpose(2, 0, 1, 3).reshape(Sq, B, Nq * D)
            m8, l8 = np.repeat(m[..., None], 8, -1), np.repeat(l[..., None], 8, -1)
            if first:
                acc.update(out=o_sbh, max=m8, sum=l8)
            else:
                acc["out"], acc["max"], acc["sum"] = oracle.merge(acc["out"], acc["max"], acc["sum"], o_sbh,
                                                                  m8, l8, S=Sq, B=B, N=Nq, D=D)

        ring.ring_attention(q, k, v, B=B, Sq=Sq, Skv=C, Nq=N, Nkv=N, D=D, scale=full.scale, dtype=W.F32,
                            acc_out=None, acc_max=None, acc_sum=None, fold=cpu_fold)
        ref, rm, rl = oracle.attn_fwd(q, full.k, full.v, B=B, Sq=Sq, Skv=C * world, Nq=N, Nkv=N, D=D,
                                      scale=full.scale, mask_mode=0, layout=W.BHSD)
        got = acc["out"].reshape(Sq, B, N, D).transpose(1, 2, 0, 3)
        results[rank] = {"err": float(np.max(np.abs(got - ref))),
                         "max_err": float(np.max(np.abs(acc["max"][..., 0] - rm))),
                         "sum_err": float(np.max(np.abs(acc["sum"][..., 3] / rl - 1))),
                         "steps": len(seen), "chunks": seen}
    finally:
        dist.destroy_process_group()


def test_ring_attention_three_ranks_gloo():
    world = 3
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_ring_worker, args=(world, port, results), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(results)
    firsts = sorted(res[r]["chunks"][0] for r in range(world))
    for r in range(world):
        assert res[r]["steps"] == world
        assert res[r]["err"] <= 1e-12 and res[r]["max_err"] <= 1e-12 and res[r]["sum_err"] <= 1e-12
        # rank r folds its own chunk first, then r-1's, r-2's, ...: each chunk once
        assert sorted(res[r]["chunks"]) == firsts
        assert res[r]["chunks"][1] == res[(r - 1) % world]["chunks"][0]
