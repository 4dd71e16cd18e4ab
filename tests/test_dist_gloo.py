"""Multi-process host logic on the CPU (gloo, world size 2).

1. Expert-parallel sharding of the FFN pool: each rank holds a disjoint expert range
   [e0, e0 + E_l) (the shared expert on rank 0 only) and produces a partial output for the
   same tokens; the sum of the partials over ranks equals the layer with all experts on
   one GPU. This is the exchange step an EP-sharded FFN pool needs (a sum of partials).
2. The bench's timing rule: every rank measures its own device time and the reported
   time is the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import ffn as offn
        full_shape = W.LayerShape(256, 128, 8, 0, 8, 1, 3)
        inp = W.make_custom_inputs(full_shape, [7, 0, 12], 12, seed=21)
        per = full_shape.num_experts_global // world
        e0 = rank * per
        S = 1 if rank == 0 else 0
        sh = W.LayerShape(256, 128, 8, e0, per, S, 3)
        idx = list(range(e0, e0 + per)) + ([full_shape.num_local_experts] if S else [])
        part = W.LayerInputs(sh, inp.w13[idx], inp.w13_scale[idx], inp.w2[idx], inp.w2_scale[idx],
                             inp.slabs, inp.counts, inp.capacity)
        y = torch.from_numpy(offn.ffn_layer(part)["out"])
        dist.all_reduce(y, op=dist.ReduceOp.SUM)
        t = torch.tensor([1.5 + rank])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            full = offn.ffn_layer(inp)["out"]
            out_q.put((y.numpy(), full, float(t.item())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_expert_parallel_partials_sum_to_full_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    y, full, tmax = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    scale = np.sqrt((full ** 2).mean(axis=1, keepdims=True))
    scale[scale == 0] = 1
    assert np.max(np.abs(y - full) / scale) < 1e-9
    assert tmax == 2.5
