"""The peer-memory EP exchange (attention_ffn_disaggregated_b200.ep.PeerEpExchange) on the
CPU: gloo, world sizes 2 and 4, shared-memory tensors standing in for peer-mapped device memory.

Each rank owns two slabs of tokens (its attention side) and 1/world of the experts (its
FFN side; the shared expert on rank 0); world sizes 2 and 4. Per step: every rank copies
its slabs into every rank's receive buffers, each FFN rank adds its partial rows for every received token
straight into the owning rank's fp32 accumulators (the ranks take turns here; on GPUs the
down projection's reductions are atomic), and after a barrier each owner rounds its sums to
bf16 and clears them. Checked on two consecutive steps: each owner's outputs are exactly
the bf16 of the fp32 sum of all shards' partials, and within the row tolerance of the full
layer with all experts on one GPU. The layer is played by the oracle (the kernels' side of
this path, adding into shared accumulators, is tested on one GPU in
tests/test_ep_shards_gpu.py).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W

FULL = W.LayerShape(256, 128, 8, 0, 8, 1, 3)
CAP = 12
COUNTS = {0: [7, 12], 1: [0, 5], 2: [12, 1], 3: [3, 0]}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _shard_inputs(weights, rank, world, slabs, counts):
    per = FULL.num_experts_global // world
    sh = W.LayerShape(FULL.hidden, FULL.intermediate, FULL.num_experts_global, rank * per, per,
                      1 if rank == 0 else 0, FULL.top_k)
    idx = list(range(sh.expert_begin, sh.expert_begin + sh.num_local_experts)) + \
        ([FULL.num_local_experts] if sh.has_shared_expert else [])
    w13, w13s, w2, w2s = weights
    return W.LayerInputs(sh, w13[idx], w13s[idx], w2[idx], w2s[idx], slabs, np.asarray(counts, np.int32), CAP)


def _worker(rank, world, port, out_q):
    torch.multiprocessing.set_sharing_strategy("file_system")
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_ffn_disaggregated_b200.ep import PeerEpExchange
        from oracle import ffn as offn
        base = W.make_custom_inputs(FULL, [1], CAP, seed=29)
        weights = (base.w13, base.w13_scale, base.w2, base.w2_scale)
        ex = PeerEpExchange(len(COUNTS[rank]), CAP, FULL.hidden, FULL.top_k, "cpu")

        def layer_fn(recv, counts, targets):
            slabs = [W.Slab(s.x.numpy().copy(), s.x_scale.numpy().copy(), s.topk_ids.numpy().copy(),
                            s.topk_weights.numpy().copy()) for s in recv]
            part = offn.ffn_layer(_shard_inputs(weights, rank, world, slabs, counts.numpy()))["out"]
            for turn in range(world):
                if turn == rank:
                    g = 0
                    for t, n in zip(targets, counts.tolist()):
                        t[:n] += torch.from_numpy(part[g:g + n].astype(np.float32))
                        g += n
                dist.barrier()

        def finalize_fn(slabs, counts, accs):
            for s, n, a in zip(slabs, counts.tolist(), accs):
                s.y[:n] = a[:n].to(torch.bfloat16)
                a.zero_()

        results = []
        for step in range(2):
            mine = W.make_custom_inputs(FULL, COUNTS[rank], CAP, seed=30 + 10 * step + rank, weights=weights)
            for m, sl in enumerate(mine.slabs):
                ex.send[m].x.copy_(torch.from_numpy(sl.x))
                ex.send[m].x_scale.copy_(torch.from_numpy(sl.x_scale))
                ex.send[m].topk_ids.copy_(torch.from_numpy(sl.topk_ids))
                ex.send[m].topk_weights.copy_(torch.from_numpy(sl.topk_weights))
            ex.send_counts.copy_(torch.tensor(COUNTS[rank], dtype=torch.int32))
            out = ex.step(layer_fn, finalize_fn)
            n_mine = COUNTS[rank]
            got = np.concatenate([out[m, :n].float().numpy() for m, n in enumerate(n_mine)])
            # expected, from the definition: the shards' partials for this rank's tokens,
            # each rounded to fp32 and added in rank order in fp32, then one bf16 rounding
            parts = [offn.ffn_layer(_shard_inputs(weights, f, world, mine.slabs, n_mine))["out"].astype(np.float32)
                     for f in range(world)]
            acc = np.zeros_like(parts[0])
            for p in parts:
                acc = (acc + p).astype(np.float32)
            exact = torch.from_numpy(acc).to(torch.bfloat16).float().numpy()
            full = offn.ffn_layer(mine)["out"]
            left = max(float(a.abs().max()) for a in ex.accs)
            results.append((got, exact, full, left))
        out_q.put((rank, results))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_peer_exchange_adds_partials_into_the_owners_accumulators(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, steps in res:
        for got, exact, full, left in steps:
            assert left == 0.0                                # accumulators cleared
            assert np.array_equal(got, exact), rank
            rms = np.sqrt((full ** 2).mean(axis=1))
            ok = rms > 0
            assert np.all(np.abs(got - full).max(axis=1)[ok] <= 2e-2 * rms[ok]), rank
