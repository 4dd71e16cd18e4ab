"""The expert-parallel exchange (attention_ffn_disaggregated_b200.ep) on the CPU: gloo,
world size 2.

Each rank owns two slabs of tokens (its attention side) and half of the experts (its FFN
side; the shared expert on rank 0). After one exchange step every rank must hold, for its
own tokens, the sum over both FFN ranks of their partial outputs: exactly the bf16 of the
fp32 sum of the two bf16 partials, and within the row tolerance of the full layer with all
experts on one GPU. The layer call is played by the oracle on the received slabs (the
exchange logic is what is tested here; the kernels' EP sharding is tested on one GPU in
tests/test_ep_shards_gpu.py).
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W

FULL = W.LayerShape(256, 128, 8, 0, 8, 1, 3)
CAP = 12
COUNTS = {0: [7, 12], 1: [0, 5]}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _shard_shape(rank, world):
    per = FULL.num_experts_global // world
    return W.LayerShape(FULL.hidden, FULL.intermediate, FULL.num_experts_global, rank * per, per,
                        1 if rank == 0 else 0, FULL.top_k)


def _shard_inputs(weights, rank, world, slabs, counts):
    sh = _shard_shape(rank, world)
    idx = list(range(sh.expert_begin, sh.expert_begin + sh.num_local_experts)) + \
        ([FULL.num_local_experts] if sh.has_shared_expert else [])
    w13, w13s, w2, w2s = weights
    return W.LayerInputs(sh, w13[idx], w13s[idx], w2[idx], w2s[idx], slabs, np.asarray(counts, np.int32), CAP)


def _rank_inputs(rank, weights):
    return W.make_custom_inputs(FULL, COUNTS[rank], CAP, seed=30 + rank, weights=weights)


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_ffn_disaggregated_b200.ep import EpExchange
        from oracle import ffn as offn
        from oracle import fp8 as ofp8
        base = W.make_custom_inputs(FULL, [1], CAP, seed=29)
        weights = (base.w13, base.w13_scale, base.w2, base.w2_scale)
        mine = _rank_inputs(rank, weights)
        ex = EpExchange(len(COUNTS[rank]), CAP, FULL.hidden, FULL.top_k, "cpu")
        for m, sl in enumerate(mine.slabs):
            ex.send[m].x.copy_(torch.from_numpy(sl.x))
            ex.send[m].x_scale.copy_(torch.from_numpy(sl.x_scale))
            ex.send[m].topk_ids.copy_(torch.from_numpy(sl.topk_ids))
            ex.send[m].topk_weights.copy_(torch.from_numpy(sl.topk_weights))
        ex.send_counts.copy_(torch.tensor(COUNTS[rank], dtype=torch.int32))

        def layer_fn(recv, counts):
            # this rank's FFN shard over every received slab, written as bf16 partials
            slabs = [W.Slab(s.x.numpy().copy(), s.x_scale.numpy().copy(), s.topk_ids.numpy().copy(),
                            s.topk_weights.numpy().copy()) for s in recv]
            part = _shard_inputs(weights, rank, world, slabs, counts.numpy())
            y = offn.ffn_layer(part)["out_bf16"]
            g = 0
            for s, n in zip(recv, counts.tolist()):
                s.y[:n] = torch.from_numpy(y[g:g + n]).to(torch.bfloat16)
                g += n

        out = ex.step(layer_fn)
        n_mine = COUNTS[rank]
        got = np.concatenate([out[m, :n].float().numpy() for m, n in enumerate(n_mine)])
        # expected, computed on this rank from the definition: every FFN shard's bf16
        # partial for this rank's tokens, summed in fp32, rounded once to bf16
        parts = [ofp8.bf16_round(offn.ffn_layer(_shard_inputs(weights, f, world, mine.slabs, n_mine))["out"])
                 for f in range(world)]
        exact = ofp8.bf16_round((parts[0].astype(np.float32) + parts[1].astype(np.float32)).astype(np.float64))
        full = offn.ffn_layer(mine)["out"]
        rows_zero = np.concatenate([out[m, n:].float().numpy().ravel() for m, n in enumerate(n_mine)])
        out_q.put((rank, got, exact, full, float(np.abs(rows_zero).max(initial=0.0))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ep_exchange_returns_the_sum_of_partials():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, got, exact, full, junk in res:
        assert junk == 0.0                                    # rows beyond n_m stay zero
        assert np.array_equal(got, exact), rank
        rms = np.sqrt((full ** 2).mean(axis=1))
        ok = rms > 0
        # two bf16 roundings (partials, then the sum): within the row tolerance
        assert np.all(np.abs(got - full).max(axis=1)[ok] <= 2e-2 * rms[ok]), rank
