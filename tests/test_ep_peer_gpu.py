"""The peer-memory EP exchange on one GPU, through the kernels: one rank (NCCL, world size
1), so that the receive buffers and the accumulators that the exchange maps are this GPU's
own. Per step the exchange copies the slabs into the receive buffers, the FFN layer's down
projection adds every token's weighted rows into the owner's accumulators (combine
targets), and afd_combine_finalize rounds the sums to bf16 into the owner's output rows.
The outputs must match the oracle on every token, on two consecutive steps (the second
starts from the accumulators that the first one cleared). What one GPU cannot show is the
transport between GPUs; the exchange logic with two ranks is tested on the CPU
(tests/test_ep_peer_gloo.py)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import workloads as W
from tests.helpers import compare_layer

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_peer_exchange_one_rank_through_the_kernels():
    from attention_ffn_disaggregated_b200 import FfnLayer
    from attention_ffn_disaggregated_b200.device import gather_outputs, to_device_weights
    from attention_ffn_disaggregated_b200.ep import PeerEpExchange
    from attention_ffn_disaggregated_b200.ffn import combine_finalize

    dist.init_process_group("nccl", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{_free_port()}",
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        shape = W.LayerShape(512, 256, 16, 0, 16, 1, 4)
        counts, cap = [100, 0, 37], 128
        ex = PeerEpExchange(len(counts), cap, shape.hidden, shape.top_k, "cuda")
        layer = None
        for step in range(2):
            inp = W.make_custom_inputs(shape, counts, cap, seed=51 + step, zipf_s=1.0,
                                       weights=None if layer is None else w_np)
            if layer is None:
                w_np = (inp.w13, inp.w13_scale, inp.w2, inp.w2_scale)
                layer = FfnLayer(shape, len(counts), cap, *to_device_weights(inp))
                layer.set_combine_targets(ex.targets)
            for m, sl in enumerate(inp.slabs):
                ex.send[m].x.copy_(torch.from_numpy(sl.x))
                ex.send[m].x_scale.copy_(torch.from_numpy(sl.x_scale))
                ex.send[m].topk_ids.copy_(torch.from_numpy(sl.topk_ids))
                ex.send[m].topk_weights.copy_(torch.from_numpy(sl.topk_weights))
            ex.send_counts.copy_(torch.tensor(counts, dtype=torch.int32))
            ex.out.fill_(float("nan"))
            ex.step(lambda recv, cnt, targets: layer(recv, cnt),
                    lambda slabs, cnt, accs: combine_finalize(slabs, cnt, accs))
            torch.cuda.synchronize()
            rc, word = layer.status()
            assert rc == 0, word
            codes, scales = layer.intermediate()
            compare_layer({"outs": [gather_outputs(inp, ex.send)], "routing": layer.routing(),
                           "h_codes": codes, "h_scales": scales}, inp)
            assert max(float(a.abs().max()) for a in ex.accs) == 0.0
        layer.close()
    finally:
        dist.destroy_process_group()
