"""The layer call inside a CUDA graph.

afd_ffn_layer only enqueues work on the given stream (no host synchronisation, device-side
counts), so a serving loop can capture it once and replay it every decode step, as a
whole-step CUDA graph does (FastAFD, "Methodology / System Design", item 5). The slab
contents and counts may change between replays; the replayed results must match the
oracle for each new input.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import ffn as offn
from tests.helpers import compare_layer

pytestmark = pytest.mark.gpu


def test_layer_replays_from_a_cuda_graph_with_new_inputs():
    from attention_ffn_disaggregated_b200 import FfnLayer
    from attention_ffn_disaggregated_b200.device import gather_outputs, to_device_weights
    sh = W.LayerShape(512, 256, 16, 0, 12, 1, 4)
    cap, M = 96, 3
    inputs = [W.make_custom_inputs(sh, counts, cap, seed=40 + i)
              for i, counts in enumerate(([96, 50, 7], [0, 96, 31], [13, 13, 13]))]
    for inp in inputs[1:]:                      # one weight set for the whole run
        inp.w13, inp.w13_scale, inp.w2, inp.w2_scale = (inputs[0].w13, inputs[0].w13_scale,
                                                         inputs[0].w2, inputs[0].w2_scale)
    layer = FfnLayer(sh, M, cap, *to_device_weights(inputs[0]))
    # static device buffers the graph reads and writes
    class S:
        pass
    slabs = []
    for m in range(M):
        s = S()
        s.x = torch.empty((cap, sh.hidden), dtype=torch.uint8, device="cuda")
        s.x_scale = torch.empty((cap, sh.hidden // 128), dtype=torch.float32, device="cuda")
        s.topk_ids = torch.empty((cap, sh.top_k), dtype=torch.int32, device="cuda")
        s.topk_weights = torch.empty((cap, sh.top_k), dtype=torch.float32, device="cuda")
        s.y = torch.empty((cap, sh.hidden), dtype=torch.bfloat16, device="cuda")
        slabs.append(s)
    counts = torch.empty(M, dtype=torch.int32, device="cuda")

    def load(inp):
        for s, src in zip(slabs, inp.slabs):
            s.x.copy_(torch.from_numpy(src.x))
            s.x_scale.copy_(torch.from_numpy(src.x_scale))
            s.topk_ids.copy_(torch.from_numpy(src.topk_ids))
            s.topk_weights.copy_(torch.from_numpy(src.topk_weights))
            s.y.fill_(float("nan"))
        counts.copy_(torch.from_numpy(np.asarray(inp.counts, np.int32)))

    load(inputs[0])
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        layer(slabs, counts)                    # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        layer(slabs, counts)
    for inp in inputs:
        load(inp)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        codes, scales = layer.intermediate()
        compare_layer({"outs": [gather_outputs(inp, slabs)], "routing": layer.routing(),
                       "h_codes": codes, "h_scales": scales}, inp)
    rc, word = layer.status()
    assert rc == 0, word
    del g
