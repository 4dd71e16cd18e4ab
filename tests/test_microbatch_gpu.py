"""Two ping-pong microbatches on two streams (FastAFD, "Methodology / System Design",
item 4: each attention GPU splits its decode batch into k = 2 microbatches, so that the
FFN pool runs one microbatch's expert layer while the attention GPUs work on the other;
"Ablation Results": k = 2 gives the lowest latency on NVL72).

On the FFN GPU the two microbatches arrive in two sets of receive slabs and are served by
two plans over the same weights (each plan owns its workspace), launched on two streams
in alternation. Every microbatch's output must match the oracle run on that microbatch,
on every step, whatever the interleaving.
"""
import pytest
import torch

import workloads as W
from tests.helpers import compare_layer

pytestmark = pytest.mark.gpu


def _microbatches(shape, counts, cap, steps, seed):
    """steps x 2 microbatch inputs with one weight set (the first draw's)."""
    out = []
    base = None
    for i in range(2 * steps):
        inp = W.make_custom_inputs(shape, counts[i % len(counts)], cap, seed=seed + i, zipf_s=1.0,
                                   weights=base)
        if base is None:
            base = (inp.w13, inp.w13_scale, inp.w2, inp.w2_scale)
        out.append(inp)
    return out


@pytest.mark.parametrize("shape,counts,cap", [
    (W.LayerShape(512, 256, 16, 0, 12, 1, 4), [[96, 50, 7], [0, 96, 31], [13, 13, 13]], 96),
    (W.LayerShape(768, 384, 32, 8, 8, 1, 6), [[200, 0], [129, 200], [1, 1]], 200),
])
def test_two_microbatches_alternate_on_two_streams(shape, counts, cap):
    from attention_ffn_disaggregated_b200 import FfnLayer
    from attention_ffn_disaggregated_b200.device import (gather_outputs, to_device_counts,
                                                          to_device_slabs, to_device_weights)
    steps = 3
    inputs = _microbatches(shape, counts, cap, steps, seed=70)
    M = len(counts[0])
    w = to_device_weights(inputs[0])
    plans = [FfnLayer(shape, M, cap, *w) for _ in range(2)]     # one weight set, two workspaces
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    dev = [(to_device_slabs(inp), to_device_counts(inp)) for inp in inputs]
    torch.cuda.synchronize()
    # step s: microbatch A on stream 0 and B on stream 1, running concurrently; each plan's
    # calls stay ordered on its own stream. After each step both microbatches are checked
    # (the intermediate a plan keeps is its last call's).
    for s in range(steps):
        for mb in range(2):
            slabs, cnt = dev[2 * s + mb]
            with torch.cuda.stream(streams[mb]):
                plans[mb](slabs, cnt, stream=streams[mb])
        torch.cuda.synchronize()
        for mb in range(2):
            inp = inputs[2 * s + mb]
            codes, scales = plans[mb].intermediate(streams[mb])
            compare_layer({"outs": [gather_outputs(inp, dev[2 * s + mb][0])],
                           "routing": plans[mb].routing(streams[mb]), "h_codes": codes,
                           "h_scales": scales}, inp)
            rc, word = plans[mb].status(streams[mb])
            assert rc == 0, word
