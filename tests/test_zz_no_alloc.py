"""The allocation-free routing entry point against the existing entry point.

afd_ffn_route_noalloc serves callers that cannot call cudaMalloc when they run the layer
(for example a serving engine whose memory pool already holds nearly all of HBM, or a
step loop that must not stall on an allocation): its scratch is a fixed device array in
the library. This test runs the regular afd_ffn_layer, reads its routing back, and checks
that two consecutive calls of the allocation-free entry point produce the same routing
arrays bit for bit (the tolerance the other routing tests use: exact). It sits in its own
file, collected last, and passes both alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import workloads as W
from tests.helpers import run_cuda_layer

pytestmark = pytest.mark.gpu


CASES = [
    ("tiny", lambda: W.make_inputs(W.CONFIGS["tiny"])),
    ("shared_zipf_ragged", lambda: W.make_custom_inputs(W.LayerShape(768, 384, 24, 8, 10, 1, 6),
                                                         [129, 255, 1, 0], 256, seed=2, zipf_s=1.0)),
    ("no_shared_bad_ids", lambda: W.make_custom_inputs(W.LayerShape(256, 128, 16, 4, 8, 0, 3),
                                                        [40, 3], 40, seed=3)),
]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_noalloc_routing_matches_layer_two_calls(name, make):
    from attention_ffn_disaggregated_b200.device import to_device_counts, to_device_slabs
    from attention_ffn_disaggregated_b200.ffn import route_noalloc
    inp = make()
    if name == "no_shared_bad_ids":
        inp.slabs[0].topk_ids[0] = [4, 4, 99]
    ref = run_cuda_layer(inp)
    rt = ref["routing"]
    slabs = to_device_slabs(inp)
    counts = to_device_counts(inp)
    for call in range(2):
        out = route_noalloc(inp.shape, slabs, counts)
        torch.cuda.synchronize()
        o = {k: v.cpu().numpy() for k, v in out.items()}
        T, R = int(o["sizes"][0]), int(o["sizes"][1])
        K = inp.shape.top_k
        assert T == rt["num_tokens"] and R == rt["num_rows"], call
        # m-tiles: 128-row GEMM tiles over all groups; the last entry is documented as 0
        assert int(o["sizes"][2]) == int(np.sum((rt["counts"] + 127) // 128)), call
        assert int(o["sizes"][3]) == 0, call
        assert np.array_equal(o["counts"], rt["counts"])
        assert np.array_equal(o["offsets"], rt["offsets"])
        assert np.array_equal(o["row_token"][:R], rt["row_token"])
        assert np.array_equal(o["row_k"][:R], rt["row_k"])
        assert np.array_equal(o["row_weight"][:R].view(np.uint32), rt["row_weight"].view(np.uint32))
        assert np.array_equal(o["pos"][:T * K], rt["pos"])
        assert int(o["status"][0]) == ref["status_word"], call
