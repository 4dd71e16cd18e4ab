"""Host-side checks of the test helpers themselves (no GPU): the structural token
selection used for the largest parity cases covers what it promises."""
import numpy as np

import workloads as W
from oracle import ffn as offn
from tests.helpers import structural_tokens


def test_structural_selection_covers_slab_ends_tile_ends_and_coolest_expert():
    sh = W.LayerShape(256, 128, 16, 0, 12, 1, 4)
    counts = [300, 0, 177, 41, 9]
    inp = W.make_custom_inputs(sh, counts, 300, seed=5, zipf_s=1.1)
    ort = offn.route_inputs(inp)
    sel = set(structural_tokens(ort, counts, 64, sh.num_local_experts).tolist())
    assert len(sel) >= 64
    base = np.concatenate([[0], np.cumsum(counts)])
    for m, n in enumerate(counts):
        if n:
            assert base[m] in sel and base[m + 1] - 1 in sel
    for e in range(ort.counts.size):
        c, o = int(ort.counts[e]), int(ort.offsets[e])
        if c:
            for r in (o, o + ((c - 1) // 128) * 128, o + c - 1):
                assert ort.row_token[r] in sel
    routed = ort.counts[:sh.num_local_experts]
    act = np.flatnonzero(routed)
    cool = act[np.argmin(routed[act])]
    assert set(ort.row_token[ort.offsets[cool]:ort.offsets[cool + 1]].tolist()) <= sel
    # a workload no larger than the budget is checked on every token
    assert np.array_equal(structural_tokens(ort, counts, 10_000, sh.num_local_experts),
                          np.arange(ort.num_tokens))
