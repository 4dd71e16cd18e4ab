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


def _perturbed_gpu_like(inp, rel, seed):
    """An intermediate as a GPU would produce it: the oracle's h with relative noise `rel`,
    requantised by the oracle's own rule."""
    ref = offn.ffn_layer(inp, keep_intermediates=True)
    rng = np.random.default_rng(seed)
    h = ref["h32"].astype(np.float64) * (1 + rel * rng.standard_normal(ref["h32"].shape))
    q, s, _ = offn.requant_rows(h)
    return ref, q, s


def test_reconcile_accepts_midpoint_flips_and_matches_outputs():
    from tests.helpers import reconcile_codes
    sh = W.LayerShape(512, 256, 8, 0, 8, 1, 2)
    inp = W.make_custom_inputs(sh, [300, 211], 300, seed=12, zipf_s=1.0)
    ref, q, s = _perturbed_gpu_like(inp, 1e-6, 0)
    rows = np.arange(ref["routing"].num_rows)
    codes, flips = reconcile_codes(q, s, ref["h32"], ref["h_codes"], ref["h_scales"], rows)
    assert flips > 0 and np.array_equal(codes, q)
    # unchanged oracle codes give back the oracle's own output
    same, n0 = reconcile_codes(ref["h_codes"], ref["h_scales"], ref["h32"], ref["h_codes"],
                               ref["h_scales"], rows)
    assert n0 == 0
    assert np.array_equal(offn.down_and_combine(inp, ref["routing"], same, ref["h_scales"]), ref["out"])


def test_reconcile_rejects_planted_mistakes():
    """Planted in the oracle's codes: a code two steps away, and a one-step change of an
    element that is not near a midpoint, must both be refused."""
    import pytest
    from tests.helpers import reconcile_codes
    sh = W.LayerShape(256, 128, 8, 0, 8, 0, 2)
    inp = W.make_custom_inputs(sh, [64], 64, seed=13)
    ref = offn.ffn_layer(inp, keep_intermediates=True)
    rows = np.arange(ref["routing"].num_rows)
    r, c = 3, 17
    for step in (2, 1):
        bad = ref["h_codes"].copy()
        code = int(bad[r, c])
        mag = code & 0x7F
        bad[r, c] = (code & 0x80) | (mag - step if mag >= step else mag + step)
        with pytest.raises(AssertionError):
            reconcile_codes(bad, ref["h_scales"], ref["h32"], ref["h_codes"], ref["h_scales"], rows)


def test_reconcile_treats_signed_zeros_as_equal():
    from tests.helpers import reconcile_codes
    sh = W.LayerShape(256, 128, 8, 0, 8, 0, 2)
    inp = W.make_custom_inputs(sh, [32], 32, seed=14)
    ref = offn.ffn_layer(inp, keep_intermediates=True)
    rows = np.arange(ref["routing"].num_rows)
    g = ref["h_codes"].copy()
    zero = np.argwhere(g == 0x00)
    assert zero.size, "the workload has exact zero codes"
    g[zero[0][0], zero[0][1]] = 0x80
    _, flips = reconcile_codes(g, ref["h_scales"], ref["h32"], ref["h_codes"], ref["h_scales"], rows)
    assert flips == 0
