"""GPU parity: the CUDA layer (through the C ABI) against the CPU oracle.

Routing arrays (counts, offsets, row order, slots, weights, pos) must be bit-exact. Each
bf16 output row must satisfy max|gpu - oracle| <= 2e-2 x RMS(oracle row); rows with no
contribution must be exactly zero. Sizes here span several 128-row and 256-column tiles
with ragged tails; the full-size workloads are checked on sampled tokens.
"""
import numpy as np
import torch
import pytest

import workloads as W
from oracle import ffn as offn
from tests.helpers import compare_layer, compare_outputs, run_cuda_layer, structural_tokens

pytestmark = pytest.mark.gpu


def _full_check(inp, calls=1, tiling=0):
    """Every output row of every call against the oracle (tests.helpers.compare_layer)."""
    res = run_cuda_layer(inp, calls=calls, tiling=tiling)
    rt = offn.route_inputs(inp)
    worst, flips = compare_layer(res, inp, routing=rt)
    return res, rt, worst


def test_tiny_config():
    inp = W.make_inputs(W.CONFIGS["tiny"])
    res, ref, _ = _full_check(inp)
    assert res["status_rc"] == 0


@pytest.mark.parametrize("seed,shape,counts,cap,zipf", [
    (1, W.LayerShape(512, 256, 16, 0, 16, 0, 4), [300, 0, 177, 41], 300, None),
    (2, W.LayerShape(768, 384, 24, 8, 10, 1, 6), [129, 255, 1], 256, 1.0),
    (3, W.LayerShape(1024, 512, 8, 0, 8, 1, 2), [1000], 1000, 0.5),
    (4, W.LayerShape(256, 128, 64, 0, 64, 0, 8), [513, 77, 0, 3, 250], 513, 1.2),
])
def test_random_shapes_several_tiles(seed, shape, counts, cap, zipf):
    inp = W.make_custom_inputs(shape, counts, cap, seed=seed, zipf_s=zipf)
    res, _, _ = _full_check(inp)
    assert res["status_rc"] == 0


@pytest.mark.parametrize("seed,shape,counts,cap", [
    # experts of a few hundred rows with ragged last tiles, an empty slab, a single token
    (21, W.LayerShape(512, 256, 4, 0, 4, 1, 2), [300, 217, 0, 65], 300),
    (22, W.LayerShape(768, 384, 6, 0, 6, 0, 3), [511, 2], 511),
    (23, W.LayerShape(1024, 256, 16, 4, 6, 1, 4), [1, 0, 130], 130),
])
def test_ragged_tiles_two_calls(seed, shape, counts, cap):
    inp = W.make_custom_inputs(shape, counts, cap, seed=seed, zipf_s=1.0)
    res, _, _ = _full_check(inp, calls=2)
    assert res["tiling"] == 1
    assert res["status_rc"] == 0


# Small batches: when the gate/up projection's tiles fill at most half of the GPU, each
# tile's K blocks are shared out among CTAs (split-K) and the CTA that completes a tile's
# rows finishes SwiGLU + requantisation from the fp32 sums. H = 1024 or 2048 gives 8 or 16
# K blocks per tile (two splits or more). Three calls check that the split workspace and
# its counters are clear again after every call.
@pytest.mark.parametrize("shape,counts,cap", [
    (W.LayerShape(1024, 1024, 8, 0, 8, 0, 2), [3], 3),
    (W.LayerShape(1024, 1024, 8, 0, 8, 0, 2), [1, 0, 16], 16),
    (W.LayerShape(1024, 1024, 16, 4, 8, 1, 4), [5, 2], 5),
    (W.LayerShape(2048, 1024, 8, 0, 6, 1, 3), [1], 1),
])
def test_split_k_small_batches(shape, counts, cap):
    inp = W.make_custom_inputs(shape, counts, cap, seed=51, zipf_s=1.0)
    res, _, _ = _full_check(inp, calls=3)
    assert res["status_rc"] == 0


# The ABI's limits in one layer: 1024 groups (1023 local experts + shared), top-K 32 and
# 128 slabs of two tokens each.
_LIMITS_SHAPE = W.LayerShape(256, 128, 1024, 0, 1023, 1, 32)


def test_limits_groups_topk_slabs():
    inp = W.make_custom_inputs(_LIMITS_SHAPE, [2] * 128, 2, seed=31)
    res, ref, _ = _full_check(inp, calls=1)
    assert res["status_rc"] == 0
    # id 1023 is not held here, so a token that picked it has 31 local rows + shared
    assert 256 * 31 < ref.num_rows <= 256 * 33


# Tiling 2: W13 on the block-scale MMA path, for power-of-two block scales. The oracle is
# the same; only the inputs' scales are rounded up to powers of two.
@pytest.mark.parametrize("seed,shape,counts,cap", [
    (21, W.LayerShape(512, 256, 4, 0, 4, 1, 2), [300, 217, 0, 65], 300),
    (22, W.LayerShape(768, 384, 6, 0, 6, 0, 3), [511, 2], 511),
    (23, W.LayerShape(1024, 256, 16, 4, 6, 1, 4), [1, 0, 130], 130),
    (24, W.LayerShape(1024, 512, 8, 0, 8, 1, 2), [1000], 1000),
])
def test_block_scale_tiling(seed, shape, counts, cap):
    inp = W.make_custom_inputs(shape, counts, cap, seed=seed, zipf_s=1.0, pow2_scales=True)
    res, _, _ = _full_check(inp, calls=2, tiling=2)
    assert res["tiling"] == 2
    assert res["status_rc"] == 0


def test_block_scale_tiling_limits():
    inp = W.make_custom_inputs(_LIMITS_SHAPE, [2] * 128, 2, seed=31, pow2_scales=True)
    res, _, _ = _full_check(inp, calls=1, tiling=2)
    assert res["tiling"] == 2 and res["status_rc"] == 0


def test_block_scale_tiling_refuses_other_weight_scales():
    """amax/448 W13 scales are not powers of two: selecting the block-scale tiling is
    refused synchronously, the plan keeps its tiling and the next call is correct."""
    from attention_ffn_disaggregated_b200 import AfdError, FfnLayer
    from attention_ffn_disaggregated_b200.device import to_device_weights
    inp = W.make_inputs(W.CONFIGS["tiny"])
    layer = FfnLayer(inp.shape, len(inp.slabs), inp.capacity, *to_device_weights(inp))
    with pytest.raises(AfdError) as e:
        layer.set_tiling(2)
    assert e.value.code == 1
    res = run_cuda_layer(inp, layer=layer)
    assert res["status_rc"] == 0 and res["tiling"] == 1
    compare_layer(res, inp)


def test_block_scale_tiling_flags_activation_scales_on_every_call():
    """Power-of-two W13 scales but amax/448 activation scales: every tiling-2 call sets
    BAD_SCALE, also after afd_ffn_get_status has cleared the word."""
    from attention_ffn_disaggregated_b200 import FfnLayer
    from attention_ffn_disaggregated_b200.device import (to_device_counts, to_device_slabs,
                                                          to_device_weights)
    from attention_ffn_disaggregated_b200.ffn import STATUS_BAD_SCALE
    sh = W.LayerShape(256, 128, 8, 0, 8, 1, 2)
    wts = W.make_custom_inputs(sh, [40], 40, seed=41, pow2_scales=True)
    acts = W.make_custom_inputs(sh, [40], 40, seed=41)
    layer = FfnLayer(sh, 1, 40, *to_device_weights(wts))
    layer.set_tiling(2)
    slabs, counts = to_device_slabs(acts), to_device_counts(acts)
    for _ in range(2):
        layer(slabs, counts)
        rc, word = layer.status()
        assert rc == 1 and word & STATUS_BAD_SCALE


def test_repeated_calls_self_clean():
    """The combine accumulators are zero again after every call: three calls, each correct."""
    inp = W.make_custom_inputs(W.LayerShape(512, 256, 12, 2, 8, 1, 4), [200, 90], 200, seed=7)
    res, _, _ = _full_check(inp, calls=3)
    assert len(res["outs"]) == 3


def test_empty_batch_and_empty_slabs():
    sh = W.LayerShape(256, 128, 8, 0, 8, 1, 2)
    inp = W.make_custom_inputs(sh, [0, 0, 0], 4, seed=8)
    res = run_cuda_layer(inp)
    assert res["routing"]["num_tokens"] == 0 and res["routing"]["num_rows"] == 0
    assert res["status_rc"] == 0
    inp = W.make_custom_inputs(sh, [0, 1, 0], 4, seed=9)
    _full_check(inp)


def test_no_local_contribution_rows_are_zero():
    """Without a shared expert, tokens whose ids are all non-local get exact zeros."""
    sh = W.LayerShape(256, 128, 16, 8, 4, 0, 2)
    inp = W.make_custom_inputs(sh, [6], 6, seed=10)
    inp.slabs[0].topk_ids[:6] = [[0, 1], [8, 2], [15, -1], [-1, -1], [9, 11], [3, 4]]
    res, ref, _ = _full_check(inp)
    out = res["outs"][0]
    assert np.all(out[0] == 0) and np.all(out[2] == 0) and np.all(out[3] == 0) and np.all(out[5] == 0)


def test_bad_ids_duplicates_and_counts_set_status():
    sh = W.LayerShape(256, 128, 8, 0, 8, 1, 3)
    inp = W.make_custom_inputs(sh, [5, 3], 5, seed=11)
    inp.slabs[0].topk_ids[1] = [2, 2, 9]      # repeat and out of range
    inp.slabs[1].topk_ids[0] = [-7, 1, 3]     # negative, not -1
    res, ref, _ = _full_check(inp)
    assert res["status_word"] & 0x1
    assert res["status_rc"] == 5               # AFD_ERR_BAD_ROUTING


def test_count_above_capacity_is_clamped_and_flagged():
    import torch
    from attention_ffn_disaggregated_b200 import FfnLayer
    from attention_ffn_disaggregated_b200.device import (gather_outputs, to_device_slabs,
                                                          to_device_weights)
    sh = W.LayerShape(256, 128, 8, 0, 8, 0, 2)
    inp = W.make_custom_inputs(sh, [4, 4], 4, seed=12)
    layer = FfnLayer(sh, 2, 4, *to_device_weights(inp))
    slabs = to_device_slabs(inp)
    layer(slabs, torch.tensor([9, 4], dtype=torch.int32, device="cuda"))
    rc, word = layer.status()
    assert word & 0x4 and rc == 5
    # counts clamp to capacity: the same layer as counts [4, 4]
    codes, scales = layer.intermediate()
    res = {"outs": [gather_outputs(inp, slabs)], "routing": layer.routing(), "h_codes": codes,
           "h_scales": scales}
    compare_layer(res, inp)


def test_single_token_single_slab():
    inp = W.make_custom_inputs(W.LayerShape(512, 256, 32, 0, 32, 1, 8), [1], 1, seed=13)
    _full_check(inp)


def test_intermediate_codes_match_oracle():
    """The intermediate itself: every FP8 code equal to the oracle's, or the adjacent value
    across a rounding midpoint that the oracle's h/scale lies within float32 noise of;
    block scales within 1e-4 relative."""
    from tests.helpers import reconcile_codes
    inp = W.make_custom_inputs(W.LayerShape(512, 256, 8, 0, 8, 0, 2), [160, 100], 160, seed=14)
    res = run_cuda_layer(inp)
    ref = offn.ffn_layer(inp, keep_intermediates=True)
    R = ref["routing"].num_rows
    assert res["h_codes"].shape == (R, 256)
    reconcile_codes(res["h_codes"], res["h_scales"], ref["h32"], ref["h_codes"], ref["h_scales"],
                    np.arange(R))


def test_timeout_injection_reports_status_and_recovers():
    """A stage that is never filled makes the bounded wait expire: TIMEOUT, no hang, and
    the next call on the same plan is correct again."""
    inp = W.make_custom_inputs(W.LayerShape(256, 128, 8, 0, 8, 1, 2), [64], 64, seed=15)
    res = run_cuda_layer(inp)
    layer = res["layer"]
    layer.set_wait_limit(50_000_000)
    layer.inject_stall(True)
    stalled = run_cuda_layer(inp, layer=layer)
    assert stalled["status_word"] & 0x2 and stalled["status_rc"] == 6
    layer.set_wait_limit(1_000_000_000)
    again = run_cuda_layer(inp, layer=layer)
    assert again["status_rc"] == 0
    compare_layer(again, inp)


# ------------------------------------------------------------------ full-size workloads

def _full_size_check(inp, n_total=None, tiling=0):
    """Routing bit-exact on every token; intermediate and outputs against the oracle on
    every token, or on the structural selection of tests.helpers.structural_tokens when
    n_total is given."""
    res = run_cuda_layer(inp, tiling=tiling)
    assert res["status_rc"] == 0, res["status_word"]
    ort = offn.route_inputs(inp)
    toks = (None if n_total is None else
            structural_tokens(ort, inp.counts, n_total, inp.shape.num_local_experts))
    worst, flips = compare_layer(res, inp, tokens=toks, routing=ort)
    print(f"worst row error {worst:.4f} x RMS, {flips} midpoint codes")
    return worst, res


@pytest.mark.parametrize("name,tiling", [("qwen3_235b_t2048", 0), ("deepseek_v3_share_t4096", 0),
                                         ("qwen3_235b_spec_q4_t8192", 0),
                                         ("deepseek_v3_share_t4096_pow2", 2)])
def test_full_size_every_token(name, tiling):
    """The three full-size workloads (and the block-scale tiling on the power-of-two twin of
    the DeepSeek-V3 share): every output row against the oracle."""
    _, res = _full_size_check(W.make_inputs(W.CONFIGS[name]), tiling=tiling)
    assert res["tiling"] == (1 if tiling == 0 else tiling)


# --------------------------------------------------------------- sweep cells (T x M)

@pytest.fixture(scope="module")
def share_weights():
    """One weight set of the DeepSeek-V3 share shape for the sweep cells (as bench.py's
    sweep uses), generated once for the module."""
    return W.make_weights(W.DEEPSEEK_V3_SHARE, torch.Generator().manual_seed(4))


@pytest.mark.parametrize("cell", ["sweep_t1_m64_uniform", "sweep_t8_m16_zipf1.2", "sweep_t64_m4_uniform",
                                  "sweep_t512_m1_uniform", "sweep_t512_m64_zipf1.2",
                                  "sweep_t512_m64_uniform", "sweep_t512_m1_zipf1.2",
                                  "sweep_t4096_m1_uniform", "sweep_t4096_m64_zipf1.2",
                                  "sweep_t4096_m64_uniform", "sweep_t4096_m1_zipf1.2"])
def test_sweep_cells_every_token(cell, share_weights):
    """Cells of the T x M sweep up to 4096 tokens, every output row against the oracle: a
    single token among 64 slabs (63 empty), skewed and uniform routing, one slab holding
    every token and 64 slabs of 8 to 64 tokens."""
    _full_size_check(W.make_inputs(W.workload_by_name(cell), weights=share_weights))


@pytest.mark.parametrize("cell", ["sweep_t16384_m1_uniform", "sweep_t16384_m64_zipf1.2",
                                  "sweep_t16384_m64_uniform", "sweep_t16384_m1_zipf1.2"])
def test_sweep_cells_16384_structural(cell, share_weights):
    """The 16384-token cells (up to ~110k routed rows): routing on every token, outputs on
    the structural selection (slab ends, every group's first row and both ends of its last
    tile, all tokens of the coolest expert) topped up to 2048 tokens."""
    _full_size_check(W.make_inputs(W.workload_by_name(cell), weights=share_weights), n_total=2048)
