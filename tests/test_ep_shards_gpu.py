"""Expert-parallel sharding on the GPU path: two FFN shards over the same slabs.

An FFN pool shards the experts: each GPU holds a disjoint id range [e0, e0 + E_l), skips
the ids it does not hold, and returns a partial sum that the attention side adds up (the
M2N push-back). Here both shards run on one GPU, as two plans with the same slabs: shard
A holds experts 0..7 and the shared expert, shard B experts 8..15. The sum of their bf16
partial outputs must match the oracle's full layer (all 16 experts + shared) within the
row tolerance; each partial must also match the oracle run on its own shard.
"""
import numpy as np
import pytest

import workloads as W
from oracle import ffn as offn
from oracle import fp8 as ofp8
from tests.helpers import TOL_ROW_RMS, compare_layer, reconcile_codes, run_cuda_layer

pytestmark = pytest.mark.gpu


def _shard(full, shape, lo, hi, with_shared):
    """The full model's inputs restricted to the weights of experts [lo, hi) (+ shared)."""
    idx = list(range(lo, hi)) + ([full.shape.num_local_experts] if with_shared else [])
    return W.LayerInputs(shape, full.w13[idx], full.w13_scale[idx], full.w2[idx], full.w2_scale[idx],
                         full.slabs, full.counts, full.capacity)


@pytest.mark.parametrize("counts,cap,zipf", [([200, 37, 0, 129], 200, None), ([512, 300], 512, 1.0)])
def test_two_expert_shards_sum_to_the_full_layer(counts, cap, zipf):
    H, I, Eg, K = 512, 256, 16, 4
    full = W.make_custom_inputs(W.LayerShape(H, I, Eg, 0, Eg, 1, K), counts, cap, seed=41, zipf_s=zipf)
    a = _shard(full, W.LayerShape(H, I, Eg, 0, 8, 1, K), 0, 8, True)
    b = _shard(full, W.LayerShape(H, I, Eg, 8, 8, 0, K), 8, 16, False)
    parts, refs = [], []
    for shard in (a, b):
        res = run_cuda_layer(shard)
        assert res["status_rc"] == 0
        compare_layer(res, shard)
        parts.append(ofp8.bf16_from_bits(res["outs"][0]))
        # the shard's oracle with the GPU's midpoint decisions (if any) taken over
        o = offn.ffn_layer(shard, keep_intermediates=True)
        rows = np.arange(o["routing"].num_rows)
        codes, _ = reconcile_codes(res["h_codes"], res["h_scales"], o["h32"], o["h_codes"],
                                   o["h_scales"], rows)
        refs.append(offn.down_and_combine(shard, o["routing"], codes, o["h_scales"]))
    # the full layer is the sum of the shards' partial sums (the oracle's own pin of this is
    # in the CPU tests); the GPU's two bf16 partials must add up to it
    ref = refs[0] + refs[1]
    total = parts[0] + parts[1]
    rms = np.sqrt((ref ** 2).mean(axis=1))
    err = np.abs(total - ref).max(axis=1)
    # two bf16 roundings instead of one: the same row tolerance still holds comfortably
    assert np.all(err <= TOL_ROW_RMS * rms), float((err / rms).max())


@pytest.mark.parametrize("counts,cap,zipf,shared_on_a", [
    ([200, 37, 0, 129], 200, None, True),
    ([96, 5], 128, 1.0, False),      # no shared expert: tokens that touch no held expert
])
def test_shards_add_into_the_owners_accumulators(counts, cap, zipf, shared_on_a):
    """The return path fused into the down projection: both shards' plans add their weighted
    expert rows straight into one set of per-slab fp32 accumulators (on an expert-parallel
    pool these are the owning attention rank's buffers, reached through peer pointers), and
    the owner's finalisation rounds each token's sum once to bf16 and clears the buffers.
    Run twice, so that the second step starts from the cleared accumulators."""
    import torch
    from attention_ffn_disaggregated_b200 import FfnLayer, kernels_per_layer
    from attention_ffn_disaggregated_b200.device import (gather_outputs, to_device_counts,
                                                          to_device_slabs, to_device_weights)
    from attention_ffn_disaggregated_b200.ffn import combine_finalize
    from tests.helpers import compare_outputs

    H, I, Eg, K = 512, 256, 16, 4
    S = 1 if shared_on_a else 0
    full = W.make_custom_inputs(W.LayerShape(H, I, Eg, 0, Eg, S, K), counts, cap, seed=43, zipf_s=zipf)
    a = _shard(full, W.LayerShape(H, I, Eg, 0, 8, S, K), 0, 8, bool(S))
    b = _shard(full, W.LayerShape(H, I, Eg, 8, 8, 0, K), 8, 16, False)
    slabs = to_device_slabs(full)
    cnt = to_device_counts(full)
    accs = [torch.zeros((cap, H), dtype=torch.float32, device="cuda") for _ in counts]
    layers = [FfnLayer(sh.shape, len(counts), cap, *to_device_weights(sh)) for sh in (a, b)]
    for L in layers:
        n0 = kernels_per_layer(L)
        L.set_combine_targets(accs)
        assert kernels_per_layer(L) == n0 - 1          # no finalisation launch
    for step in range(2):
        for s in slabs:
            s.y.fill_(float("nan"))
        for L in layers:
            L(slabs, cnt)
        # the plans write no slab output of their own
        torch.cuda.synchronize()
        assert all(bool(torch.isnan(s.y[:n].float()).all()) for s, n in zip(slabs, counts) if n)
        combine_finalize(slabs, cnt, accs)
        torch.cuda.synchronize()
        y = gather_outputs(full, slabs)
        # the oracle: each shard's partial on that shard's codes (the GPU's midpoint
        # decisions taken over), added in float64
        ref = 0.0
        for L, shard in zip(layers, (a, b)):
            assert L.status()[0] == 0
            codes_g, scales_g = L.intermediate()
            o = offn.ffn_layer(shard, keep_intermediates=True)
            rows = np.arange(o["routing"].num_rows)
            codes, _ = reconcile_codes(codes_g, scales_g, o["h32"], o["h_codes"], o["h_scales"], rows)
            ref = ref + offn.down_and_combine(shard, o["routing"], codes, o["h_scales"])
        compare_outputs(y, ref)
        for acc, n in zip(accs, counts):
            assert float(acc.abs().max()) == 0.0             # cleared for the next step
    # targets removed: the plan writes its own bf16 partial again
    layers[0].set_combine_targets(None)
    for s in slabs:
        s.y.fill_(float("nan"))
    layers[0](slabs, cnt)
    torch.cuda.synchronize()
    compare_layer({"outs": [gather_outputs(a, slabs)], "routing": layers[0].routing(),
                   "h_codes": layers[0].intermediate()[0], "h_scales": layers[0].intermediate()[1]}, a)
    for L in layers:
        L.close()
