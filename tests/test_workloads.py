"""The seeded input generator's power-of-two scale option (CPU).

Power-of-two workloads draw the same numbers as their fp32-scale twins; only each block
scale is rounded up to a power of two, and the codes are taken against it. The tiling that
runs W13 on the block-scale MMA path relies on that property, so it is checked here.
"""
import numpy as np
import torch

import workloads as W


def _is_pow2(a: np.ndarray) -> bool:
    b = a.astype(np.float32).view(np.uint32)
    e = (b >> 23) & 0xFF
    return bool(np.all((b & 0x807FFFFF) == 0) and np.all(e > 0) and np.all(e < 255))


def test_pow2_ceil_exact():
    s = torch.tensor([1.0, 0.5, 0.75, 3.0, 4.0, 1e-30, 2.0 ** -126, 1.0000001], dtype=torch.float32)
    want = torch.tensor([1.0, 0.5, 1.0, 4.0, 4.0, 2.0 ** -99, 2.0 ** -126, 2.0], dtype=torch.float32)
    assert torch.equal(W._pow2_ceil(s), want)


def _dequant(codes, scale, rb, cb):
    x = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return x * np.kron(scale.astype(np.float64), np.ones((rb, cb)))


def test_pow2_workload_scales_and_values():
    a = W.make_inputs(W.CONFIGS["tiny"])
    b = W.make_inputs(W.CONFIGS["tiny_pow2"])
    for sa, sb in [(a.w13_scale, b.w13_scale), (a.w2_scale, b.w2_scale),
                   (a.slabs[0].x_scale, b.slabs[0].x_scale)]:
        assert _is_pow2(sb)
        assert np.all(sb >= sa) and np.all(sb < 2 * sa)
    # same draws: the two quantisations of each value differ by at most the coarser
    # grid's rounding, half an e4m3 step (2^-3 relative) of the block's largest scale
    for e in range(a.shape.num_weight_experts):
        da = _dequant(a.w13[e], a.w13_scale[e], 128, 128)
        db = _dequant(b.w13[e], b.w13_scale[e], 128, 128)
        bound = np.kron(b.w13_scale[e].astype(np.float64), np.ones((128, 128))) * 448 * 2.0 ** -3
        assert np.all(np.abs(da - db) <= bound)
    da = _dequant(a.slabs[1].x, a.slabs[1].x_scale, 1, 128)
    db = _dequant(b.slabs[1].x, b.slabs[1].x_scale, 1, 128)
    assert np.all(np.abs(da - db) <= np.kron(b.slabs[1].x_scale.astype(np.float64), np.ones((1, 128))) * 448 * 2.0 ** -3)
    # routing and weights are the same draws
    for sa, sb in zip(a.slabs, b.slabs):
        assert np.array_equal(sa.topk_ids, sb.topk_ids) and np.array_equal(sa.topk_weights, sb.topk_weights)
