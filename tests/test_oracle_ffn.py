"""Pins for the oracle's layer arithmetic.

Each test fixes the oracle to something other than itself:
  * a closed-form case (constant codes, so every dot product is a sum of equal terms);
  * a dense SwiGLU FFN built only from torch routines (float8 cast, matmul, silu);
  * identical experts whose combine weights sum to 1 reproduce one expert;
  * the grouped form equals the per-token brute-force twin;
  * re-splitting the same tokens over a different number of slabs changes nothing;
  * computing a subset of tokens gives the same rows as computing all of them.
A dropped term, swapped gate/up, wrong scale index or wrong combine weight fails one.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import ffn, fp8


def _inputs_from_arrays(shape, w13, w13s, w2, w2s, slabs_x, slabs_xs, slabs_ids, slabs_w, counts):
    slabs = [W.Slab(x, xs, i, w) for x, xs, i, w in zip(slabs_x, slabs_xs, slabs_ids, slabs_w)]
    return W.LayerInputs(shape, w13, w13s, w2, w2s, slabs, np.array(counts, np.int32),
                         slabs_x[0].shape[0])


# ------------------------------------------------------------------------------- closed form

def test_closed_form_constant_codes():
    """x codes all 1.0, weight codes all 1.0: every dot product is (block size) x (scales)."""
    H, I = 256, 128
    sh = W.LayerShape(H, I, 4, 0, 2, 1, 2)
    a = {0: (0.01, 0.02), 1: (-0.02, 0.01), 2: (0.005, 0.005)}      # gate scales per col block
    b = {0: (0.03, -0.01), 1: (0.015, 0.02), 2: (0.01, 0.02)}      # up scales per col block
    c = {0: (0.002, 0.004), 1: (-0.003, 0.001), 2: (0.001, -0.002)}  # W2 scales per row block
    E = 3
    w13 = np.full((E, 2 * I, H), 0x38, np.uint8)
    w2 = np.full((E, H, I), 0x38, np.uint8)
    w13s = np.zeros((E, 2, 2), np.float32)
    w2s = np.zeros((E, 2, 1), np.float32)
    for e in range(E):
        w13s[e, 0] = a[e]
        w13s[e, 1] = b[e]
        w2s[e, :, 0] = c[e]
    xs_val = np.array([0.5, 0.25], np.float32)
    x = np.full((1, H), 0x38, np.uint8)
    xs = xs_val[None, :]
    ids = np.array([[1, 0]], np.int32)
    wts = np.array([[0.625, 0.375]], np.float32)
    inp = _inputs_from_arrays(sh, w13, w13s, w2, w2s, [x], [xs], [ids], [wts], [1])

    def expert(e):
        f32 = lambda v: float(np.float32(v))
        g = 128 * f32(xs_val[0]) * f32(a[e][0]) + 128 * f32(xs_val[1]) * f32(a[e][1])
        u = 128 * f32(xs_val[0]) * f32(b[e][0]) + 128 * f32(xs_val[1]) * f32(b[e][1])
        h = g * u / (1 + math.exp(-g))
        h32 = np.float32(h)
        s32 = np.float32(abs(h32)) / np.float32(448.0)      # amax over equal values
        hq = math.copysign(448.0, h) * float(s32)           # every element quantises to +-448
        return np.array([128 * hq * f32(c[e][0])] * 128 + [128 * hq * f32(c[e][1])] * 128)

    expect = 0.625 * expert(1) + 0.375 * expert(0) + expert(2)
    got = ffn.ffn_layer(inp)
    np.testing.assert_allclose(got["out"][0], expect, rtol=1e-12, atol=0)
    assert np.array_equal(got["out_bf16"][0], fp8.bf16_round(expect))


# ----------------------------------------------------------------------- dense torch FFN

def _torch_dense(xc, xs, w13c, w13s, w2c, w2s, I):
    dq = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).to(torch.float64)
    rep = lambda s, r, c: torch.from_numpy(s).double().repeat_interleave(r, 0).repeat_interleave(c, 1)
    x = dq(xc) * torch.from_numpy(xs).double().repeat_interleave(128, 1)
    w13 = dq(w13c) * rep(w13s, 128, 128)
    w2 = dq(w2c) * rep(w2s, 128, 128)
    G = torch.matmul(x, w13.T)
    h = torch.nn.functional.silu(G[:, :I]) * G[:, I:]
    n = h.shape[0]
    hb = h.float().reshape(n, I // 128, 128)
    amax = hb.abs().amax(-1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (hb / s[..., None]).clamp(-448, 448).to(torch.float8_e4m3fn)
    hq = (q.to(torch.float64) * s[..., None].double()).reshape(n, I)
    return torch.matmul(hq, w2.T).numpy()


def test_one_expert_top1_equals_dense_swiglu_ffn():
    H, I, T = 384, 256, 40
    sh = W.LayerShape(H, I, 1, 0, 1, 0, 1)
    inp = W.make_custom_inputs(sh, [T], T, seed=3)
    for s in inp.slabs:
        s.topk_ids[:] = 0
        s.topk_weights[:] = 1.0
    got = ffn.ffn_layer(inp)["out"]
    ref = _torch_dense(inp.slabs[0].x[:T], inp.slabs[0].x_scale[:T], inp.w13[0], inp.w13_scale[0],
                       inp.w2[0], inp.w2_scale[0], I)
    scale = np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(got - ref) / scale) < 1e-9


def test_shared_expert_only_equals_dense_ffn():
    """No local experts, S = 1: output is the dense FFN of the shared expert, weight 1."""
    H, I, T = 256, 128, 9
    sh = W.LayerShape(H, I, 16, 16, 0, 1, 4)   # router ids never local (e0 = 16 = E_g)
    inp = W.make_custom_inputs(sh, [4, 5], 5, seed=4)
    got = ffn.ffn_layer(inp)["out"]
    xc = np.concatenate([inp.slabs[0].x[:4], inp.slabs[1].x[:5]])
    xs = np.concatenate([inp.slabs[0].x_scale[:4], inp.slabs[1].x_scale[:5]])
    ref = _torch_dense(xc, xs, inp.w13[0], inp.w13_scale[0], inp.w2[0], inp.w2_scale[0], I)
    scale = np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(got - ref) / scale) < 1e-9


# ------------------------------------------------------------------- identical experts

def test_identical_experts_weights_sum_to_one():
    H, I, T, E = 256, 128, 24, 4
    sh4 = W.LayerShape(H, I, E, 0, E, 1, E)
    inp = W.make_custom_inputs(sh4, [T], T, seed=5)
    for arr in (inp.w13, inp.w13_scale, inp.w2, inp.w2_scale):
        arr[1:E] = arr[0]                      # experts 0..3 identical; shared (index 4) differs
    rng = np.random.default_rng(0)
    for s in inp.slabs:
        s.topk_ids[:] = np.stack([rng.permutation(E) for _ in range(T)])
        w = rng.random((T, E))
        s.topk_weights[:] = (w / w.sum(1, keepdims=True)).astype(np.float32)
    got = ffn.ffn_layer(inp)["out"]
    sh1 = W.LayerShape(H, I, 1, 0, 1, 1, 1)
    one = W.LayerInputs(sh1, inp.w13[[0, E]], inp.w13_scale[[0, E]], inp.w2[[0, E]],
                        inp.w2_scale[[0, E]],
                        [W.Slab(s.x, s.x_scale, np.zeros((T, 1), np.int32), np.ones((T, 1), np.float32))
                         for s in inp.slabs], inp.counts, T)
    ref = ffn.ffn_layer(one)["out"]
    wsum = np.stack([s.topk_weights.astype(np.float64).sum(1) for s in inp.slabs])[0]
    # sum_k w_k Y = (sum_k w_k) Y; the float32 weights sum to 1 within a few ulp
    assert np.max(np.abs(wsum - 1)) < 1e-6
    scale = np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(got - ref) / scale) < 1e-6


# ------------------------------------------------------------------------- brute force

def test_grouped_equals_bruteforce_tiny():
    inp = W.make_inputs(W.CONFIGS["tiny"])
    g = ffn.ffn_layer(inp)["out"]
    b = ffn.ffn_layer_bruteforce(inp)
    scale = np.sqrt((b ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(g - b) / scale) < 1e-9


def test_grouped_equals_bruteforce_with_shared_bad_ids_and_nonlocal():
    sh = W.LayerShape(256, 256, 12, 3, 5, 1, 3)
    inp = W.make_custom_inputs(sh, [5, 0, 7, 2], 7, seed=6)
    inp.slabs[0].topk_ids[1] = [4, 4, 13]       # duplicate and out-of-range
    inp.slabs[2].topk_ids[0] = [-1, 0, 11]      # empty slot, non-local ids
    g = ffn.ffn_layer(inp)
    assert g["routing"].status != 0
    b = ffn.ffn_layer_bruteforce(inp)
    scale = np.sqrt((b ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(g["out"] - b) / scale) < 1e-9


# ------------------------------------------------------------------- splitting / subsets

def test_resplitting_slabs_changes_nothing():
    inp = W.make_inputs(W.CONFIGS["tiny"])
    rt = ffn.route_inputs(inp)
    xc, xs = ffn.gather_tokens(inp, rt)
    T = rt.num_tokens
    ids = np.concatenate([inp.slabs[m].topk_ids[:n] for m, n in enumerate(inp.counts)])
    ws = np.concatenate([inp.slabs[m].topk_weights[:n] for m, n in enumerate(inp.counts)])
    base = ffn.ffn_layer(inp)["out"]
    for split in ([T], [1, 0, 20, 3, 0, 30, 10], [T // 2, 0, T - T // 2]):
        cap = max(split)
        slabs, g = [], 0
        for n in split:
            pad = lambda a: np.concatenate([a[g:g + n], np.zeros((cap - n,) + a.shape[1:], a.dtype)])
            slabs.append(W.Slab(pad(xc), pad(xs), pad(ids), pad(ws)))
            g += n
        re = W.LayerInputs(inp.shape, inp.w13, inp.w13_scale, inp.w2, inp.w2_scale, slabs,
                           np.array(split, np.int32), cap)
        assert np.array_equal(ffn.ffn_layer(re)["out"], base)


def test_token_subset_matches_full():
    inp = W.make_inputs(W.CONFIGS["tiny"])
    full = ffn.ffn_layer(inp)["out"]
    sub = ffn.ffn_layer(inp, tokens=[0, 5, 17, 63])["out"]
    ref = full[[0, 5, 17, 63]]
    # BLAS may block a 4-row product differently from a 64-row one: last-bit differences only
    scale = np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(sub - ref) / scale) < 1e-12


def test_no_contribution_rows_are_zero():
    sh = W.LayerShape(128, 128, 8, 4, 4, 0, 2)
    inp = W.make_custom_inputs(sh, [3], 3, seed=8)
    inp.slabs[0].topk_ids[:] = [[0, 1], [2, -1], [5, 1]]
    out = ffn.ffn_layer(inp)["out"]
    assert np.all(out[0] == 0) and np.all(out[1] == 0) and np.any(out[2] != 0)


# ------------------------------------------------- power-of-two block scales (inputs)

def test_grouped_equals_bruteforce_pow2_inputs():
    """The same layer definition on inputs whose block scales are powers of two (the
    inputs of the block-scale W13 tiling): grouped form and per-token twin agree."""
    inp = W.make_inputs(W.CONFIGS["tiny_pow2"])
    g = ffn.ffn_layer(inp, keep_intermediates=True)
    b = ffn.ffn_layer_bruteforce(inp)
    scale = np.sqrt((b ** 2).mean(axis=1, keepdims=True))
    assert np.max(np.abs(g["out"] - b) / scale) < 1e-9
