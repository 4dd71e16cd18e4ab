"""Shared helpers for the GPU parity tests: run the CUDA layer, compare with the oracle."""
from __future__ import annotations

import numpy as np

from oracle import ffn as offn
from oracle import fp8 as ofp8

# Output tolerance: each bf16 row's max-abs error against the oracle must be at most
# TOL_ROW_RMS x RMS(oracle row); rows whose oracle RMS is zero must be exactly zero.
TOL_ROW_RMS = 2e-2


def run_cuda_layer(inp, calls: int = 1, layer=None, tiling: int = 0):
    """Plan (unless given), run `calls` times on the current stream, return outputs/routing.
    tiling: 0 = default (1), 1 = single-CTA tiles, W13 and W2 as two launches, 2 = CTA-pair
    tiles, 3 = single-CTA tiles with the W13 rows gathered from the slabs, 4 = single-CTA
    tiles, W13 and W2 in one persistent launch, 5 = W13 on the block-scale MMA path
    (power-of-two scales only)."""
    import torch
    from attention_ffn_disaggregated_b200 import FfnLayer
    from attention_ffn_disaggregated_b200.device import (gather_outputs, to_device_counts,
                                                          to_device_slabs, to_device_weights)
    own = layer is None
    if own:
        w = to_device_weights(inp)
        layer = FfnLayer(inp.shape, len(inp.slabs), inp.capacity, *w)
    layer.set_tiling(tiling)
    slabs = to_device_slabs(inp)
    counts = to_device_counts(inp)
    outs = []
    for _ in range(calls):
        for s in slabs:
            s.y.fill_(float("nan"))
        layer(slabs, counts)
        torch.cuda.synchronize()
        outs.append(gather_outputs(inp, slabs))
    rc, word = layer.status()
    rt = layer.routing()
    res = {"outs": outs, "status_rc": rc, "status_word": word, "routing": rt, "layer": layer,
           "slabs": slabs, "tiling": layer.tiling()}
    return res


def compare_routing(gpu_rt: dict, ort) -> None:
    """Bit-exact comparison of every routing array."""
    assert gpu_rt["num_tokens"] == ort.num_tokens
    assert gpu_rt["num_rows"] == ort.num_rows
    assert np.array_equal(gpu_rt["counts"], ort.counts)
    assert np.array_equal(gpu_rt["offsets"], ort.offsets)
    assert np.array_equal(gpu_rt["row_token"], ort.row_token)
    assert np.array_equal(gpu_rt["row_k"], ort.row_k)
    assert np.array_equal(gpu_rt["row_weight"].view(np.uint32), ort.row_weight.view(np.uint32))
    assert np.array_equal(gpu_rt["pos"], ort.pos)


def compare_outputs(gpu_bits: np.ndarray, oracle_out: np.ndarray, tokens=None, tol=TOL_ROW_RMS):
    """gpu_bits: uint16 bf16 [T, H]; oracle_out: float64 [n, H] for `tokens` (default all)."""
    g = ofp8.bf16_from_bits(gpu_bits if tokens is None else gpu_bits[np.asarray(tokens)])
    ref = oracle_out
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), "non-finite outputs"
    rms = np.sqrt((ref ** 2).mean(axis=1))
    err = np.abs(g - ref).max(axis=1) if ref.size else np.zeros(0)
    zero = rms == 0
    assert np.all(g[zero] == 0), "rows with no contribution must be exactly zero"
    ratio = err[~zero] / rms[~zero]
    worst = float(ratio.max()) if ratio.size else 0.0
    assert worst <= tol, f"worst row error {worst:.4g} x RMS (tolerance {tol})"
    return worst


def structural_tokens(ort, slab_counts, n_total: int, num_routed_groups: int,
                      seed: int = 0) -> np.ndarray:
    """Tokens whose rows cover the layer's structure, for workloads too large to check
    every token against the oracle (all tokens when T <= n_total):

      * the first and last token of every non-empty slab (slab boundaries);
      * for every group with rows: the tokens of its first row, of the first row of its
        last 128-row tile and of its last row (ragged last tiles);
      * every token routed to the coolest active routed expert;
      * random tokens up to n_total.
    """
    T = ort.num_tokens
    if T <= n_total:
        return np.arange(T)
    sel = set()
    base = np.concatenate([[0], np.cumsum(np.asarray(slab_counts, np.int64))])
    for m in range(len(slab_counts)):
        if slab_counts[m] > 0:
            sel.update((int(base[m]), int(base[m + 1]) - 1))
    counts, offsets, row_token = ort.counts, ort.offsets, ort.row_token
    for e in range(counts.size):
        c = int(counts[e])
        if c == 0:
            continue
        o = int(offsets[e])
        sel.update(int(row_token[r]) for r in (o, o + ((c - 1) // 128) * 128, o + c - 1))
    routed = counts[:num_routed_groups]
    active = np.flatnonzero(routed > 0)
    if active.size:
        e = int(active[np.argmin(routed[active])])
        sel.update(int(t) for t in row_token[offsets[e]:offsets[e + 1]])
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.fromiter(sel, np.int64))
    need = max(0, n_total - len(sel))
    if need:
        sel.update(int(t) for t in rng.choice(rest, size=min(need, rest.size), replace=False))
    return np.array(sorted(sel), np.int64)
