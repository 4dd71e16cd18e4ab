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
    tiling: 0 = default (1), 1 = software-promoted block-FP8 GEMMs, 2 = W13 on the
    block-scale MMA path (power-of-two scales only)."""
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
    h_codes, h_scales = layer.intermediate()
    res = {"outs": outs, "status_rc": rc, "status_word": word, "routing": rt, "layer": layer,
           "slabs": slabs, "tiling": layer.tiling(), "h_codes": h_codes, "h_scales": h_scales}
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


# ----------------------------------------------------------------------------------------
# FP8 decisions with two correct answers
# ----------------------------------------------------------------------------------------
# The intermediate h is requantised to e4m3 per (row, 128 channels). Both sides take the
# decision in float32, but on h values that differ in the last bits (the GPU accumulates
# the K loop in fp32 in tile order, the oracle in float64): where h/scale lies within that
# noise of a rounding midpoint between two e4m3 values, either code is a correct result
# of the method, and one flipped large code moves an output row by up to ~3e-2 x RMS (the
# oracle with 3e-7 relative noise on h shows this on the DeepSeek-V3 share). So the codes
# are compared first: every GPU code that differs from the oracle's must be the adjacent
# e4m3 value on the other side of a midpoint that the oracle's h/scale lies within
# MIDPOINT_WINDOW of; the outputs are then compared, at the stated tolerance, with the
# oracle's second half evaluated on those codes.
MIDPOINT_WINDOW = 2e-5          # relative to max(|midpoint|, 8) in units of the scale
MAX_FLIP_FRACTION = 1e-4


def _e4m3_rank():
    """Rank of every code among the distinct finite e4m3 values (+0 and -0 share one;
    NaN codes get -10**6 so they are never adjacent to anything)."""
    from oracle import fp8 as f
    vals = f.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = np.isfinite(vals)
    uniq = np.unique(vals[finite])
    rank = np.full(256, -10 ** 6, np.int64)
    rank[finite] = np.searchsorted(uniq, vals[finite])
    return rank, vals


def reconcile_codes(gpu_codes, gpu_scales, h32, ora_codes, ora_scales, rows):
    """Check the GPU's intermediate against the oracle's on `rows`; return the oracle codes
    with the GPU's boundary decisions taken over, and the number of such decisions.
    Raises AssertionError for any difference that is not a midpoint case."""
    rank, vals = _e4m3_rank()
    rows = np.asarray(rows, np.int64)
    gs, os_ = gpu_scales[rows], ora_scales[rows]
    assert np.all(np.abs(gs - os_) <= 1e-4 * os_), "intermediate block scales differ"
    gc, oc = gpu_codes[rows], ora_codes[rows]
    # codes of equal value (+0 and -0) are the same decision
    diff = np.argwhere((gc != oc) & (vals[gc] != vals[oc]))
    codes = ora_codes.copy()
    if diff.size == 0:
        return codes, 0
    assert diff.shape[0] <= max(4, MAX_FLIP_FRACTION * gc.size), f"{diff.shape[0]} intermediate codes differ"
    r, c = diff[:, 0], diff[:, 1]
    a, b = oc[r, c], gc[r, c]
    s = os_[r, c // 128].astype(np.float32)
    ratio = (h32[rows[r], c] / s).astype(np.float32).astype(np.float64)

    def examples(mask):
        i = np.flatnonzero(mask)[:5]
        return [(int(rows[r[j]]), int(c[j]), hex(int(a[j])), hex(int(b[j])), float(ratio[j])) for j in i]

    adjacent = np.abs(rank[a] - rank[b]) == 1
    assert np.all(adjacent), f"a differing code is not the adjacent e4m3 value (row, col, oracle, gpu, h/s): {examples(~adjacent)}"
    mid = 0.5 * (vals[a] + vals[b])
    dist = np.abs(ratio - mid) / np.maximum(np.abs(mid), 8.0)
    near = dist <= MIDPOINT_WINDOW
    assert np.all(near), f"a differing code is {dist.max():.3g} from the midpoint: {examples(~near)}"
    codes[rows[r], c] = b
    return codes, int(diff.shape[0])


def compare_layer(res, inp, tokens=None, routing=None, tol=TOL_ROW_RMS):
    """Routing bit-exact; intermediate codes equal except midpoint cases (checked);
    every output of every call within `tol` x RMS of the oracle evaluated with those codes.
    Returns (worst row error, number of midpoint codes taken over)."""
    rt = routing if routing is not None else offn.route_inputs(inp)
    compare_routing(res["routing"], rt)
    ref = offn.ffn_layer(inp, tokens=tokens, routing=rt, keep_intermediates=True)
    toks = ref["tokens"]
    want = np.zeros(rt.num_tokens, bool)
    want[toks] = True
    rows = np.flatnonzero(want[rt.row_token]) if rt.num_rows else np.zeros(0, np.int64)
    codes, flips = reconcile_codes(res["h_codes"], res["h_scales"], ref["h32"], ref["h_codes"],
                                   ref["h_scales"], rows)
    out = ref["out"] if flips == 0 else offn.down_and_combine(inp, rt, codes, ref["h_scales"], tokens=tokens)
    worst = max(compare_outputs(o, out, tokens=tokens, tol=tol) for o in res["outs"])
    return worst, flips
