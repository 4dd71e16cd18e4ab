"""The FFN-pool expert layer, written as a plain float64 CPU computation.

Follows FastAFD, "Methodology / System Design", item 3 (the FFN GPU runs block-FP8
grouped GEMMs with the activation between them and pushes results back to the attention
ranks) and the vLLM AFD plugin's "FFN service" (receive activations and metadata, compute
the FFN output, return it). Readings of what the pages leave open:

  * activation = SwiGLU: h = silu(g) * u with g = first I outputs of W13 (gate), u = the
    next I (up);
  * both GEMMs are block-FP8, so h is requantised to e4m3fn per row per 128 channels with
    scale = amax/448 (scale 1 for an all-zero block) before W2. The quantisation decision
    (the division h/scale and the rounding to e4m3) is taken in float32, the precision the
    GPU kernel takes it in; everything else is float64;
  * combine: out[g] = sum over local slots k (ascending) of w[g,k] * Y[row of (g,k)]
    + S * Y[shared row of g], rounded once to bf16 (RNE); a token with no contribution
    gets exact zeros. topk_weights are used as given (renormalised over all K ids by the
    router), so the result is this GPU's partial sum.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .fp8 import E4M3_MAX, bf16_round, e4m3_decode, e4m3_encode
from .routing import Routing, route

QB = 128


def dequant_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Activation rows: value[r, c] = dec(code[r, c]) * scale[r, c // 128]."""
    return e4m3_decode(codes) * np.repeat(np.asarray(scales, np.float64), QB, axis=1)


def dequant_weight(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Weight matrix [N, C]: value[n, c] = dec(code[n, c]) * scale[n // 128, c // 128]."""
    s = np.repeat(np.repeat(np.asarray(scales, np.float64), QB, axis=0), QB, axis=1)
    return e4m3_decode(codes) * s


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """silu(g) * u = g * u / (1 + exp(-g))."""
    return g * u / (1.0 + np.exp(-g))


def requant_rows(h: np.ndarray):
    """Per row, per 128 channels: s = amax/448 (1 if amax == 0); q = e4m3(h/s).

    Returns (codes uint8 [n, C], scales float32 [n, C/128], dequantised float64 [n, C]).
    The decision is taken in float32.
    """
    h32 = np.asarray(h, np.float32)
    n, C = h32.shape
    hb = h32.reshape(n, C // QB, QB)
    amax = np.abs(hb).max(axis=2) if n else np.zeros((0, C // QB), np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    ratio = (hb / s[:, :, None]).astype(np.float32)
    q = e4m3_encode(ratio)
    hq = e4m3_decode(q) * s[:, :, None].astype(np.float64)
    return q.reshape(n, C), s, hq.reshape(n, C)


def expert_forward(x: np.ndarray, w13: np.ndarray, w2: np.ndarray, I: int):
    """One expert on dequantised rows x [r, H] with dequantised W13 [2I, H], W2 [H, I]."""
    G = x @ w13.T
    h = swiglu(G[:, :I], G[:, I:])
    q, s, hq = requant_rows(h)
    return hq @ w2.T, q, s


def gather_tokens(inp, routing: Routing):
    """Codes and scales of every token in global (slab-major) order."""
    H = inp.shape.hidden
    T = routing.num_tokens
    xc = np.zeros((T, H), np.uint8)
    xs = np.zeros((T, H // QB), np.float32)
    for g in range(T):
        sl = inp.slabs[routing.token_slab[g]]
        xc[g] = sl.x[routing.token_row[g]]
        xs[g] = sl.x_scale[routing.token_row[g]]
    return xc, xs


def route_inputs(inp) -> Routing:
    return route(inp.shape, inp.counts, [s.topk_ids for s in inp.slabs],
                 [s.topk_weights for s in inp.slabs])


def _wanted_rows(rt: Routing, e: int, want: np.ndarray) -> np.ndarray:
    r0, r1 = int(rt.offsets[e]), int(rt.offsets[e + 1])
    rows = np.arange(r0, r1)
    return rows[want[rt.row_token[rows]]]


def _combine(rt: Routing, Y: np.ndarray, toks: np.ndarray, K: int, El: int, S: int) -> np.ndarray:
    """out[g] = sum over local slots k (ascending) of w[g,k] * Y[pos[g,k]] + S * Y[shared
    row of g], in float64."""
    out = np.zeros((toks.size, Y.shape[1]), np.float64)
    for i, g in enumerate(toks):
        acc = np.zeros(Y.shape[1], np.float64)
        for k in range(K):
            r = rt.pos[g * K + k]
            if r >= 0:
                acc += np.float64(rt.row_weight[r]) * Y[r]
        if S:
            acc += Y[rt.offsets[El] + g]
        out[i] = acc
    return out


def _want(rt: Routing, tokens) -> tuple:
    T = rt.num_tokens
    toks = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    want = np.zeros(T, bool)
    want[toks] = True
    return toks, want


def ffn_layer(inp, tokens: Optional[Sequence[int]] = None, routing: Optional[Routing] = None,
              keep_intermediates: bool = False):
    """Grouped form: rows grouped by expert, one dense product per expert.

    Returns a dict with 'out' (float64 [n, H], before bf16 rounding), 'out_bf16'
    (float64 values of the bf16 result), 'tokens' (the global token ids of the rows of
    'out'), 'routing', and optionally per-row 'h32' (the float32 intermediate the
    quantisation decision is taken on), 'h_codes' / 'h_scales' and 'Y'. Rows of tokens
    outside `tokens` are left zero.
    """
    sh = inp.shape
    H, I, El, S = sh.hidden, sh.intermediate, sh.num_local_experts, sh.has_shared_expert
    rt = routing if routing is not None else route_inputs(inp)
    toks, want = _want(rt, tokens)
    xc, xs = gather_tokens(inp, rt)
    R = rt.num_rows
    Y = np.zeros((R, H), np.float64)
    if keep_intermediates:
        h32 = np.zeros((R, I), np.float32)
        h_codes = np.zeros((R, I), np.uint8)
        h_scales = np.zeros((R, I // QB), np.float32)
    for e in range(El + S):
        rows = _wanted_rows(rt, e, want)
        if rows.size == 0:
            continue
        x = dequant_rows(xc[rt.row_token[rows]], xs[rt.row_token[rows]])
        w13 = dequant_weight(inp.w13[e], inp.w13_scale[e])
        w2 = dequant_weight(inp.w2[e], inp.w2_scale[e])
        G = x @ w13.T
        h = swiglu(G[:, :I], G[:, I:])
        q, s, hq = requant_rows(h)
        Y[rows] = hq @ w2.T
        if keep_intermediates:
            h32[rows], h_codes[rows], h_scales[rows] = h.astype(np.float32), q, s
    out = _combine(rt, Y, toks, sh.top_k, El, S)
    res = {"out": out, "out_bf16": bf16_round(out), "tokens": toks, "routing": rt}
    if keep_intermediates:
        res.update(h32=h32, h_codes=h_codes, h_scales=h_scales, Y=Y)
    return res


def down_and_combine(inp, routing: Routing, h_codes: np.ndarray, h_scales: np.ndarray,
                     tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """The layer's second half from a given intermediate: for every row of the wanted
    tokens, Y = dequant(h_codes, h_scales) . W2_f^T of its expert, then the combine.
    With the codes and scales ffn_layer computes itself this returns its 'out' exactly.
    Returns float64 [n, H] before bf16 rounding."""
    sh = inp.shape
    H, El, S = sh.hidden, sh.num_local_experts, sh.has_shared_expert
    rt = routing
    toks, want = _want(rt, tokens)
    Y = np.zeros((rt.num_rows, H), np.float64)
    for e in range(El + S):
        rows = _wanted_rows(rt, e, want)
        if rows.size == 0:
            continue
        w2 = dequant_weight(inp.w2[e], inp.w2_scale[e])
        Y[rows] = dequant_rows(h_codes[rows], h_scales[rows]) @ w2.T
    return _combine(rt, Y, toks, sh.top_k, El, S)


def ffn_layer_bruteforce(inp) -> np.ndarray:
    """Per-token twin: no permutation, one expert evaluation per (token, slot).

    Applies the same slot rules independently: -1 skipped; ids outside [0, E_g) or
    repeated within the token skipped; only ids in [e0, e0+E_l) contribute here.
    Returns float64 [T, H] before bf16 rounding.
    """
    sh = inp.shape
    H, I, K = sh.hidden, sh.intermediate, sh.top_k
    e0, El, Eg, S = sh.expert_begin, sh.num_local_experts, sh.num_experts_global, sh.has_shared_expert
    outs = []
    for m, n in enumerate(inp.counts):
        sl = inp.slabs[m]
        for t in range(int(n)):
            x = dequant_rows(sl.x[t:t + 1], sl.x_scale[t:t + 1])
            acc = np.zeros(H, np.float64)
            seen = []
            for k in range(K):
                i = int(sl.topk_ids[t, k])
                if i < 0 or i >= Eg or i in seen:
                    continue
                seen.append(i)
                if not (e0 <= i < e0 + El):
                    continue
                e = i - e0
                y, _, _ = expert_forward(x, dequant_weight(inp.w13[e], inp.w13_scale[e]),
                                         dequant_weight(inp.w2[e], inp.w2_scale[e]), I)
                acc += np.float64(sl.topk_weights[t, k]) * y[0]
            if S:
                y, _, _ = expert_forward(x, dequant_weight(inp.w13[El], inp.w13_scale[El]),
                                         dequant_weight(inp.w2[El], inp.w2_scale[El]), I)
                acc += y[0]
            outs.append(acc)
    return np.array(outs).reshape(len(outs), H)
