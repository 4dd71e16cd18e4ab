"""Canonical routing for the FFN-pool expert layer.

The attention side computes top-K routing and publishes expert ids and weights with the
FP8 tokens into the FFN GPU's receive buffers (FastAFD, "Methodology / System Design",
items 1-2). The FFN side groups the routed (token, slot) pairs by expert so that each
expert runs as one GEMM over its rows ("grouped GEMMs", item 3).

Definition followed here (the pages are silent on the order; this is the reading used):
  * tokens are numbered slab-major: g = sum_{m' < m} n_{m'} + t for row t of slab m;
  * pairs (g, k) are visited in ascending (g, k); slot k of token g is *local* iff
    e0 <= id < e0 + E_l, with group key le = id - e0;
  * id == -1 marks an empty slot (skipped); an id outside [0, E_g) or a repeat of an
    id already seen earlier in the same token is a routing error: it is skipped and
    reported (BAD_ROUTING);
  * counts[le] = number of local pairs with key le; offsets = exclusive prefix sum;
  * inside a group, rows keep ascending (g, k) order (a stable counting sort);
  * with a shared expert (S = 1) a final group at index E_l holds one row per token,
    in ascending g, with weight 1.0 and slot -1;
  * pos[g*K + k] = the row of pair (g, k), or -1 if it is not local.
"""
from __future__ import annotations

import dataclasses
from typing import Sequence

import numpy as np

BAD_ROUTING = 1


@dataclasses.dataclass
class Routing:
    num_tokens: int
    counts: np.ndarray      # int32 [G]   G = E_l + S
    offsets: np.ndarray     # int32 [G+1]
    row_token: np.ndarray   # int32 [R]
    row_k: np.ndarray       # int32 [R]   (-1 for shared rows)
    row_weight: np.ndarray  # float32 [R]
    pos: np.ndarray         # int32 [T*K]
    token_slab: np.ndarray  # int32 [T]
    token_row: np.ndarray   # int32 [T]
    status: int             # BAD_ROUTING bit if any bad id was seen

    @property
    def num_rows(self) -> int:
        return int(self.offsets[-1])

    def row_expert(self) -> np.ndarray:
        """Group index of every row (E_l for shared rows)."""
        return np.repeat(np.arange(self.counts.size, dtype=np.int32), self.counts)


def token_order(counts: Sequence[int]):
    """Global token index -> (slab, row) in slab-major order."""
    slab = np.concatenate([np.full(int(n), m, np.int32) for m, n in enumerate(counts)] +
                          [np.zeros(0, np.int32)])
    row = np.concatenate([np.arange(int(n), dtype=np.int32) for n in counts] +
                         [np.zeros(0, np.int32)])
    return slab, row


def route(shape, counts: Sequence[int], slab_ids: Sequence[np.ndarray],
          slab_weights: Sequence[np.ndarray]) -> Routing:
    K, e0, El, Eg, S = (shape.top_k, shape.expert_begin, shape.num_local_experts,
                        shape.num_experts_global, shape.has_shared_expert)
    tslab, trow = token_order(counts)
    T = int(tslab.size)
    G = El + S
    status = 0
    # 1. visit pairs in (g, k) order, classify
    keys = np.full(T * K, -1, dtype=np.int64)
    wts = np.zeros(T * K, dtype=np.float32)
    for g in range(T):
        ids = slab_ids[tslab[g]][trow[g]]
        ws = slab_weights[tslab[g]][trow[g]]
        seen = set()
        for k in range(K):
            i = int(ids[k])
            if i == -1:
                continue
            if i < 0 or i >= Eg or i in seen:
                status |= BAD_ROUTING
                continue
            seen.add(i)
            if e0 <= i < e0 + El:
                keys[g * K + k] = i - e0
                wts[g * K + k] = ws[k]
    # 2. histogram and exclusive scan
    counts_g = np.zeros(G, dtype=np.int64)
    for key in keys:
        if key >= 0:
            counts_g[key] += 1
    if S:
        counts_g[El] = T
    offsets = np.zeros(G + 1, dtype=np.int64)
    for i in range(G):
        offsets[i + 1] = offsets[i] + counts_g[i]
    R = int(offsets[G])
    # 3. stable placement: walk pairs in (g, k) order, append to the key's group
    fill = offsets[:G].copy()
    row_token = np.zeros(R, np.int32)
    row_k = np.zeros(R, np.int32)
    row_w = np.zeros(R, np.float32)
    pos = np.full(T * K, -1, np.int32)
    for p in range(T * K):
        key = keys[p]
        if key < 0:
            continue
        r = fill[key]
        fill[key] += 1
        pos[p] = r
        row_token[r] = p // K
        row_k[r] = p % K
        row_w[r] = wts[p]
    if S:
        for g in range(T):
            r = offsets[El] + g
            row_token[r] = g
            row_k[r] = -1
            row_w[r] = 1.0
    return Routing(T, counts_g.astype(np.int32), offsets.astype(np.int32), row_token, row_k,
                   row_w, pos, tslab, trow, status)
