"""Pins for the oracle's routing (stable counting sort of routed pairs by local expert).

Checked against a sort-based brute force (numpy's stable argsort on the composite key),
against histogram/scan invariants, and on the edge cases the layer must handle.
"""
import numpy as np
import pytest

import workloads as W
from oracle import routing


def _brute(shape, counts, ids_list, w_list):
    """Enumerate all pairs, keep valid local ones, stable-sort by expert key."""
    K, e0, El, Eg, S = (shape.top_k, shape.expert_begin, shape.num_local_experts,
                        shape.num_experts_global, shape.has_shared_expert)
    keys, toks, ks, ws, bad = [], [], [], [], False
    g = 0
    for m, n in enumerate(counts):
        for t in range(n):
            row = list(ids_list[m][t])
            for k in range(K):
                i = row[k]
                if i == -1:
                    continue
                if not (0 <= i < Eg) or i in row[:k]:
                    bad = True
                    continue
                if e0 <= i < e0 + El:
                    keys.append(i - e0)
                    toks.append(g)
                    ks.append(k)
                    ws.append(w_list[m][t][k])
            g += 1
    keys = np.array(keys, np.int64)
    order = np.argsort(keys, kind="stable")
    T = g
    rt = np.array(toks, np.int64)[order] if keys.size else np.zeros(0, np.int64)
    rk = np.array(ks, np.int64)[order] if keys.size else np.zeros(0, np.int64)
    rw = np.array(ws, np.float32)[order] if keys.size else np.zeros(0, np.float32)
    cnt = np.bincount(keys, minlength=El) if keys.size else np.zeros(El, np.int64)
    if S:
        rt = np.concatenate([rt, np.arange(T)])
        rk = np.concatenate([rk, -np.ones(T, np.int64)])
        rw = np.concatenate([rw, np.ones(T, np.float32)])
        cnt = np.concatenate([cnt, [T]])
    return rt, rk, rw, cnt, bad


def _check(shape, counts, ids_list, w_list):
    r = routing.route(shape, counts, ids_list, w_list)
    rt, rk, rw, cnt, bad = _brute(shape, counts, ids_list, w_list)
    assert np.array_equal(r.counts, cnt)
    assert np.array_equal(r.offsets, np.concatenate([[0], np.cumsum(cnt)]))
    assert np.array_equal(r.row_token, rt)
    assert np.array_equal(r.row_k, rk)
    assert np.array_equal(r.row_weight, rw)
    assert bool(r.status & routing.BAD_ROUTING) == bad
    # pos is a bijection from local pairs onto the routed (non-shared) rows
    K = shape.top_k
    local_rows = r.pos[r.pos >= 0]
    n_local = int(r.offsets[shape.num_local_experts])
    assert np.array_equal(np.sort(local_rows), np.arange(n_local))
    for p in np.nonzero(r.pos >= 0)[0]:
        row = r.pos[p]
        assert r.row_token[row] == p // K and r.row_k[row] == p % K
    # stability: inside each group rows ascend in (g, k)
    for e in range(r.counts.size):
        a, b = r.offsets[e], r.offsets[e + 1]
        key = r.row_token[a:b].astype(np.int64) * (K + 1) + (r.row_k[a:b] + 1)
        assert np.all(np.diff(key) > 0)
    return r


@pytest.mark.parametrize("name", ["tiny"])
def test_route_tiny_config(name):
    inp = W.make_inputs(W.CONFIGS[name])
    _check(inp.shape, inp.counts, [s.topk_ids for s in inp.slabs], [s.topk_weights for s in inp.slabs])


@pytest.mark.parametrize("seed", range(6))
def test_route_random_shapes(seed):
    rng = np.random.default_rng(seed)
    Eg = int(rng.integers(4, 40))
    El = int(rng.integers(0, Eg + 1))
    e0 = int(rng.integers(0, Eg - El + 1))
    S = int(rng.integers(0, 2))
    if El + S == 0:
        S = 1
    K = int(rng.integers(1, min(Eg, 8) + 1))
    sh = W.LayerShape(128, 128, Eg, e0, El, S, K)
    M = int(rng.integers(1, 6))
    cap = int(rng.integers(1, 20))
    counts = [int(rng.integers(0, cap + 1)) for _ in range(M)]
    ids = [rng.integers(-1, Eg, size=(cap, K)).astype(np.int32) for _ in range(M)]
    ws = [rng.random((cap, K)).astype(np.float32) for _ in range(M)]
    _check(sh, counts, ids, ws)


def test_route_bad_ids_and_duplicates():
    sh = W.LayerShape(128, 128, 8, 2, 4, 1, 4)
    ids = [np.array([[2, 3, 2, -1],      # duplicate 2 -> the second is skipped
                     [9, 5, -5, 0],      # 9 and -5 out of range
                     [0, 1, 6, 7]],      # all non-local
                    np.int32)]
    ws = [np.arange(12, dtype=np.float32).reshape(3, 4)]
    r = _check(sh, [3], ids, ws)
    assert r.status & routing.BAD_ROUTING
    assert list(r.counts) == [1, 1, 0, 1, 3]   # ids 2,3,4,5 local; shared
    assert r.pos[2] == -1 and r.pos[0] == 0


def test_route_empty():
    sh = W.LayerShape(128, 128, 8, 0, 8, 1, 2)
    r = _check(sh, [0, 0], [np.zeros((1, 2), np.int32)] * 2, [np.zeros((1, 2), np.float32)] * 2)
    assert r.num_tokens == 0 and r.num_rows == 0


def test_route_empty_slabs_between_full_ones():
    sh = W.LayerShape(128, 128, 6, 0, 6, 0, 2)
    rng = np.random.default_rng(5)
    ids = [rng.permuted(np.tile(np.arange(6), (5, 1)), axis=1)[:, :2].astype(np.int32) for _ in range(4)]
    ws = [rng.random((5, 2)).astype(np.float32) for _ in range(4)]
    r = _check(sh, [3, 0, 5, 0], ids, ws)
    assert r.num_tokens == 8
    assert list(r.token_slab) == [0, 0, 0, 2, 2, 2, 2, 2]
