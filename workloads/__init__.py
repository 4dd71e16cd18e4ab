"""Seeded synthetic inputs for the FFN-pool expert layer of attention-FFN disaggregation.

This module is shared by the CUDA path's tests/bench and by the oracle's tests. It holds
none of the layer's arithmetic: it only draws random numbers and quantises the *inputs*
(activations and weights) the way an attention rank and a checkpoint loader would hand
them to the FFN pool (block-FP8, FastAFD "Methodology / System Design", item 1).

Recipe (readings the pages leave open are stated here and in the design notes):
  * weights: N(0, 1/sqrt(fan_in)), fan_in = H for W13 and I for W2, quantised to
    e4m3fn with one fp32 scale per 128x128 block (scale = block amax / 448);
  * activations: N(0, 1), quantised to e4m3fn with one fp32 scale per token per
    128 channels;
  * power-of-two variant (workloads named *_pow2, `pow2_scales=True`): every block scale
    is amax / 448 rounded up to a power of two (an 8-bit exponent, as FP8 recipes with
    UE8M0 scales quantise); the codes are then taken against that scale;
  * routing: K distinct expert ids per token, drawn without replacement with
    probability proportional to a popularity vector (Gumbel-top-k on log-popularity);
    uniform = equal popularity, Zipf(s) = popularity of id i proportional to 1/(i+1)^s;
  * topk_weights: softmax of K N(0,1) logits, i.e. renormalised over the K chosen ids
    (including ids owned by other FFN ranks);
  * slab split: n_m = floor(T/M) + [m < T mod M]; capacity = max(1, ceil(T/M)).
    Rows at or beyond n_m hold random junk, which the layer must never read.

Generation order for one seed: weights, activations, routing, logits.
Random draws use torch's CPU generator for the bulk (weights, activations) and
numpy's default_rng for routing and logits.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

E4M3_MAX = 448.0
QBLOCK = 128


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape of one FFN-pool MoE layer as held by one GPU."""
    hidden: int                # H
    intermediate: int          # I (per expert)
    num_experts_global: int    # E_g, ids the router may emit
    expert_begin: int          # e0, first id held here
    num_local_experts: int     # E_l, ids [e0, e0+E_l) are held here
    has_shared_expert: int     # S in {0, 1}; the shared expert sees every token with weight 1
    top_k: int                 # K

    @property
    def num_weight_experts(self) -> int:
        """Experts whose weights this GPU stores: E_l routed + S shared (shared last)."""
        return self.num_local_experts + self.has_shared_expert


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    num_tokens: int            # T = sum of slab counts
    num_slabs: int             # M
    zipf_s: Optional[float]    # None = uniform popularity
    zero_pop_mod: Optional[int] = None   # ids with id % mod == mod-1 get popularity 0
    seed: Sequence[int] = (0, 0)
    pow2_scales: bool = False  # block scales rounded up to powers of two

    @property
    def slab_counts(self) -> List[int]:
        T, M = self.num_tokens, self.num_slabs
        return [T // M + (1 if m < T % M else 0) for m in range(M)]

    @property
    def slab_capacity(self) -> int:
        return max(1, -(-self.num_tokens // self.num_slabs))


QWEN3_235B = LayerShape(4096, 1536, 128, 0, 128, 0, 8)
DEEPSEEK_V3_SHARE = LayerShape(7168, 2048, 256, 0, 32, 1, 8)
TINY = LayerShape(256, 128, 8, 0, 8, 0, 2)

CONFIGS = {
    "tiny": Workload("tiny", TINY, 64, 2, None, seed=(0, 0)),
    "qwen3_235b_t2048": Workload("qwen3_235b_t2048", QWEN3_235B, 2048, 8, None, seed=(1, 0)),
    "deepseek_v3_share_t4096": Workload("deepseek_v3_share_t4096", DEEPSEEK_V3_SHARE, 4096, 16, 1.0,
                                        seed=(2, 0)),
    "qwen3_235b_spec_q4_t8192": Workload("qwen3_235b_spec_q4_t8192", QWEN3_235B, 8192, 32, 0.8,
                                         zero_pop_mod=16, seed=(3, 0)),
    # the same draws with power-of-two block scales
    "tiny_pow2": Workload("tiny_pow2", TINY, 64, 2, None, seed=(0, 0), pow2_scales=True),
    "deepseek_v3_share_t4096_pow2": Workload("deepseek_v3_share_t4096_pow2", DEEPSEEK_V3_SHARE,
                                             4096, 16, 1.0, seed=(2, 0), pow2_scales=True),
}


def sweep_workloads() -> List[Workload]:
    """The batch / fan-in sweep at the DeepSeek-V3 share shape (T x M x routing)."""
    out = []
    cell = 0
    for zipf in (None, 1.2):
        for T in (1, 8, 64, 512, 4096, 16384):
            for M in (1, 4, 16, 64):
                tag = "uniform" if zipf is None else f"zipf{zipf}"
                out.append(Workload(f"sweep_t{T}_m{M}_{tag}", DEEPSEEK_V3_SHARE, T, M, zipf,
                                    seed=(4, cell)))
                cell += 1
    return out


def workload_by_name(name: str) -> Workload:
    if name in CONFIGS:
        return CONFIGS[name]
    for w in sweep_workloads():
        if w.name == name:
            return w
    raise KeyError(name)


# ----------------------------------------------------------------------------------------
# quantisation of inputs (library cast; the layer's own requantisation lives elsewhere)
# ----------------------------------------------------------------------------------------

def _pow2_ceil(s: torch.Tensor) -> torch.Tensor:
    """Smallest power of two >= s (s > 0), exactly: s = m * 2^e with m in [0.5, 1)."""
    m, e = torch.frexp(s)
    return torch.ldexp(torch.ones_like(s), torch.where(m == 0.5, e - 1, e))


def _quant_blocks(x: torch.Tensor, rb: int, cb: int, pow2: bool = False):
    """Quantise a 2-D fp32 tensor to e4m3fn codes with one scale per (rb x cb) block."""
    R, C = x.shape
    assert R % rb == 0 and C % cb == 0
    xb = x.reshape(R // rb, rb, C // cb, cb)
    amax = xb.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    if pow2:
        scale = _pow2_ceil(scale)
    q = (xb / scale[:, None, :, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8).reshape(R, C)
    return codes, scale.to(torch.float32)


def quantise_weight(w: torch.Tensor, pow2: bool = False):
    """[N, C] fp32 -> (uint8 codes [N, C], fp32 scales [N/128, C/128])."""
    return _quant_blocks(w, QBLOCK, QBLOCK, pow2)


def quantise_activation(x: torch.Tensor, pow2: bool = False):
    """[n, C] fp32 -> (uint8 codes [n, C], fp32 scales [n, C/128])."""
    return _quant_blocks(x, 1, QBLOCK, pow2)


@dataclasses.dataclass
class Slab:
    x: np.ndarray          # uint8 [cap, H]
    x_scale: np.ndarray    # f32 [cap, H/128]
    topk_ids: np.ndarray   # int32 [cap, K]
    topk_weights: np.ndarray  # f32 [cap, K]


@dataclasses.dataclass
class LayerInputs:
    shape: LayerShape
    w13: np.ndarray        # uint8 [E, 2I, H]  (gate rows 0..I-1, up rows I..2I-1)
    w13_scale: np.ndarray  # f32 [E, 2I/128, H/128]
    w2: np.ndarray         # uint8 [E, H, I]
    w2_scale: np.ndarray   # f32 [E, H/128, I/128]
    slabs: List[Slab]
    counts: np.ndarray     # int32 [M]
    capacity: int


def make_weights(shape: LayerShape, gen: torch.Generator, pow2_scales: bool = False):
    H, I, E = shape.hidden, shape.intermediate, shape.num_weight_experts
    w13 = np.empty((E, 2 * I, H), np.uint8)
    w13s = np.empty((E, 2 * I // QBLOCK, H // QBLOCK), np.float32)
    w2 = np.empty((E, H, I), np.uint8)
    w2s = np.empty((E, H // QBLOCK, I // QBLOCK), np.float32)
    for e in range(E):
        a = torch.randn(2 * I, H, generator=gen, dtype=torch.float32).mul_(1.0 / math.sqrt(H))
        c, s = quantise_weight(a, pow2_scales)
        w13[e], w13s[e] = c.numpy(), s.numpy()
        b = torch.randn(H, I, generator=gen, dtype=torch.float32).mul_(1.0 / math.sqrt(I))
        c, s = quantise_weight(b, pow2_scales)
        w2[e], w2s[e] = c.numpy(), s.numpy()
    return w13, w13s, w2, w2s


def popularity(wl: Workload) -> np.ndarray:
    Eg = wl.shape.num_experts_global
    ids = np.arange(Eg, dtype=np.float64)
    p = np.ones(Eg) if wl.zipf_s is None else 1.0 / np.power(ids + 1.0, wl.zipf_s)
    if wl.zero_pop_mod:
        p[(np.arange(Eg) % wl.zero_pop_mod) == wl.zero_pop_mod - 1] = 0.0
    return p / p.sum()


def sample_routing(wl: Workload, rng: np.random.Generator, n: int):
    """n tokens -> (ids int32 [n, K], weights f32 [n, K])."""
    K = wl.shape.top_k
    with np.errstate(divide="ignore"):
        logp = np.log(popularity(wl))       # -inf for zero-popularity ids
    g = rng.gumbel(size=(n, logp.size))
    keys = logp[None, :] + g
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :K].astype(np.int32)
    logits = rng.standard_normal((n, K))
    ex = np.exp(logits - logits.max(axis=1, keepdims=True))
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids, w


def make_inputs(wl: Workload, weights=None) -> LayerInputs:
    """Draw one workload's inputs. `weights` (a tuple from make_weights) may be reused."""
    sh = wl.shape
    H = sh.hidden
    gen = torch.Generator().manual_seed(int(np.random.SeedSequence(list(wl.seed)).generate_state(1)[0]))
    if weights is None:
        weights = make_weights(sh, gen, wl.pow2_scales)
    else:
        # keep the activation stream independent of whether weights were drawn
        gen = torch.Generator().manual_seed(
            int(np.random.SeedSequence(list(wl.seed) + [1]).generate_state(1)[0]))
    w13, w13s, w2, w2s = weights
    rng = np.random.default_rng(list(wl.seed))
    cap, M = wl.slab_capacity, wl.num_slabs
    counts = np.array(wl.slab_counts, dtype=np.int32)
    slabs = []
    for m in range(M):
        x = torch.randn(cap, H, generator=gen, dtype=torch.float32)
        xc, xs = quantise_activation(x, wl.pow2_scales)
        slabs.append(Slab(xc.numpy(), xs.numpy(), None, None))
    for m in range(M):
        ids, w = sample_routing(wl, rng, cap)
        n = counts[m]
        # junk beyond n_m: plausible-looking ids and weights that must be ignored
        if n < cap:
            ids[n:] = rng.integers(-1, sh.num_experts_global, size=(cap - n, sh.top_k))
            w[n:] = rng.standard_normal((cap - n, sh.top_k)).astype(np.float32)
        slabs[m].topk_ids, slabs[m].topk_weights = ids, w
    return LayerInputs(sh, w13, w13s, w2, w2s, slabs, counts, cap)


def make_custom_inputs(shape: LayerShape, counts: Sequence[int], capacity: int, seed: int,
                       zipf_s: Optional[float] = None, weights=None,
                       pow2_scales: bool = False) -> LayerInputs:
    """Inputs for an arbitrary slab split (used for ragged and edge-case tests)."""
    wl = Workload("custom", shape, int(sum(counts)), len(counts), zipf_s, seed=(99, seed),
                  pow2_scales=pow2_scales)
    sh = shape
    gen = torch.Generator().manual_seed(seed * 7919 + 17)
    if weights is None:
        weights = make_weights(sh, gen, pow2_scales)
    w13, w13s, w2, w2s = weights
    rng = np.random.default_rng([99, seed])
    slabs = []
    for m, n in enumerate(counts):
        x = torch.randn(capacity, sh.hidden, generator=gen, dtype=torch.float32)
        xc, xs = quantise_activation(x, pow2_scales)
        ids, w = sample_routing(wl, rng, capacity)
        if n < capacity:
            ids[n:] = rng.integers(-1, sh.num_experts_global, size=(capacity - n, sh.top_k))
        slabs.append(Slab(xc.numpy(), xs.numpy(), ids, w))
    return LayerInputs(sh, w13, w13s, w2, w2s, slabs, np.array(counts, np.int32), capacity)
