// Routing of the FFN-pool expert layer: slab intake, per-expert histogram, exclusive
// scan with the GEMM tile schedule, stable (token, slot)-ordered permutation, and the
// gather of routed FP8 rows into expert order.
//
// The attention ranks publish FP8 tokens and top-K routing metadata into this GPU's
// receive buffers (FastAFD, "Methodology / System Design", item 2); the FFN GPU groups the
// routed rows by expert for its grouped GEMMs (item 3). The order inside an expert's group
// is ascending (token, slot) with tokens numbered slab-major, which makes the result
// deterministic and independent of how the work is split across CTAs.
#pragma once

#include "ptx.cuh"

namespace afd {

constexpr int kRouteThreads = 256;
constexpr int kChunkTokens = 256;   // tokens per routing CTA (one per thread)
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kTokensPerWarp = kChunkTokens / kRouteWarps;
constexpr int kTileM = 128;

struct SlabTable {
  const uint8_t* x[AFD_MAX_SLABS];
  const float* xs[AFD_MAX_SLABS];
  const int32_t* ids[AFD_MAX_SLABS];
  const float* w[AFD_MAX_SLABS];
  __nv_bfloat16* y[AFD_MAX_SLABS];
};

struct RouteParams {
  const int32_t* counts;  // device [M]
  int M, cap, K, H, e0, El, Eg, S, G;
  int num_chunks;
  int rpad;               // row stride of the transposed scale arrays, >= max_rows + 128
  int32_t* slab_base;     // [M+1]
  int32_t* info;          // [0] T, [1] R, [2] m-tiles
  int32_t* chunk_hist;    // [num_chunks][max(El,1)]
  int32_t* chunk_off;     // [num_chunks][max(El,1)]
  int32_t* group_count;   // [G]
  int32_t* group_off;     // [G+1]
  int32_t* mtile_off;     // [G+1] 128-row m-tiles
  int* scan_ticket;       // zero between calls: route_count runs the scan; null: separate
  int tiling;             // as set on the plan: 0 (default, = 1) .. 2; -1: routing only
  int32_t* tok_mt;        // [Tmax] (slab << 24) | row
  int32_t* tok_need;      // [Tmax] contributions this GPU adds to the token
  int32_t* pos;           // [Tmax*K]
  int32_t* row_token;     // [rpad]
  int32_t* row_mt;        // [rpad] (slab << 24) | row of the row's token (may be null)
  int32_t* row_k;         // [rpad]
  float* row_w;           // [rpad]
  uint8_t* a_perm;        // [rpad][H]
  float* sa_t;            // [H/128][rpad]
  int* status;
  int zero_y;             // zero the slab rows of tokens that receive nothing from this GPU
};

// Slab-major prefix of the valid row counts, clamped to [0, cap].
__device__ __forceinline__ void load_slab_base(const RouteParams& p, int32_t* s_base) {
  if (threadIdx.x == 0) {
    int run = 0;
    bool bad = false;
    for (int m = 0; m < p.M; ++m) {
      s_base[m] = run;
      int n = p.counts[m];
      if (n < 0 || n > p.cap) {
        bad = true;
        n = n < 0 ? 0 : p.cap;
      }
      run += n;
    }
    s_base[p.M] = run;
    if (bad) atomicOr(p.status, AFD_STATUS_BAD_COUNT);
  }
  __syncthreads();
}

__device__ __forceinline__ int find_slab(const int32_t* s_base, int M, int g) {
  int lo = 0, hi = M - 1;           // largest m with s_base[m] <= g
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (s_base[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Classify the K slots of one token, in shared memory: keys[0..K) hold the token's ids on
// entry and, on return, the local group of each slot (-1 if the slot is not used here).
// Returns the mask of the slots that are valid and local. Sets *bad for ids that are
// neither -1 nor in [0, E_g), and for ids repeated from an earlier slot. (No per-thread
// arrays, so no local memory.)
__device__ __forceinline__ uint32_t classify_keys(int32_t* keys, int K, int e0, int El, int Eg, bool* bad) {
  uint32_t mask = 0;
  for (int k = 0; k < K; ++k) {
    const int id = keys[k];
    if (id == -1) continue;
    if (id < 0 || id >= Eg) { *bad = true; continue; }
    bool dup = false;
    for (int j = 0; j < k; ++j) dup |= (keys[j] == id);
    if (dup) { *bad = true; continue; }
    if (id >= e0 && id < e0 + El) mask |= 1u << k;
  }
  for (int k = 0; k < K; ++k) keys[k] = (mask >> k & 1u) ? keys[k] - e0 : -1;
  return mask;
}

// Block-wide exclusive scan of one value per thread (whole warps, up to 1024 threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (blockDim.x >> 5) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? s_warp[warp - 1] : 0);
  *total = s_warp[(blockDim.x >> 5) - 1];
  __syncthreads();
  return excl;
}

// 2. chunk offsets per group, group offsets (exclusive scan) and the m-tile schedule,
// computed by one block of any whole-warp size.
__device__ void route_scan_body(const RouteParams& p, int T, int* s_warp) {
  const int chunks = (T + kChunkTokens - 1) / kChunkTokens;
  const int El1 = max(p.El, 1);
  for (int e = threadIdx.x; e < p.El; e += blockDim.x) {
    int run = 0;
    for (int c = 0; c < chunks; ++c) {
      const size_t i = static_cast<size_t>(c) * El1 + e;
      const int h = p.chunk_hist[i];
      p.chunk_off[i] = run;
      run += h;
    }
    p.group_count[e] = run;
  }
  __syncthreads();
  if (p.S && threadIdx.x == 0) p.group_count[p.El] = T;
  __syncthreads();
  int base_rows = 0, base_tiles = 0;
  for (int g0 = 0; g0 < p.G; g0 += blockDim.x) {
    const int g = g0 + threadIdx.x;
    const int cnt = g < p.G ? p.group_count[g] : 0;
    int tot_rows, tot_tiles;
    const int ex_rows = block_exclusive_scan(cnt, s_warp, &tot_rows);
    const int ex_tiles = block_exclusive_scan((cnt + kTileM - 1) / kTileM, s_warp, &tot_tiles);
    if (g < p.G) {
      p.group_off[g] = base_rows + ex_rows;
      p.mtile_off[g] = base_tiles + ex_tiles;
    }
    base_rows += tot_rows;
    base_tiles += tot_tiles;
  }
  if (threadIdx.x == 0) {
    p.group_off[p.G] = base_rows;
    p.mtile_off[p.G] = base_tiles;
    p.info[1] = base_rows;
    p.info[2] = base_tiles;
    // the tiling this call runs (the host launches only its kernels); 0 for routing
    // without a layer
    p.info[3] = p.tiling < 0 ? 0 : (p.tiling == 0 ? 1 : p.tiling);
  }
}

// 2 as its own launch (one block of 1024 threads).
__global__ void __launch_bounds__(1024) route_scan_kernel(const __grid_constant__ RouteParams p) {
  __shared__ int s_warp[32];
  route_scan_body(p, p.info[0], s_warp);
}

// 1 for one chunk of 256 tokens (thread = token): classification, histogram of the local
// groups in shared memory, token bookkeeping; the histogram goes to chunk_hist[chunk].
// s_keys: shared memory [256][K] for the tokens' ids. Called by all threads of the block.
__device__ __forceinline__ void route_count_chunk(const RouteParams& p, const SlabTable& slabs,
                                                  const int32_t* s_base, int T, int chunk,
                                                  int32_t* s_hist, int32_t* s_keys) {
  for (int e = threadIdx.x; e < p.El; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int g = chunk * kChunkTokens + threadIdx.x;
  if (g < T) {
    const int m = find_slab(s_base, p.M, g);
    const int t = g - s_base[m];
    int32_t* keys = s_keys + threadIdx.x * p.K;
    const int32_t* src = slabs.ids[m] + static_cast<size_t>(t) * p.K;
    for (int k = 0; k < p.K; ++k) keys[k] = src[k];
    bool bad = false;
    const uint32_t mask = classify_keys(keys, p.K, p.e0, p.El, p.Eg, &bad);
    for (int k = 0; k < p.K; ++k)
      if (mask >> k & 1u) atomicAdd(&s_hist[keys[k]], 1);
    p.tok_mt[g] = (m << 24) | t;
    p.tok_need[g] = __popc(mask) + p.S;
    if (bad) atomicOr(p.status, AFD_STATUS_BAD_ROUTING);
  }
  __syncthreads();
  int32_t* out = p.chunk_hist + static_cast<size_t>(chunk) * max(p.El, 1);
  for (int e = threadIdx.x; e < p.El; e += blockDim.x) out[e] = s_hist[e];
  __syncthreads();   // s_hist is read above before a next chunk clears it
}

// 1. per-chunk histogram of local groups; token bookkeeping. With p.scan_ticket set, the
// block that finishes last also runs step 2 (every block publishes its histogram, fences,
// then takes a ticket; the counter is returned to zero for the next call).
// Dynamic shared memory: the ids of the chunk's tokens, [256][K] int32.
__global__ void __launch_bounds__(kRouteThreads) route_count_kernel(
    const __grid_constant__ RouteParams p, const __grid_constant__ SlabTable slabs) {
  extern __shared__ int32_t s_keys[];
  __shared__ int32_t s_base[AFD_MAX_SLABS + 1];
  __shared__ int32_t s_hist[AFD_MAX_GROUPS];
  load_slab_base(p, s_base);
  const int T = s_base[p.M];
  if (blockIdx.x == 0) {
    for (int m = threadIdx.x; m <= p.M; m += blockDim.x) p.slab_base[m] = s_base[m];
    if (threadIdx.x == 0) p.info[0] = T;
  }
  route_count_chunk(p, slabs, s_base, T, blockIdx.x, s_hist, s_keys);
  if (!p.scan_ticket) return;
  __shared__ int s_last;
  __shared__ int s_warp[32];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(p.scan_ticket, 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  route_scan_body(p, T, s_warp);
  if (threadIdx.x == 0) *p.scan_ticket = 0;
}

// 3 for one chunk: stable placement of its local (token, slot) pairs and of its tokens'
// shared rows; zero output rows of its tokens that receive nothing. s_run [warps][El],
// s_key [warps][32*K] and s_wt [warps][32*K] are shared memory (the pairs' groups and
// top-K weights, read once per token with its ids). Called by all threads of the block.
__device__ __forceinline__ void route_scatter_chunk(const RouteParams& p, const SlabTable& slabs,
                                                    const int32_t* s_base, int T, int chunk,
                                                    int32_t* s_run, int32_t* s_key, float* s_wt) {
  const int El1 = max(p.El, 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kRouteWarps * El1; i += blockDim.x) s_run[i] = 0;
  __syncthreads();
  const int K = p.K;
  const int g = chunk * kChunkTokens + warp * kTokensPerWarp + lane;
  int m = 0, t = 0;
  int32_t* mykeys = s_key + warp * 32 * K;
  float* mywt = s_wt + warp * 32 * K;
  if (g < T) {
    m = find_slab(s_base, p.M, g);
    t = g - s_base[m];
    const int32_t* src = slabs.ids[m] + static_cast<size_t>(t) * K;
    const float* wsrc = slabs.w[m] + static_cast<size_t>(t) * K;
    int32_t* keys = mykeys + lane * K;
    for (int k = 0; k < K; ++k) {
      keys[k] = src[k];
      mywt[lane * K + k] = wsrc[k];
    }
    bool bad = false;
    const uint32_t mask = classify_keys(keys, K, p.e0, p.El, p.Eg, &bad);
    for (int k = 0; k < K; ++k)
      if (mask >> k & 1u) atomicAdd(&s_run[warp * El1 + keys[k]], 1);
  } else {
    for (int k = 0; k < K; ++k) mykeys[lane * K + k] = -1;
  }
  __syncthreads();
  // per-warp starting row of every group: group base + chunk base + earlier warps
  const int32_t* coff = p.chunk_off + static_cast<size_t>(chunk) * El1;
  for (int e = threadIdx.x; e < p.El; e += blockDim.x) {
    int run = p.group_off[e] + coff[e];
    for (int w = 0; w < kRouteWarps; ++w) {
      const int v = s_run[w * El1 + e];
      s_run[w * El1 + e] = run;
      run += v;
    }
  }
  __syncthreads();
  // walk this warp's pairs in (token, slot) order, 32 at a time
  const int gw0 = chunk * kChunkTokens + warp * kTokensPerWarp;
  for (int r = 0; r < K; ++r) {
    const int pidx = r * 32 + lane;             // pair index inside the warp
    const int tl = pidx / K, k = pidx - tl * K;
    const int key = mykeys[pidx];
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (key >= 0) {
      const int rank = __popc(peers & lanemask_lt());
      const int row = s_run[warp * El1 + key] + rank;
      const int gg = gw0 + tl;
      p.pos[static_cast<size_t>(gg) * K + k] = row;
      p.row_token[row] = gg;
      p.row_k[row] = k;
      p.row_w[row] = mywt[pidx];
      if (p.row_mt) {
        const int mm = find_slab(s_base, p.M, gg);
        p.row_mt[row] = (mm << 24) | (gg - s_base[mm]);
      }
    } else {
      const int gg = gw0 + tl;
      if (gg < T) p.pos[static_cast<size_t>(gg) * K + k] = -1;
    }
    __syncwarp();
    if (key >= 0 && (31 - __clz(peers)) == static_cast<int>(lane))
      s_run[warp * El1 + key] += __popc(peers);
    __syncwarp();
  }
  if (g < T && p.S) {
    const int row = p.group_off[p.El] + g;
    p.row_token[row] = g;
    if (p.row_mt) p.row_mt[row] = (m << 24) | t;
    p.row_k[row] = -1;
    p.row_w[row] = 1.0f;
  }
  // tokens that receive nothing from this GPU get zeros (only possible without a shared
  // expert); everything else is written by the down-projection's combine
  if (!p.S && p.zero_y) {
    unsigned need0 = __ballot_sync(0xffffffffu, g < T && p.tok_need[g] == 0);
    while (need0) {
      const int src_lane = __ffs(need0) - 1;
      need0 &= need0 - 1;
      const int mm = __shfl_sync(0xffffffffu, m, src_lane);
      const int tt = __shfl_sync(0xffffffffu, t, src_lane);
      uint4* dst = reinterpret_cast<uint4*>(slabs.y[mm] + static_cast<size_t>(tt) * p.H);
      for (int i = lane; i < p.H / 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    }
  }
  __syncthreads();
}

// Dynamic shared memory of the placement: s_run [warps][El] int32, s_key [warps][32*K]
// int32, s_wt [warps][32*K] float.
__host__ __device__ constexpr size_t scatter_smem_bytes(int El, int K) {
  return sizeof(int32_t) * (static_cast<size_t>(kRouteWarps) * (El > 1 ? El : 1) +
                            2 * static_cast<size_t>(kRouteWarps) * 32 * K);
}

// 3. stable placement of every local (token, slot) pair and of the shared rows, one
// chunk per block.
__global__ void __launch_bounds__(kRouteThreads) route_scatter_kernel(
    const __grid_constant__ RouteParams p, const __grid_constant__ SlabTable slabs) {
  extern __shared__ int32_t s_dyn[];
  __shared__ int32_t s_base[AFD_MAX_SLABS + 1];
  for (int m = threadIdx.x; m <= p.M; m += blockDim.x) s_base[m] = p.slab_base[m];
  __syncthreads();
  int32_t* s_key = s_dyn + kRouteWarps * max(p.El, 1);
  route_scatter_chunk(p, slabs, s_base, s_base[p.M], blockIdx.x, s_dyn, s_key,
                      reinterpret_cast<float*>(s_key + kRouteWarps * 32 * p.K));
}

// 1-3 in one block for one-chunk plans (at most 256 tokens, thread = token). The slab
// counts are loaded in parallel and scanned; every token's ids and weights are read once;
// the histogram, the group scan and the running rows stay in shared memory, so the block
// waits on two global round trips (counts, then ids and weights) instead of one per step.
// The placement is route_scatter_chunk's (per-warp counts, then ranks inside the warp in
// (token, slot) order), so the routing is the same bit for bit.
constexpr int kSmallRouteChunks = 1;
__global__ void __launch_bounds__(kRouteThreads) route_small_kernel(
    const __grid_constant__ RouteParams p, const __grid_constant__ SlabTable slabs) {
  extern __shared__ int32_t s_dyn[];
  __shared__ int32_t s_base[AFD_MAX_SLABS + 1];
  __shared__ int32_t s_goff[AFD_MAX_GROUPS + 1];
  __shared__ int s_warp[32];
  const int El1 = max(p.El, 1);
  const int K = p.K;
  int32_t* s_run = s_dyn;                         // [warps][El]
  int32_t* s_key = s_dyn + kRouteWarps * El1;     // [warps][32*K]
  float* s_wt = reinterpret_cast<float*>(s_key + kRouteWarps * 32 * K);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the gather may be scheduled now; it waits for this kernel's results on the device
  pdl_trigger();

  // slab bases: one count per thread (M <= 128), clamped, block scan
  int n = 0;
  if (tid < p.M) {
    n = p.counts[tid];
    if (n < 0 || n > p.cap) {
      atomicOr(p.status, AFD_STATUS_BAD_COUNT);
      n = n < 0 ? 0 : p.cap;
    }
  }
  for (int i = tid; i < kRouteWarps * El1; i += blockDim.x) s_run[i] = 0;
  int T;
  const int ex = block_exclusive_scan(n, s_warp, &T);
  if (tid < p.M) {
    s_base[tid] = ex;
    p.slab_base[tid] = ex;
  }
  if (tid == 0) {
    s_base[p.M] = T;
    p.slab_base[p.M] = T;
    p.info[0] = T;
  }
  __syncthreads();

  // tokens: ids and weights, classification, per-warp group counts, token bookkeeping
  const int g = tid;
  int m = 0, t = 0, need = 0;
  int32_t* mykeys = s_key + warp * 32 * K;
  float* mywt = s_wt + warp * 32 * K;
  if (g < T) {
    m = find_slab(s_base, p.M, g);
    t = g - s_base[m];
    const int32_t* src = slabs.ids[m] + static_cast<size_t>(t) * K;
    const float* wsrc = slabs.w[m] + static_cast<size_t>(t) * K;
    int32_t* keys = mykeys + lane * K;
    for (int k = 0; k < K; ++k) {
      keys[k] = src[k];
      mywt[lane * K + k] = wsrc[k];
    }
    bool bad = false;
    const uint32_t mask = classify_keys(keys, K, p.e0, p.El, p.Eg, &bad);
    for (int k = 0; k < K; ++k)
      if (mask >> k & 1u) atomicAdd(&s_run[warp * El1 + keys[k]], 1);
    need = __popc(mask) + p.S;
    p.tok_mt[g] = (m << 24) | t;
    p.tok_need[g] = need;
    if (bad) atomicOr(p.status, AFD_STATUS_BAD_ROUTING);
  } else {
    for (int k = 0; k < K; ++k) mykeys[lane * K + k] = -1;
  }
  __syncthreads();

  // group counts, offsets and the m-tile schedule (exclusive scans over the groups)
  int base_rows = 0, base_tiles = 0;
  for (int g0 = 0; g0 < p.G; g0 += blockDim.x) {
    const int e = g0 + tid;
    int cnt = 0;
    if (e < p.El) {
      for (int w = 0; w < kRouteWarps; ++w) cnt += s_run[w * El1 + e];
    } else if (e < p.G) {
      cnt = T;                                    // the shared expert: every token
    }
    if (e < p.G) p.group_count[e] = cnt;
    int tot_rows, tot_tiles;
    const int ex_rows = block_exclusive_scan(cnt, s_warp, &tot_rows);
    const int ex_tiles = block_exclusive_scan((cnt + kTileM - 1) / kTileM, s_warp, &tot_tiles);
    if (e < p.G) {
      s_goff[e] = base_rows + ex_rows;
      p.group_off[e] = base_rows + ex_rows;
      p.mtile_off[e] = base_tiles + ex_tiles;
    }
    base_rows += tot_rows;
    base_tiles += tot_tiles;
  }
  if (tid == 0) {
    s_goff[p.G] = base_rows;
    p.group_off[p.G] = base_rows;
    p.mtile_off[p.G] = base_tiles;
    p.info[1] = base_rows;
    p.info[2] = base_tiles;
    p.info[3] = p.tiling < 0 ? 0 : (p.tiling == 0 ? 1 : p.tiling);
  }
  __syncthreads();
  // per-warp starting row of every group
  for (int e = tid; e < p.El; e += blockDim.x) {
    int run = s_goff[e];
    for (int w = 0; w < kRouteWarps; ++w) {
      const int v = s_run[w * El1 + e];
      s_run[w * El1 + e] = run;
      run += v;
    }
  }
  __syncthreads();

  // placement: this warp's pairs in (token, slot) order, 32 at a time
  const int gw0 = warp * kTokensPerWarp;
  for (int r = 0; r < K; ++r) {
    const int pidx = r * 32 + lane;
    const int tl = pidx / K, k = pidx - tl * K;
    const int key = mykeys[pidx];
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int gg = gw0 + tl;
    if (key >= 0) {
      const int row = s_run[warp * El1 + key] + __popc(peers & lanemask_lt());
      p.pos[static_cast<size_t>(gg) * K + k] = row;
      p.row_token[row] = gg;
      p.row_k[row] = k;
      p.row_w[row] = mywt[pidx];
      if (p.row_mt) {
        const int mm = find_slab(s_base, p.M, gg);
        p.row_mt[row] = (mm << 24) | (gg - s_base[mm]);
      }
    } else if (gg < T) {
      p.pos[static_cast<size_t>(gg) * K + k] = -1;
    }
    __syncwarp();
    if (key >= 0 && (31 - __clz(peers)) == static_cast<int>(lane)) s_run[warp * El1 + key] += __popc(peers);
    __syncwarp();
  }
  if (g < T && p.S) {
    const int row = s_goff[p.El] + g;
    p.row_token[row] = g;
    if (p.row_mt) p.row_mt[row] = (m << 24) | t;
    p.row_k[row] = -1;
    p.row_w[row] = 1.0f;
  }
  // tokens that receive nothing from this GPU get zeros (only possible without a shared
  // expert)
  if (!p.S && p.zero_y) {
    unsigned need0 = __ballot_sync(0xffffffffu, g < T && need == 0);
    while (need0) {
      const int src_lane = __ffs(need0) - 1;
      need0 &= need0 - 1;
      const int mm = __shfl_sync(0xffffffffu, m, src_lane);
      const int tt = __shfl_sync(0xffffffffu, t, src_lane);
      uint4* dst = reinterpret_cast<uint4*>(slabs.y[mm] + static_cast<size_t>(tt) * p.H);
      for (int i = lane; i < p.H / 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    }
  }
}

// 4. copy routed rows (FP8 codes and their per-128 scales) into expert order.
// One warp per token: the token's row is read once, 4 KiB at a time (eight 16-byte loads
// in flight per lane), and written to each of its destination rows (its local top-K
// slots, then its shared-expert row). Scales are stored transposed ([H/128][rpad]) so
// that a GEMM tile reads one block's scales for 32 consecutive rows with one load.
__global__ void __launch_bounds__(kRouteThreads) gather_rows_kernel(
    const __grid_constant__ RouteParams p, const __grid_constant__ SlabTable slabs) {
  pdl_trigger();
  pdl_wait();
  const int T = p.info[0];
  const int K = p.K;
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int KB = p.H / AFD_QBLOCK;
  const int n16 = p.H / 16;               // H is a multiple of 256: n16 a multiple of 16
  for (int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < T; g += nwarps) {
    const int mt = p.tok_mt[g];
    const int m = mt >> 24, t = mt & 0xFFFFFF;
    // destination rows: lane k < K holds slot k's row (or -1), the shared row follows
    int myrow = -1;
    if (lane < K) myrow = p.pos[static_cast<size_t>(g) * K + lane];
    unsigned dmask = __ballot_sync(0xffffffffu, myrow >= 0);
    const int shared_row = p.S ? p.group_off[p.El] + g : -1;
    const uint4* __restrict__ src =
        reinterpret_cast<const uint4*>(slabs.x[m] + static_cast<size_t>(t) * p.H);
    for (int i0 = 0; i0 < n16; i0 += 8 * 32) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + 32 * j + lane;
        if (i < n16) v[j] = __ldg(src + i);
      }
      unsigned d = dmask;
      int r = -1;
      while (true) {
        if (d) {
          const int k = __ffs(d) - 1;
          d &= d - 1;
          r = __shfl_sync(0xffffffffu, myrow, k);
        } else if (r != shared_row) {
          r = shared_row;
        } else {
          break;
        }
        if (r < 0) break;
        uint4* __restrict__ dst = reinterpret_cast<uint4*>(p.a_perm + static_cast<size_t>(r) * p.H);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = i0 + 32 * j + lane;
          if (i < n16) dst[i] = v[j];
        }
      }
    }
    const float* ssrc = slabs.xs[m] + static_cast<size_t>(t) * KB;
    for (int kb = lane; kb < KB; kb += 32) {
      const float sc = ssrc[kb];
      float* dcol = p.sa_t + static_cast<size_t>(kb) * p.rpad;
      unsigned d = dmask;
      while (d) {
        const int k = __ffs(d) - 1;
        d &= d - 1;
        dcol[p.pos[static_cast<size_t>(g) * K + k]] = sc;
      }
      if (shared_row >= 0) dcol[shared_row] = sc;
    }
  }
}

}  // namespace afd
