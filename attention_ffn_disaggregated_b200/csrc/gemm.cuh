// Persistent block-FP8 grouped GEMM for sm_100a (tcgen05 + TMEM + TMA), used for both
// expert projections of the FFN-pool layer (FastAFD, "Methodology / System Design",
// item 3: "block-FP8 grouped GEMMs, activation and push-back").
//
// Output tile per CTA: 128 routed rows of one expert x 256 output columns; K runs in
// blocks of 128 (the quantisation block). Each K block is one tcgen05 partial product
// (4 x kind::f8f6f4 MMAs of K=32) into one of two TMEM buffers; the epilogue warps read
// the partial, multiply it by (row scale x weight-block scale) and accumulate in fp32
// registers ("software promotion": the scales are arbitrary fp32, so they cannot ride on
// the hardware's UE8M0 block-scale path; gemm_mx.cuh holds the block-scale kernel for
// inputs whose scales are all powers of two).
//
// Warp roles (384 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues MMAs,
// warps 2..3 load the weight-block scales of the CTA's next tile into a two-slot ring,
// warps 4..11 are the epilogue (two per TMEM lane quadrant, splitting the columns).
//
// Epilogues:
//   SWIGLU   (W13) columns are [gate 128 | up 128] of intermediate block nt; h = silu(g)*u
//            is requantised to e4m3 per (row, 128 channels) and stored with its scale.
//   COMBINE  (W2)  the row's result times its top-K weight is added into the token's fp32
//            accumulator by the bulk-copy engine (cp.reduce.async.bulk ... .add.f32: one
//            512-byte row segment per operation, staged through shared memory), so the
//            epilogue warps hand the reductions off and return to the next tile's partial
//            products; combine_finalize_kernel then writes every token's sum as bf16 into
//            its slab row and clears the accumulator. The accumulator of token t of slab m
//            is found through a per-slab pointer table (the plan's own buffers, or the
//            tokens' owners' under expert parallelism).
//
// Small batches: when the tiles fill at most half of the grid, each tile's K blocks are
// shared out among several CTAs (split-K); W13's splits meet in an fp32 workspace and the
// last one finishes the tile, W2's partial sums are reduced into the accumulators like
// whole tiles. Under programmatic dependent launch a CTA allocates TMEM and prefetches
// its descriptors before waiting for the previous kernel.
#pragma once

#include "ptx.cuh"
#include "route.cuh"

namespace afd {

constexpr int kBN = 256;
constexpr int kBK = 128;
constexpr int kGemmThreads = 384;
constexpr int kEpiWarps = 8;
constexpr uint32_t kABytes = kTileM * kBK;   // 16 KiB: 128 rows of one K block
constexpr uint32_t kBBytes = kBN * kBK;      // 32 KiB: 256 weight rows of one K block
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 512;          // two 256-column fp32 partial buffers
constexpr int kMaxStages = 4;
// Register split: the block launches with kLaunchRegs per thread; warpgroup 0 (TMA, MMA,
// two idle warps) drops to kProducerRegs and the two epilogue warpgroups rise to
// kEpilogueRegs. 128*40 + 256*232 == 384*168, so the increase never waits for registers
// the block does not own; the host refuses to launch if the compiled count differs.
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 40;
constexpr int kEpilogueRegs = 232;
static_assert(128 * kProducerRegs + 256 * kEpilogueRegs <= kGemmThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

enum EpiKind { EPI_SWIGLU = 0, EPI_COMBINE = 1 };

// Combine staging: per epilogue warp two buffers of 8 rows x 128 fp32 (+16 bytes of
// padding per row, so that eight lanes storing one float4 each at the same column hit
// disjoint banks); a buffer row is the source of one 512-byte bulk reduction.
constexpr int kStgRows = 8;
constexpr uint32_t kStgRowBytes = 128 * 4 + 16;
constexpr uint32_t kStgBufBytes = kStgRows * kStgRowBytes;
constexpr uint32_t kStgWarpBytes = 2 * kStgBufBytes;

template <int EPI>
struct GemmCfg {
  // W13 keeps four operand stages; W2 gives one up for the combine staging
  static constexpr int kStages = EPI == EPI_SWIGLU ? 4 : 3;
  static constexpr size_t kStaging = EPI == EPI_SWIGLU ? 0 : static_cast<size_t>(kEpiWarps) * kStgWarpBytes;
};

struct YTable {
  __nv_bfloat16* y[AFD_MAX_SLABS];
};

// Destination of the combine: token t of slab m adds into a[m] + t*H (the plan's own
// accumulators, or buffers of the tokens' owners, possibly on other GPUs).
struct AccTable {
  float* a[AFD_MAX_SLABS];
};

struct GemmParams {
  const int32_t* info;        // [0] tokens, [1] rows, [2] m-tiles of this call
  const int32_t* group_off;   // [G+1] first row of each group
  const int32_t* mtile_off;   // [G+1] first 128-row m-tile of each group
  int G;
  int n_tiles;                // 256-column tiles per m-tile
  int num_kb;                 // K blocks of 128
  int slice_first;            // tile order: 0 = m-tile major, 1 = column-tile major
  const float* sa_t;          // A scales, [num_kb][rpad]
  int rpad;
  const float* w_scale;       // [E][ws_rows][num_kb]
  int ws_rows;
  int I;
  int H;
  // SWIGLU epilogue outputs
  uint8_t* hq;                // [rpad][I]
  float* sh_t;                // [I/128][rpad]
  // COMBINE epilogue inputs/outputs
  const int32_t* row_token;
  const int32_t* row_mt;      // (slab << 24) | row of each routed row's token
  const float* row_w;
  AccTable acc;               // per slab: fp32 [cap][H], zero between calls
  // split-K for gate/up launches whose tiles fill less than half of the grid: the K blocks
  // of a tile are shared out among several CTAs, whose partial sums go to the fp32 workspace g_ws [g_rows][2I], and the CTA whose
  // partial completes a tile's 32-row quadrant (g_cnt) finishes SwiGLU + requantisation
  // for those rows from it and clears it.
  int split_ok;
  float* g_ws;
  int g_rows;
  int* g_cnt;                 // [grid][4], zero between calls
  // weights every call of a small plan reads (the shared expert's), prefetched into L2 by
  // the CTAs, spread over all of them, while the previous kernels still run; null when
  // not used
  const uint8_t* pf_base;
  unsigned long long pf_bytes;
  int* status;
  unsigned long long wait_limit_ns;
  int inject_stall;
};

constexpr int kMinSplitKb = 4;    // K blocks per split, at least
constexpr int kMaxKb = AFD_MAX_QBLOCKS;   // K blocks of one projection (H/128, I/128)
constexpr int kMaxSplits = 8;

// 16-byte multiple: the combine staging that follows it is the source of bulk copies
struct alignas(16) GemmSmem {
  // weight-block scales of a tile: [slot][row][K block]; SWIGLU rows = gate, up block;
  // COMBINE rows = the two 128-row halves of the 256 output columns
  float wring[2][2][kMaxKb];
  uint64_t wfull[2];
  uint64_t wempty[2];
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t pair[4];           // SWIGLU: amax exchange between the two warps of a quadrant
  uint32_t tmem_base;
  int abort_flag;
  float amax[2][2][kTileM];
  int32_t mtile[AFD_MAX_GROUPS + 1];
  int32_t goff[AFD_MAX_GROUPS + 1];   // first row of each group (tile decoding)
};
static_assert(sizeof(GemmSmem) % 16 == 0, "staging after GemmSmem must stay 16-byte aligned");

template <int EPI>
__host__ __device__ constexpr size_t gemm_smem_bytes() {
  return 1024 + static_cast<size_t>(GemmCfg<EPI>::kStages) * kStageBytes + sizeof(GemmSmem) +
         GemmCfg<EPI>::kStaging;
}
static_assert(gemm_smem_bytes<EPI_SWIGLU>() <= 232448, "W13 shared memory");
static_assert(gemm_smem_bytes<EPI_COMBINE>() <= 232448, "W2 shared memory");

// A wait that ignores the abort flag; used only to drain copies/MMAs already in flight.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

struct TileCoord {
  int e, row0, rows, nt, mt;
};

// Tile -> (expert, first row, valid rows, column tile). Tiles are numbered m-tile major
// (all column tiles of m-tile 0, then of m-tile 1, ...) or, with slice_first, column-tile
// major (every m-tile of column tile 0, then of column tile 1, ...).
__device__ __forceinline__ TileCoord decode_tile(int tile, int n_tiles, int slice_first,
                                                 const int32_t* s_mtile, int G,
                                                 const int32_t* group_off) {
  TileCoord c;
  int mt;
  if (slice_first) {
    const int n_mt = s_mtile[G];
    c.nt = tile / n_mt;
    mt = tile - c.nt * n_mt;
  } else {
    mt = tile / n_tiles;
    c.nt = tile - mt * n_tiles;
  }
  c.mt = mt;
  int lo = 0, hi = G - 1;               // last group whose first m-tile is <= mt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_mtile[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  c.e = lo;
  const int g0 = group_off[lo], g1 = group_off[lo + 1];
  c.row0 = g0 + (mt - s_mtile[lo]) * kTileM;
  c.rows = min(kTileM, g1 - c.row0);
  return c;
}

// silu(g) * u = g / (1 + exp(-g)) * u with branch-free fast exp and division; g is clamped
// at -80, where silu is 0 to fp32 precision, so exp(-g) stays finite
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float gx = fmaxf(g, -80.0f);
  return __fdividef(gx, 1.0f + __expf(-gx)) * u;
}

// Split-K W13: SwiGLU + requantisation of intermediate block nt for `nrows` consecutive
// rows from `row0`, from the fp32 sums in G (gate at columns nt*128.., up at I + nt*128..),
// which are then cleared. The whole warp works on four rows at a time (lane = 4 channels
// of each), so a few rows cost one round trip to L2 rather than one per 4 channels. The
// same arithmetic as the one-CTA epilogue; the block amax is a warp max.
__device__ __forceinline__ void split_swiglu_rows(const GemmParams& p, int row0, int nrows, int nt,
                                                  int lane) {
  for (int r0 = 0; r0 < nrows; r0 += 4) {
    float4 gv[4], uv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (r0 + j < nrows) {
        const float* gr = p.g_ws + static_cast<size_t>(row0 + r0 + j) * (2 * p.I) + nt * 128 + 4 * lane;
        gv[j] = __ldcg(reinterpret_cast<const float4*>(gr));
        uv[j] = __ldcg(reinterpret_cast<const float4*>(gr + p.I));
      } else {
        gv[j] = uv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float h0 = silu_mul(gv[j].x, uv[j].x), h1 = silu_mul(gv[j].y, uv[j].y);
      const float h2 = silu_mul(gv[j].z, uv[j].z), h3 = silu_mul(gv[j].w, uv[j].w);
      float amax = fmaxf(fmaxf(fabsf(h0), fabsf(h1)), fmaxf(fabsf(h2), fabsf(h3)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (r0 + j < nrows) {
        const int row = row0 + r0 + j;
        const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
        const float rsc = __frcp_rn(sc);
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.hq + static_cast<size_t>(row) * p.I + nt * 128);
        dst[lane] = static_cast<uint32_t>(pack_e4m3x2(h0 * rsc, h1 * rsc)) |
                    (static_cast<uint32_t>(pack_e4m3x2(h2 * rsc, h3 * rsc)) << 16);
        float* gr = p.g_ws + static_cast<size_t>(row) * (2 * p.I) + nt * 128 + 4 * lane;
        __stcg(reinterpret_cast<float4*>(gr), make_float4(0.f, 0.f, 0.f, 0.f));
        __stcg(reinterpret_cast<float4*>(gr + p.I), make_float4(0.f, 0.f, 0.f, 0.f));
        if (lane == 0) p.sh_t[static_cast<size_t>(nt) * p.rpad + row] = sc;
      }
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmParams p,
                        const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b) {
  constexpr int kStages = GemmCfg<EPI>::kStages;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = base;
  uint8_t* sB = base + kStages * kABytes;
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(base + kStages * kStageBytes);
  uint8_t* stg = base + kStages * kStageBytes + sizeof(GemmSmem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.tfull[b], 1);
      mbar_init(&S.tempty[b], kEpiWarps);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&S.pair[i], 64);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.wfull[i], 2);
      mbar_init(&S.wempty[i], kEpiWarps);
    }
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (p.pf_bytes && warp == 2) {
    // this CTA's share of the always-read weights, in 16-byte multiples, 32 KiB per request
    const unsigned long long share = ((p.pf_bytes + gridDim.x - 1) / gridDim.x + 15ull) & ~15ull;
    const unsigned long long lo = share * blockIdx.x;
    const unsigned long long hi = lo + share < p.pf_bytes ? lo + share : p.pf_bytes;
    for (unsigned long long o = lo + 32768ull * lane; o < hi; o += 32768ull * 32)
      bulk_prefetch_l2(p.pf_base + o, static_cast<uint32_t>(hi - o < 32768ull ? hi - o : 32768ull));
  }

  // everything above is local set-up (a kernel launched early under programmatic
  // dependent launch does it while its predecessor drains; no predecessor holds tensor
  // memory on this SM, whose shared memory this kernel fills); the tile schedule and the
  // operands come from the previous kernels
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i <= p.G; i += blockDim.x) {
    S.mtile[i] = p.mtile_off[i];
    S.goff[i] = p.group_off[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;
  const int nkb = p.num_kb;
  // split-K when the tiles fill at most half of the grid (small batches). W13's splits
  // meet in the fp32 workspace G and the last one finishes the tile; W2's partial sums
  // are reduced into the token accumulators like whole tiles, so they need nothing more.
  const int n_tiles0 = S.mtile[p.G] * p.n_tiles;
  int splits = 1;
  if (p.split_ok && n_tiles0 > 0 && 2 * n_tiles0 <= static_cast<int>(gridDim.x) &&
      (EPI == EPI_COMBINE || S.mtile[p.G] * kTileM <= p.g_rows))
    splits = max(1, min(min(static_cast<int>(gridDim.x) / n_tiles0, nkb / kMinSplitKb), kMaxSplits));
  const int total_units = n_tiles0 * splits;

  if (warp < 4) {
    // each role's code sits inside the branch that sets its register budget
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      // A rows are re-read by every column tile of their m-tile. W13 weight blocks are
      // re-read by every m-tile of their expert; W2's stream past the L2-resident combine
      // accumulators, so they go first.
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = EPI == EPI_SWIGLU ? policy_evict_last() : policy_evict_first();
      int it = 0;
      bool ok = true;
      int skipped = -1;
      for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
        const int tile = u / splits, sp = u - tile * splits;
        const int kb0 = sp * nkb / splits, kb1 = (sp + 1) * nkb / splits;
        const TileCoord c = decode_tile(tile, p.n_tiles, p.slice_first, S.mtile, p.G, S.goff);
        // B rows of this tile: [brow0, +128) and [brow1, +128)
        int brow0, brow1;
        if (EPI == EPI_SWIGLU) {
          brow0 = c.nt * 128;               // gate block
          brow1 = p.I + c.nt * 128;         // up block
        } else {
          brow0 = c.nt * kBN;
          brow1 = c.nt * kBN + 128;
        }
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&S.empty[s], ph ^ 1, abort_flag, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          if (p.inject_stall && blockIdx.x == 0 && it == 0) {
            skipped = it;       // test hook: never fill this stage
            continue;
          }
          uint8_t* a = sA + s * kABytes;
          uint8_t* b = sB + s * kBBytes;
          mbar_arrive_expect_tx(&S.full[s], kStageBytes);
          tma_load_2d(a, &tm_a, &S.full[s], kb * kBK, c.row0, pol_a);
          tma_load_3d(b, &tm_b, &S.full[s], kb * kBK, brow0, c.e, pol_b);
          tma_load_3d(b + kBBytes / 2, &tm_b, &S.full[s], kb * kBK, brow1, c.e, pol_b);
        }
      }
      if (!ok) {
        // wait (bounded) for copies that may still be landing on this CTA's barriers
        for (int j = max(0, it - kStages); j < it; ++j) {
          if (j == skipped) continue;
          mbar_wait_drain(&S.full[j % kStages], (j / kStages) & 1, p.wait_limit_ns);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_e4m3_f32(kTileM, kBN);
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
        const int sp = u % splits;
        const int nk = (sp + 1) * nkb / splits - sp * nkb / splits;
        for (int k = 0; k < nk; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&S.full[s], ph, abort_flag, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          const int b = it & 1;
          const uint32_t tph = (it >> 1) & 1;
          if (!mbar_wait(&S.tempty[b], tph ^ 1, abort_flag, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + b * kBN;
          const uint64_t a0 = sdesc_k_sw128(smem_u32(sA + s * kABytes));
          const uint64_t b0 = sdesc_k_sw128(smem_u32(sB + s * kBBytes));
#pragma unroll
          for (int k32 = 0; k32 < kBK / 32; ++k32)
            umma_e4m3(d, a0 + 2 * k32, b0 + 2 * k32, idesc, k32 > 0 ? 1u : 0u);
          umma_commit(&S.empty[s]);
          umma_commit(&S.tfull[b]);
        }
      }
      if (!ok && it > 0) {
        const int last = it - 1;
        mbar_wait_drain(&S.tfull[last & 1], (last >> 1) & 1, p.wait_limit_ns);
      }
    } else if (warp == 2 || warp == 3) {
      // ------------------------------------------------ weight-scale loader (64 threads)
      // one tile ahead of the epilogue: the two weight-block scale rows of every tile this
      // CTA runs, in the order it runs them
      const int tl = threadIdx.x - 64;
      int j = 0;
      for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++j) {
        const int tile = u / splits;
        const TileCoord c = decode_tile(tile, p.n_tiles, p.slice_first, S.mtile, p.G, S.goff);
        const int r0 = EPI == EPI_SWIGLU ? c.nt : 2 * c.nt;
        const int r1 = EPI == EPI_SWIGLU ? p.I / 128 + c.nt : 2 * c.nt + 1;
        const float* w0 = p.w_scale + (static_cast<size_t>(c.e) * p.ws_rows + r0) * nkb;
        const float* w1 = p.w_scale + (static_cast<size_t>(c.e) * p.ws_rows + r1) * nkb;
        const int slot = j & 1;
        int got = 1;
        if (lane == 0) got = mbar_wait(&S.wempty[slot], ((j >> 1) & 1) ^ 1, abort_flag, p.status, p.wait_limit_ns);
        if (!__shfl_sync(0xffffffffu, got, 0)) break;
        for (int i = tl; i < nkb; i += 64) {
          S.wring[slot][0][i] = __ldg(w0 + i);
          S.wring[slot][1][i] = __ldg(w1 + i);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.wfull[slot]);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpilogueRegs));
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 4;
    const int half = ew >> 2;
    const int q = warp & 3;                 // TMEM lane quadrant this warp may access
    const int trow = 32 * q + lane;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    int kbg = 0, titer = 0;
    bool ok = true;
    // the combine reductions go to L2 as evict-first: in column-slice order a token row's
    // accumulators of one slice are live only while the slice runs, and the intermediate
    // (evict-last, re-read by every slice) should keep its place (W2 DRAM traffic 1.45 ->
    // 1.2 GB per launch on the 4096-token DeepSeek-V3 share, 10 us faster)
    const uint64_t pol_acc = policy_evict_first();
    for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x, ++titer) {
      const int tile = u / splits, sp = u - tile * splits;
      const int kb0 = sp * nkb / splits, kb1 = (sp + 1) * nkb / splits;
      const TileCoord c = decode_tile(tile, p.n_tiles, p.slice_first, S.mtile, p.G, S.goff);
      const int grow = c.row0 + trow;
      const bool valid = trow < c.rows;
      int c0, c1;
      if (EPI == EPI_SWIGLU) {
        c0 = 64 * half;
        c1 = 128 + 64 * half;
      } else {
        c0 = 128 * half;
        c1 = 128 * half + 64;
      }
      // this tile's weight-block scales, loaded by warps 2..3: SWIGLU gate row (s0) and up
      // row (s1); COMBINE the row of this warp's 128 output columns (both)
      const int wslot = titer & 1;
      // every lane waits (acquire) before reading the slot the loader warps wrote
      if (!__all_sync(0xffffffffu, mbar_wait(&S.wfull[wslot], (titer >> 1) & 1, abort_flag, p.status,
                                            p.wait_limit_ns))) {
        ok = false;
        break;
      }
      const float* ws0 = S.wring[wslot][EPI == EPI_SWIGLU ? 0 : half];
      const float* ws1 = S.wring[wslot][EPI == EPI_SWIGLU ? 1 : half];
      // COMBINE: the row's destination and top-K weight, fetched before the K loop
      int dst_mt = -1;
      float wgt = 0.f;
      if (EPI == EPI_COMBINE && valid) {
        dst_mt = p.row_mt[grow];
        wgt = p.row_w[grow];
      }
      // acc[j] holds columns (2j, 2j+1) of this thread's 128: [0,32) from the first
      // 64-column group, [32,64) from the second
      float2 acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
      // the row scales of K block kb+2 are fetched while block kb is processed (their L2
      // latency under the operand stream is longer than one K block)
      const float* sap = p.sa_t + grow;
      float sa_n = sap[static_cast<size_t>(kb0) * p.rpad];
      float sa_n2 = kb0 + 1 < kb1 ? sap[static_cast<size_t>(kb0 + 1) * p.rpad] : 0.f;
      // W13: two K blocks per loop body, and the row-scale fetch branch-free (the last
      // block's scale is fetched again at the end), so that the compiler schedules the
      // TMEM loads and FMAs of two blocks together (W13 780 -> 700 us on the 4096-token
      // DeepSeek-V3 share; W2, with 16 K blocks per tile, is better left as it is)
#pragma unroll(EPI == EPI_SWIGLU ? 2 : 1)
      for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
        const float s0 = sa_n * ws0[kb];
        const float s1 = sa_n * ws1[kb];
        sa_n = sa_n2;
        if (EPI == EPI_SWIGLU)
          sa_n2 = sap[static_cast<size_t>(min(kb + 2, kb1 - 1)) * p.rpad];
        else if (kb + 2 < kb1)
          sa_n2 = sap[static_cast<size_t>(kb + 2) * p.rpad];
        const int b = kbg & 1;
        const uint32_t tph = (kbg >> 1) & 1;
        int got = 1;
        if (lane == 0) got = mbar_wait(&S.tfull[b], tph, abort_flag, p.status, p.wait_limit_ns);
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tq + b * kBN;
        const float2 S0 = make_float2(s0, s0), S1 = make_float2(s1, s1);
        {
          float v[32], w[32];
          tmem_ld32(tb + c0, v);
          tmem_ld32(tb + c0 + 32, w);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), S0, acc[i]);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            acc[16 + i] = __ffma2_rn(make_float2(w[2 * i], w[2 * i + 1]), S0, acc[16 + i]);
        }
        {
          float v[32], w[32];
          tmem_ld32(tb + c1, v);
          tmem_ld32(tb + c1 + 32, w);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.tempty[b]);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            acc[32 + i] = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), S1, acc[32 + i]);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            acc[48 + i] = __ffma2_rn(make_float2(w[2 * i], w[2 * i + 1]), S1, acc[48 + i]);
        }
      }
      if (!ok) break;
      // the tile's weight scales are read: their slot may be refilled
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.wempty[wslot]);

      if (EPI == EPI_SWIGLU && splits > 1) {
        // this unit's partial sum into G; the warp whose partial completes the tile's
        // quadrant (two warps per split) finishes those 32 rows from G
        if (valid) {
          float* gr = p.g_ws + static_cast<size_t>(grow) * (2 * p.I) + c.nt * 128 + 64 * half;
#pragma unroll
          for (int i = 0; i < 16; ++i) red_add_v4(gr + 4 * i, acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x, acc[2 * i + 1].y);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            red_add_v4(gr + p.I + 4 * i, acc[32 + 2 * i].x, acc[32 + 2 * i].y, acc[33 + 2 * i].x, acc[33 + 2 * i].y);
        }
        // one add per warp after every lane has fenced its reductions (two warps per split)
        __threadfence();
        __syncwarp();
        int* cnt = p.g_cnt + tile * 4 + q;
        int old = 0;
        if (lane == 0) old = atomicAdd(cnt, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == 2 * splits - 1) {
          __threadfence();
          split_swiglu_rows(p, c.row0 + 32 * q, min(32, max(0, c.rows - 32 * q)), c.nt, lane);
          __syncwarp();
          if (lane == 0) *cnt = 0;          // zero again for the next call
        }
        continue;
      }
      if (EPI == EPI_SWIGLU) {
        // h = silu(g) * u on this thread's 64 channels; block amax shared with the partner
        // warp that holds the other 64 channels of the same rows
        float amax = 0.f;
        float hv[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 g = acc[i], u = acc[32 + i];
          hv[2 * i] = silu_mul(g.x, u.x);
          hv[2 * i + 1] = silu_mul(g.y, u.y);
          amax = fmaxf(amax, fmaxf(fabsf(hv[2 * i]), fabsf(hv[2 * i + 1])));
        }
        float* ax = &S.amax[titer & 1][0][0];
        ax[half * kTileM + trow] = amax;
        mbar_arrive(&S.pair[q]);
        if (!mbar_wait(&S.pair[q], titer & 1, abort_flag, p.status, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        amax = fmaxf(amax, ax[(half ^ 1) * kTileM + trow]);
        // block scale amax/448; codes = e4m3(h * (1/scale)), decided in fp32 with one
        // correctly rounded reciprocal per row block
        const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
        const float rsc = __frcp_rn(sc);
        if (valid) {
          uint4 out[4];
          uint16_t* o16 = reinterpret_cast<uint16_t*>(out);
#pragma unroll
          for (int i = 0; i < 32; ++i) o16[i] = pack_e4m3x2(hv[2 * i] * rsc, hv[2 * i + 1] * rsc);
          uint4* dst = reinterpret_cast<uint4*>(p.hq + static_cast<size_t>(grow) * p.I +
                                                c.nt * 128 + 64 * half);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = out[j];
          if (half == 0) p.sh_t[static_cast<size_t>(c.nt) * p.rpad + grow] = sc;
        }
      } else {
        // weighted combine: this warp's 32 rows x 128 columns, times each row's top-K
        // weight, go to the token accumulators as bulk reductions (one 512-byte row
        // segment each). Eight lanes at a time fill one of the warp's two staging buffers
        // and issue their rows; before a buffer is refilled, the lanes that issued from it
        // last wait until the bulk engine has read it.
        const int col0 = c.nt * kBN + half * 128;
        float* dst = nullptr;
        if (dst_mt >= 0)
          dst = p.acc.a[dst_mt >> 24] + static_cast<size_t>(dst_mt & 0xFFFFFF) * p.H + col0;
        uint8_t* wst = stg + ew * kStgWarpBytes;
#pragma unroll
        for (int r8 = 0; r8 < 4; ++r8) {
          uint8_t* buf = wst + (r8 & 1) * kStgBufBytes;
          if ((lane >> 3) == ((r8 + 2) & 3)) bulk_wait_read_all();
          __syncwarp();
          if ((lane >> 3) == r8) {
            float* row = reinterpret_cast<float*>(buf + (lane & 7) * kStgRowBytes);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float2 a = acc[2 * i], bb = acc[2 * i + 1];
              *reinterpret_cast<float4*>(row + 4 * i) = make_float4(a.x * wgt, a.y * wgt, bb.x * wgt, bb.y * wgt);
            }
            fence_proxy_async_shared();
            if (dst) bulk_reduce_add_f32(dst, row, 512, pol_acc);
            bulk_commit();
          }
        }
      }
    }
    // every bulk reduction issued by this thread has been performed before the CTA exits
    if (EPI == EPI_COMBINE) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Combine, last step: every token's fp32 sum -> bf16 into its slab row; the accumulator
// is cleared for the next call. One warp per (token row, 256-column segment), 16-byte
// stores, so that a few tokens still spread over many warps (the row's segments are
// independent requests, not a chain of them).
__global__ void __launch_bounds__(256) combine_finalize_kernel(const int32_t* __restrict__ info,
                                                               const int32_t* __restrict__ tok_mt,
                                                               const __grid_constant__ AccTable acc, int H,
                                                               const __grid_constant__ YTable ytab) {
  pdl_trigger();
  pdl_wait();
  const int T = info[0];
  const int lane = threadIdx.x & 31;
  const int nseg = H / 256;                 // H is a multiple of 256
  const int items = T * nseg;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int it = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
    const int g = it / nseg;
    const int c = (it - g * nseg) * 256 + lane * 8;
    const int mt = tok_mt[g];
    const int m = mt >> 24, t = mt & 0xFFFFFF;
    float* row = acc.a[m] + static_cast<size_t>(t) * H;
    __nv_bfloat16* y = ytab.y[m] + static_cast<size_t>(t) * H;
    const float4 a = __ldcg(reinterpret_cast<const float4*>(row + c));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(row + c + 4));
    uint4 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    o.z = pack_bf16x2(b.x, b.y);
    o.w = pack_bf16x2(b.z, b.w);
    *reinterpret_cast<uint4*>(y + c) = o;
    __stcg(reinterpret_cast<float4*>(row + c), make_float4(0.f, 0.f, 0.f, 0.f));
    __stcg(reinterpret_cast<float4*>(row + c + 4), make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

// Expert-parallel return path, on the owner of the slabs: once every FFN GPU has added
// its partial rows, token t < n_m of slab m becomes bf16 in y[m] and its accumulator row
// is cleared. One warp per (slab, token, 256-column segment); blockIdx.y = slab.
__global__ void __launch_bounds__(256) combine_finalize_slabs_kernel(const int32_t* __restrict__ counts,
                                                                     int cap, int H,
                                                                     const __grid_constant__ AccTable acc,
                                                                     const __grid_constant__ YTable ytab) {
  const int m = blockIdx.y;
  const int n = min(max(counts[m], 0), cap);
  const int lane = threadIdx.x & 31;
  const int nseg = H / 256;
  const int items = n * nseg;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int it = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
    const int t = it / nseg;
    const int c = (it - t * nseg) * 256 + lane * 8;
    float* row = acc.a[m] + static_cast<size_t>(t) * H;
    __nv_bfloat16* y = ytab.y[m] + static_cast<size_t>(t) * H;
    const float4 a = __ldcg(reinterpret_cast<const float4*>(row + c));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(row + c + 4));
    uint4 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    o.z = pack_bf16x2(b.x, b.y);
    o.w = pack_bf16x2(b.z, b.w);
    *reinterpret_cast<uint4*>(y + c) = o;
    __stcg(reinterpret_cast<float4*>(row + c), make_float4(0.f, 0.f, 0.f, 0.f));
    __stcg(reinterpret_cast<float4*>(row + c + 4), make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

}  // namespace afd
