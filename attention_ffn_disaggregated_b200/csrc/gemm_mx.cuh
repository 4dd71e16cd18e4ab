// W13 grouped GEMM on the tensor core's block-scale path (tiling 2), for inputs whose
// block scales are all powers of two: FastAFD, "Methodology / System Design", item 1
// (block-FP8 expert precision) and item 3 (block-FP8 grouped GEMMs, activation).
//
// A power-of-two fp32 scale 2^e is exactly the UE8M0 factor whose byte is e + 127, i.e.
// its fp32 exponent field. tcgen05.mma kind::mxf8f6f4.block_scale multiplies each 32-wide
// K slice of a row of A and of a column of B by such factors inside the tensor core, so
// TMEM accumulates a tile's whole K loop and the epilogue reads the accumulator once per
// tile, instead of promoting one partial product per K block in registers as
// grouped_gemm_kernel must for arbitrary fp32 scales. Each per-128 scale serves the four
// K slices of its block.
//
// Factor images. The MMA reads its factors from TMEM, where tcgen05.cp places them from
// shared memory. For 128 rows (or B columns) and one 128-wide K block the image is 512
// bytes: byte (i % 32) * 16 + (i / 32) * 4 + j holds the factor of row i for K slice j
// (the four j are equal here). mx_act_sf_kernel writes the images of the activation rows
// of every m-tile and K block after the gather; mx_weight_sf_kernel writes those of every
// 128-row block of W13 once per plan. The producer copies three images per stage (A, gate
// block, up block) next to the operand tiles. In TMEM an image occupies four columns: row
// i at lane i % 32 of every lane quadrant, column i / 32.
//
// Roles (384 threads, the register split of grouped_gemm_kernel): warp 0 loads, warp 1
// owns TMEM and issues the factor copies and the MMAs, warps 4..11 read the accumulator
// and run the SwiGLU + requantisation epilogue. TMEM: the 128 x 256 fp32 accumulator in
// columns [0, 256), then 16 columns of factors per pipeline stage (A at +0, B at +8). With
// one accumulator the next tile's first MMA waits until the epilogue has copied the
// previous tile's accumulator into registers, not for the rest of its epilogue.
#pragma once

#include "gemm.cuh"

namespace afd {

constexpr int kMxStages = 4;
constexpr uint32_t kSfImage = 512;                 // bytes per 128 rows x one 128-wide K block
constexpr uint32_t kSfStage = 3 * kSfImage;        // A rows, W13 gate block, W13 up block
constexpr uint32_t kMxSfCol = 256;                 // first factor column in TMEM
constexpr uint32_t kMxSfCols = 16;                 // factor columns per stage
constexpr size_t kMxTiles = static_cast<size_t>(kMxStages) * kStageBytes;
static_assert(kMxSfCol + kMxStages * kMxSfCols <= kTmemCols, "factor columns exceed TMEM");

struct alignas(16) MxSmem {
  uint64_t full[kMxStages];
  uint64_t empty[kMxStages];
  uint64_t tfull;
  uint64_t tempty;
  uint64_t pair[4];           // amax exchange between the two warps of a lane quadrant
  uint32_t tmem_base;
  int abort_flag;
  float amax[2][2][kTileM];
  int32_t mtile[AFD_MAX_GROUPS + 1];
};

__host__ __device__ constexpr size_t mx_smem_bytes() {
  return 1024 + kMxTiles + kMxStages * kSfStage + sizeof(MxSmem);
}

struct MxArgs {
  const uint8_t* sfa;         // [m-tiles][num_kb] images of the activation rows
  const uint8_t* sfb;         // [E][2I/128][num_kb] images of the W13 row blocks
};

// UE8M0 byte of a power-of-two scale; `bad` when the scale is not a positive normal power
// of two (the factor would not equal it).
__device__ __forceinline__ uint32_t ue8m0_of(float s, bool& bad) {
  const uint32_t bits = __float_as_uint(s);
  const uint32_t e = (bits >> 23) & 0xFFu;
  bad = (bits & 0x807FFFFFu) != 0 || e == 0u || e == 0xFFu;
  return e;
}

// Images of every (expert, 128-row block, 128-wide K block) of W13: image u belongs to
// scale u of the [E][2I/128][H/128] scale array. One warp per image, 16 bytes per lane.
__global__ void __launch_bounds__(256) mx_weight_sf_kernel(const float* __restrict__ w_scale,
                                                           int n_images, uint8_t* __restrict__ img,
                                                           int* status) {
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int u = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; u < n_images; u += nwarps) {
    bool bad;
    const uint32_t e = ue8m0_of(w_scale[u], bad);
    if (bad && lane == 0) atomicOr(status, AFD_STATUS_BAD_SCALE);
    const uint32_t w = e * 0x01010101u;
    reinterpret_cast<uint4*>(img + static_cast<size_t>(u) * kSfImage)[lane] = make_uint4(w, w, w, w);
  }
}

// Images of the activation rows of every (m-tile, K block), from the expert-ordered scales
// `sa_t` [num_kb][rpad] written by the gather stage. One block of 128 threads per image,
// thread i for row i of the m-tile; rows past the expert's last row are imaged too (their
// results are discarded) but only the expert's own rows are checked.
__global__ void __launch_bounds__(128) mx_act_sf_kernel(const int32_t* __restrict__ mtile_off,
                                                        const int32_t* __restrict__ group_off, int G,
                                                        const float* __restrict__ sa_t, int rpad,
                                                        int num_kb, uint8_t* __restrict__ img,
                                                        int* status) {
  const int n_img = mtile_off[G] * num_kb;
  const int i = threadIdx.x;
  for (int u = blockIdx.x; u < n_img; u += gridDim.x) {
    const int mt = u / num_kb, kb = u - mt * num_kb;
    const TileCoord c = decode_tile(mt, 1, 0, mtile_off, G, group_off);
    bool bad;
    const uint32_t e = ue8m0_of(sa_t[static_cast<size_t>(kb) * rpad + c.row0 + i], bad);
    if (bad && i < c.rows) atomicOr(status, AFD_STATUS_BAD_SCALE);
    *reinterpret_cast<uint32_t*>(img + static_cast<size_t>(u) * kSfImage + (i & 31) * 16 + (i >> 5) * 4) =
        e * 0x01010101u;
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    w13_mx_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tm_a,
                  const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ MxArgs mx) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = base;
  uint8_t* sB = base + kMxStages * kABytes;
  uint8_t* sF = base + kMxTiles;
  MxSmem& S = *reinterpret_cast<MxSmem*>(sF + kMxStages * kSfStage);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMxStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.tfull, 1);
    mbar_init(&S.tempty, kEpiWarps);
    for (int i = 0; i < 4; ++i) mbar_init(&S.pair[i], 64);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  // everything above is local set-up; the tile schedule and the operands come from the
  // previous kernels
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i <= p.G; i += blockDim.x) S.mtile[i] = p.mtile_off[i];
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;
  const int total_tiles = S.mtile[p.G] * p.n_tiles;
  const int nkb = p.num_kb;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- loads
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      // A rows are re-read by every column tile of their m-tile, W13 blocks by every m-tile
      // of their expert
      const uint64_t pol = policy_evict_last();
      const int nbw = 2 * p.I / 128;       // 128-row blocks of one expert's W13
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileCoord c = decode_tile(tile, p.n_tiles, 0, S.mtile, p.G, p.group_off);
        const int brow0 = c.nt * 128;              // gate block
        const int brow1 = p.I + c.nt * 128;        // up block
        const uint8_t* fa = mx.sfa + static_cast<size_t>(c.mt) * nkb * kSfImage;
        const uint8_t* fg = mx.sfb + (static_cast<size_t>(c.e) * nbw + c.nt) * nkb * kSfImage;
        const uint8_t* fu = mx.sfb + (static_cast<size_t>(c.e) * nbw + p.I / 128 + c.nt) * nkb * kSfImage;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kMxStages;
          const uint32_t ph = (it / kMxStages) & 1;
          if (!mbar_wait(&S.empty[s], ph ^ 1, abort_flag, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          uint8_t* a = sA + s * kABytes;
          uint8_t* b = sB + s * kBBytes;
          uint8_t* f = sF + s * kSfStage;
          mbar_arrive_expect_tx(&S.full[s], kStageBytes + kSfStage);
          tma_load_2d(a, &tm_a, &S.full[s], kb * kBK, c.row0, pol);
          tma_load_3d(b, &tm_b, &S.full[s], kb * kBK, brow0, c.e, pol);
          tma_load_3d(b + kBBytes / 2, &tm_b, &S.full[s], kb * kBK, brow1, c.e, pol);
          bulk_load(f, fa + static_cast<size_t>(kb) * kSfImage, kSfImage, &S.full[s]);
          bulk_load(f + kSfImage, fg + static_cast<size_t>(kb) * kSfImage, kSfImage, &S.full[s]);
          bulk_load(f + 2 * kSfImage, fu + static_cast<size_t>(kb) * kSfImage, kSfImage, &S.full[s]);
        }
      }
      if (!ok) {
        // wait (bounded) for copies that may still be landing on this CTA's barriers
        for (int j = max(0, it - kMxStages); j < it; ++j)
          mbar_wait_drain(&S.full[j % kMxStages], (j / kMxStages) & 1, p.wait_limit_ns);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- factor copies + MMA
      constexpr uint32_t idesc = idesc_mx_e4m3(kTileM, kBN);
      int it = 0, titer = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++titer) {
        // the accumulator is free once the epilogue has read the previous tile's
        if (!mbar_wait(&S.tempty, (titer & 1) ^ 1, abort_flag, p.status, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kMxStages;
          const uint32_t ph = (it / kMxStages) & 1;
          if (!mbar_wait(&S.full[s], ph, abort_flag, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t f = smem_u32(sF + s * kSfStage);
          const uint32_t tsfa = tmem_base + kMxSfCol + s * kMxSfCols;
          const uint32_t tsfb = tsfa + 8;
          tmem_cp_32x128b_x4(tsfa, sdesc_rows16(f));
          tmem_cp_32x128b_x4(tsfb, sdesc_rows16(f + kSfImage));           // columns 0..127
          tmem_cp_32x128b_x4(tsfb + 4, sdesc_rows16(f + 2 * kSfImage));   // columns 128..255
          const uint64_t a0 = sdesc_k_sw128(smem_u32(sA + s * kABytes));
          const uint64_t b0 = sdesc_k_sw128(smem_u32(sB + s * kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            umma_mx_e4m3(tmem_base, a0 + 2 * k, b0 + 2 * k, idesc, tsfa, tsfb, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&S.empty[s]);
        }
        if (!ok) break;
        umma_commit(&S.tfull);
      }
      if (!ok && it > 0) {
        // wait (bounded) for the MMAs already issued before TMEM is released
        const int last = it - 1;
        mbar_wait_drain(&S.empty[last % kMxStages], (last / kMxStages) & 1, p.wait_limit_ns);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpilogueRegs));
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 4;
    const int half = ew >> 2;               // which 64 of the 128 gate (and up) columns
    const int q = warp & 3;                 // TMEM lane quadrant this warp may access
    const int trow = 32 * q + lane;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    const int c0 = 64 * half, c1 = 128 + 64 * half;
    int titer = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++titer) {
      const TileCoord c = decode_tile(tile, p.n_tiles, 0, S.mtile, p.G, p.group_off);
      const int grow = c.row0 + trow;
      const bool valid = trow < c.rows;
      int got = 1;
      if (lane == 0) got = mbar_wait(&S.tfull, titer & 1, abort_flag, p.status, p.wait_limit_ns);
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      float g0[32], g1[32], u0[32], u1[32];   // gate and up channels of this thread's row
      tmem_ld32(tq + c0, g0);
      tmem_ld32(tq + c0 + 32, g1);
      tmem_ld32(tq + c1, u0);
      tmem_ld32(tq + c1 + 32, u1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.tempty);

      // h = silu(g) * u on this thread's 64 channels (into g0, g1); silu(g) = g / (1 +
      // exp(-g)) with branch-free fast exp and division, g clamped at -80 where silu is 0
      // to fp32 precision
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float ga = fmaxf(g0[i], -80.0f), gb = fmaxf(g1[i], -80.0f);
        g0[i] = __fdividef(ga, 1.0f + __expf(-ga)) * u0[i];
        g1[i] = __fdividef(gb, 1.0f + __expf(-gb)) * u1[i];
        amax = fmaxf(amax, fmaxf(fabsf(g0[i]), fabsf(g1[i])));
      }
      // block amax shared with the partner warp that holds the other 64 channels
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
        for (int i = 0; i < 16; ++i) {
          o16[i] = pack_e4m3x2(g0[2 * i] * rsc, g0[2 * i + 1] * rsc);
          o16[16 + i] = pack_e4m3x2(g1[2 * i] * rsc, g1[2 * i + 1] * rsc);
        }
        uint4* dst = reinterpret_cast<uint4*>(p.hq + static_cast<size_t>(grow) * p.I + c.nt * 128 + 64 * half);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = out[j];
        if (half == 0) p.sh_t[static_cast<size_t>(c.nt) * p.rpad + grow] = sc;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace afd
