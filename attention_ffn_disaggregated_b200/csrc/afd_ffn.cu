// Host side of the C ABI declared in include/afd_ffn.h: argument validation, workspace
// layout, TMA descriptor encoding and the launch sequence of one layer call
// (route count -> route scan -> route scatter -> row gather -> W13 GEMM -> W2 GEMM ->
// combine finalisation).
//
// The FFN service of an AFD deployment receives activations and routing metadata,
// computes the FFN output and returns it (vLLM AFD plugin, "FFN service"); FastAFD runs
// the FFN side as one persistent kernel per layer (FastAFD, "Methodology / System
// Design", item 3). Here the work is split into seven stream-ordered launches that never
// synchronise with the host.
#include <cuda_runtime.h>
#include <cuda.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>

#include "afd_ffn.h"
#include "gemm.cuh"
#include "gemm_mx.cuh"
#include "route.cuh"

using namespace afd;

// Tile order of the down projection: column-tile major (every m-tile of a 256-column
// slice before the next slice). Each slice's weight rows are then read from DRAM once,
// while the intermediate (re-read by every slice, evict-last) and the slice's live
// accumulators stay in L2; in m-tile-major order the 117 MB of accumulators crowd the
// weights out of L2 between an expert's m-tiles (3.8x the algorithmic DRAM traffic on the
// DeepSeek-V3 share) at the same kernel time.
#ifndef AFD_W2_SLICE_FIRST
#define AFD_W2_SLICE_FIRST 1
#endif


namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn) return fn;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  fn = reinterpret_cast<EncodeTiledFn>(p);
  return fn;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// One kernel launch; with `pdl` the kernel may start while the previous kernel in the
// stream is still running (programmatic stream serialisation) and waits for it on the
// device (pdl_wait) before touching its results.
template <typename... KArgs, typename... Args>
static void launch(bool pdl, void (*kernel)(KArgs...), int grid, int block, size_t smem,
                   cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace

struct afd_ffn_plan_s {
  afd_ffn_config_t cfg;
  afd_ffn_weights_t w;
  int device = 0, num_sms = 0;
  int G = 0, Tmax = 0, Rmax = 0, rpad = 0, num_chunks = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int32_t *slab_base, *info, *chunk_hist, *chunk_off, *group_count, *group_off, *mtile_off;
  int tiling = 0;  // 0 = default (1); 2 = block-scale W13
  int32_t *tok_mt, *tok_need, *pos, *row_token, *row_mt, *row_k;
  float* g_ws;        // split-K W13: fp32 sums [g_rows][2I], zero between calls
  int g_rows = 0;
  int* g_cnt;         // split-K W13: per (tile, quadrant) counters [num_sms][4]
  float *row_w, *sa_t, *sh_t, *acc;
  uint8_t *a_perm, *hq;
  int* status;
  int* scan_ticket;   // route_count's last-block counter, zero between calls
  // tiling 2 (block-scale W13): factor images of the activation rows (workspace) and of
  // W13 (allocated and built when the tiling is first selected)
  uint8_t* mx_sfa;
  uint8_t* mx_sfb = nullptr;
  CUtensorMap tm_a13, tm_w13, tm_a2, tm_w2;
  int w2_slice_first = AFD_W2_SLICE_FIRST;
  bool timing = false, ev_valid = false;
  cudaEvent_t ev[AFD_NUM_KERNELS + 1] = {};
  unsigned long long wait_limit_ns = 1000000000ull;
  int inject_stall = 0;
  size_t scatter_smem = 0;
  // combine destinations: the plan's own accumulators (slab m at acc + m*cap*H), or the
  // caller's (afd_ffn_set_combine_targets; the layer then stops after W2)
  AccTable own_acc;
  AccTable ext_acc;
  bool external_acc = false;
};

extern "C" {

const char* afd_status_string(afd_status_t s) {
  switch (s) {
    case AFD_OK: return "AFD_OK";
    case AFD_ERR_INVALID_ARGUMENT: return "AFD_ERR_INVALID_ARGUMENT";
    case AFD_ERR_UNSUPPORTED: return "AFD_ERR_UNSUPPORTED";
    case AFD_ERR_OUT_OF_MEMORY: return "AFD_ERR_OUT_OF_MEMORY";
    case AFD_ERR_CUDA: return "AFD_ERR_CUDA";
    case AFD_ERR_BAD_ROUTING: return "AFD_ERR_BAD_ROUTING";
    case AFD_ERR_TIMEOUT: return "AFD_ERR_TIMEOUT";
  }
  return "unknown";
}

// route count (+ scan), scatter, gather, W13, W2, finalisation (a plan of at most
// kSmallRouteChunks routing chunks runs the routing as one launch); the block-scale
// tiling adds the activation factor images
int32_t afd_ffn_kernels_per_layer(afd_ffn_plan_t P) {
  if (!P) return -1;
  return (P->num_chunks <= kSmallRouteChunks ? 5 : 6) + (P->tiling == 2 ? 1 : 0) - (P->external_acc ? 1 : 0);
}

afd_status_t afd_ffn_check_config(const afd_ffn_config_t* c) {
  if (!c) return AFD_ERR_INVALID_ARGUMENT;
  if (c->hidden < AFD_QBLOCK || c->hidden % AFD_QBLOCK) return AFD_ERR_INVALID_ARGUMENT;
  if (c->intermediate < AFD_QBLOCK || c->intermediate % AFD_QBLOCK) return AFD_ERR_INVALID_ARGUMENT;
  if (c->num_experts_global < 1 || c->expert_begin < 0 || c->num_local_experts < 0)
    return AFD_ERR_INVALID_ARGUMENT;
  if (static_cast<int64_t>(c->expert_begin) + c->num_local_experts > c->num_experts_global)
    return AFD_ERR_INVALID_ARGUMENT;
  if (c->has_shared_expert != 0 && c->has_shared_expert != 1) return AFD_ERR_INVALID_ARGUMENT;
  if (c->num_local_experts + c->has_shared_expert < 1) return AFD_ERR_INVALID_ARGUMENT;
  if (c->top_k < 1 || c->top_k > c->num_experts_global) return AFD_ERR_INVALID_ARGUMENT;
  if (c->num_slabs < 1 || c->slab_capacity < 1) return AFD_ERR_INVALID_ARGUMENT;
  // supported limits
  if (c->hidden % 256) return AFD_ERR_UNSUPPORTED;   // W2 output tiles are 256 columns
  if (c->hidden > AFD_QBLOCK * AFD_MAX_QBLOCKS || c->intermediate > AFD_QBLOCK * AFD_MAX_QBLOCKS)
    return AFD_ERR_UNSUPPORTED;                      // K blocks held in the GEMMs' scale ring
  if (c->top_k > AFD_MAX_TOP_K) return AFD_ERR_UNSUPPORTED;
  if (c->num_slabs > AFD_MAX_SLABS) return AFD_ERR_UNSUPPORTED;
  if (c->num_local_experts + c->has_shared_expert > AFD_MAX_GROUPS) return AFD_ERR_UNSUPPORTED;
  if (c->slab_capacity >= (1 << 24)) return AFD_ERR_UNSUPPORTED;
  const int64_t tmax = static_cast<int64_t>(c->num_slabs) * c->slab_capacity;
  const int64_t kl = std::min(c->top_k, c->num_local_experts) + c->has_shared_expert;
  if (tmax * c->top_k >= (int64_t{1} << 31) || tmax * kl + 256 >= (int64_t{1} << 31))
    return AFD_ERR_UNSUPPORTED;
  if ((tmax * kl + 256) * std::max(c->hidden, c->intermediate) >= (int64_t{1} << 40))
    return AFD_ERR_UNSUPPORTED;
  return AFD_OK;
}

static afd_status_t encode_2d(EncodeTiledFn enc, CUtensorMap* m, void* base, uint64_t inner,
                              uint64_t rows) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? AFD_OK : AFD_ERR_CUDA;
}

static afd_status_t encode_3d(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t inner,
                              uint64_t rows, uint64_t experts, uint32_t box_rows) {
  cuuint64_t dims[3] = {inner, rows, experts};
  cuuint64_t strides[2] = {inner, inner * rows};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? AFD_OK : AFD_ERR_CUDA;
}

afd_status_t afd_ffn_plan(const afd_ffn_config_t* cfg, const afd_ffn_weights_t* weights,
                          afd_ffn_plan_t* out) {
  if (!out) return AFD_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  afd_status_t st = afd_ffn_check_config(cfg);
  if (st != AFD_OK) return st;
  if (!weights || !weights->w13 || !weights->w2 || !weights->w13_scale || !weights->w2_scale)
    return AFD_ERR_INVALID_ARGUMENT;
  if (!aligned(weights->w13, 16) || !aligned(weights->w2, 16) || !aligned(weights->w13_scale, 4) ||
      !aligned(weights->w2_scale, 4))
    return AFD_ERR_INVALID_ARGUMENT;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AFD_ERR_UNSUPPORTED;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return AFD_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return AFD_ERR_UNSUPPORTED;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return AFD_ERR_CUDA;
  // The GEMM kernels split the block's registers between warpgroups with setmaxnreg; that
  // is only safe when the block is launched with exactly the budget the split assumes.
  {
    const void* fns[3] = {reinterpret_cast<const void*>(w13_mx_kernel),
                          reinterpret_cast<const void*>(grouped_gemm_kernel<EPI_SWIGLU>),
                          reinterpret_cast<const void*>(grouped_gemm_kernel<EPI_COMBINE>)};
    for (const void* fn : fns) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return AFD_ERR_CUDA;
      if (fa.numRegs != kLaunchRegs || fa.maxThreadsPerBlock < kGemmThreads) return AFD_ERR_UNSUPPORTED;
    }
  }

  afd_ffn_plan_s* P = new (std::nothrow) afd_ffn_plan_s();
  if (!P) return AFD_ERR_OUT_OF_MEMORY;
  P->cfg = *cfg;
  P->w = *weights;
  P->device = dev;
  P->num_sms = prop.multiProcessorCount;
  const int H = cfg->hidden, I = cfg->intermediate, K = cfg->top_k;
  const int El = cfg->num_local_experts, S = cfg->has_shared_expert;
  P->G = El + S;
  P->Tmax = cfg->num_slabs * cfg->slab_capacity;
  P->Rmax = P->Tmax * (std::min(K, El) + S);
  // a 128-row tile may start up to 127 rows before the end of the routed rows, and its
  // row-scale copy reads 132 entries from the 16-byte boundary at or below its first row
  P->rpad = ((P->Rmax + 256 + 127) / 128) * 128;
  P->num_chunks = (P->Tmax + kChunkTokens - 1) / kChunkTokens;
  const int El1 = std::max(El, 1);

  // workspace layout
  size_t off = 0;
  auto take = [&](size_t bytes, size_t align) {
    off = (off + align - 1) / align * align;
    size_t o = off;
    off += bytes;
    return o;
  };
  const size_t o_slab_base = take(sizeof(int32_t) * (cfg->num_slabs + 1), 16);
  const size_t o_info = take(sizeof(int32_t) * 16, 16);
  const size_t o_status = take(sizeof(int32_t) * 4, 16);
  const size_t o_ticket = take(sizeof(int32_t) * 4, 16);
  const size_t o_chunk_hist = take(sizeof(int32_t) * P->num_chunks * El1, 16);
  const size_t o_chunk_off = take(sizeof(int32_t) * P->num_chunks * El1, 16);
  const size_t o_group_count = take(sizeof(int32_t) * (P->G + 1), 16);
  const size_t o_group_off = take(sizeof(int32_t) * (P->G + 1), 16);
  const size_t o_mtile_off = take(sizeof(int32_t) * (P->G + 1), 16);
  const size_t o_tok_mt = take(sizeof(int32_t) * P->Tmax, 16);
  const size_t o_tok_need = take(sizeof(int32_t) * P->Tmax, 16);
  const size_t o_pos = take(sizeof(int32_t) * static_cast<size_t>(P->Tmax) * K, 16);
  const size_t o_row_token = take(sizeof(int32_t) * P->rpad, 16);
  const size_t o_row_mt = take(sizeof(int32_t) * P->rpad, 16);
  const size_t o_row_k = take(sizeof(int32_t) * P->rpad, 16);
  const size_t o_row_w = take(sizeof(float) * P->rpad, 16);
  const size_t o_a_perm = take(static_cast<size_t>(P->rpad) * H, 1024);
  const size_t o_sa_t = take(sizeof(float) * static_cast<size_t>(H / 128) * P->rpad, 256);
  const size_t o_hq = take(static_cast<size_t>(P->rpad) * I, 1024);
  const size_t o_sh_t = take(sizeof(float) * static_cast<size_t>(I / 128) * P->rpad, 256);
  const size_t o_acc = take(sizeof(float) * static_cast<size_t>(P->Tmax) * H, 256);
  // split-K W13 runs only while its tiles fill at most half of the grid: m-tiles <=
  // num_sms / (2 * I/128), so that many 128-row tiles bound the rows it touches
  P->g_rows = std::min(P->rpad, (P->num_sms / (2 * (I / 128)) + 1) * 128);
  const size_t o_g_ws = take(sizeof(float) * static_cast<size_t>(P->g_rows) * 2 * I, 256);
  const size_t o_g_cnt = take(sizeof(int) * static_cast<size_t>(P->num_sms) * 4, 16);
  const size_t o_mx_sfa = take(static_cast<size_t>(P->rpad / 128 + P->G) * (H / 128) * kSfImage, 256);
  P->ws_bytes = take(0, 256);

  if (cudaMalloc(&P->ws, P->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete P;
    return AFD_ERR_OUT_OF_MEMORY;
  }
  if (cudaMemset(P->ws, 0, P->ws_bytes) != cudaSuccess) {
    cudaFree(P->ws);
    delete P;
    return AFD_ERR_CUDA;
  }
  uint8_t* b = static_cast<uint8_t*>(P->ws);
  P->slab_base = reinterpret_cast<int32_t*>(b + o_slab_base);
  P->info = reinterpret_cast<int32_t*>(b + o_info);
  P->status = reinterpret_cast<int*>(b + o_status);
  P->scan_ticket = reinterpret_cast<int*>(b + o_ticket);
  P->chunk_hist = reinterpret_cast<int32_t*>(b + o_chunk_hist);
  P->chunk_off = reinterpret_cast<int32_t*>(b + o_chunk_off);
  P->group_count = reinterpret_cast<int32_t*>(b + o_group_count);
  P->group_off = reinterpret_cast<int32_t*>(b + o_group_off);
  P->mtile_off = reinterpret_cast<int32_t*>(b + o_mtile_off);
  P->tok_mt = reinterpret_cast<int32_t*>(b + o_tok_mt);
  P->tok_need = reinterpret_cast<int32_t*>(b + o_tok_need);
  P->pos = reinterpret_cast<int32_t*>(b + o_pos);
  P->row_token = reinterpret_cast<int32_t*>(b + o_row_token);
  P->row_mt = reinterpret_cast<int32_t*>(b + o_row_mt);
  P->row_k = reinterpret_cast<int32_t*>(b + o_row_k);
  P->row_w = reinterpret_cast<float*>(b + o_row_w);
  P->a_perm = b + o_a_perm;
  P->sa_t = reinterpret_cast<float*>(b + o_sa_t);
  P->hq = b + o_hq;
  P->sh_t = reinterpret_cast<float*>(b + o_sh_t);
  P->acc = reinterpret_cast<float*>(b + o_acc);
  memset(&P->own_acc, 0, sizeof(P->own_acc));
  for (int m = 0; m < cfg->num_slabs; ++m)
    P->own_acc.a[m] = P->acc + static_cast<size_t>(m) * cfg->slab_capacity * H;
  P->g_ws = reinterpret_cast<float*>(b + o_g_ws);
  P->g_cnt = reinterpret_cast<int*>(b + o_g_cnt);
  P->mx_sfa = b + o_mx_sfa;

  const int E = P->G;
  st = encode_2d(enc, &P->tm_a13, P->a_perm, H, P->rpad);
  if (st == AFD_OK) st = encode_3d(enc, &P->tm_w13, weights->w13, H, 2 * static_cast<uint64_t>(I), E, 128);
  if (st == AFD_OK) st = encode_2d(enc, &P->tm_a2, P->hq, I, P->rpad);
  if (st == AFD_OK) st = encode_3d(enc, &P->tm_w2, weights->w2, I, H, E, 128);

  if (st != AFD_OK) {
    cudaFree(P->ws);
    delete P;
    return st;
  }
  P->scatter_smem = scatter_smem_bytes(El1, K);
  if (cudaFuncSetAttribute(w13_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(mx_smem_bytes())) != cudaSuccess ||
      cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(gemm_smem_bytes<EPI_SWIGLU>())) != cudaSuccess ||
      cudaFuncSetAttribute(grouped_gemm_kernel<EPI_COMBINE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(gemm_smem_bytes<EPI_COMBINE>())) != cudaSuccess ||
      // the limit is a per-function setting shared by every plan: set the largest any
      // configuration can need, so that a later plan never lowers an earlier plan's limit
      cudaFuncSetAttribute(route_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(scatter_smem_bytes(AFD_MAX_GROUPS, AFD_MAX_TOP_K))) !=
          cudaSuccess ||
      cudaFuncSetAttribute(route_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(scatter_smem_bytes(AFD_MAX_GROUPS, AFD_MAX_TOP_K))) !=
          cudaSuccess) {
    cudaGetLastError();
    cudaFree(P->ws);
    delete P;
    return AFD_ERR_CUDA;
  }
  for (int i = 0; i <= AFD_NUM_KERNELS; ++i) {
    if (cudaEventCreate(&P->ev[i]) != cudaSuccess) {
      cudaGetLastError();
      for (int j = 0; j < i; ++j) cudaEventDestroy(P->ev[j]);
      cudaFree(P->ws);
      delete P;
      return AFD_ERR_CUDA;
    }
  }
  *out = P;
  return AFD_OK;
}

void afd_ffn_destroy(afd_ffn_plan_t P) {
  if (!P) return;
  cudaDeviceSynchronize();
  for (int i = 0; i <= AFD_NUM_KERNELS; ++i)
    if (P->ev[i]) cudaEventDestroy(P->ev[i]);
  if (P->ws) cudaFree(P->ws);
  if (P->mx_sfb) cudaFree(P->mx_sfb);
  delete P;
}

afd_status_t afd_ffn_get_info(afd_ffn_plan_t P, afd_ffn_plan_info_t* info) {
  if (!P || !info) return AFD_ERR_INVALID_ARGUMENT;
  info->num_groups = P->G;
  info->max_tokens = P->Tmax;
  info->max_rows = P->Rmax;
  info->num_sms = P->num_sms;
  info->workspace_bytes = static_cast<int64_t>(P->ws_bytes);
  return AFD_OK;
}

static void fill_route_params(afd_ffn_plan_t P, const int32_t* d_counts, RouteParams& rp) {
  const afd_ffn_config_t& c = P->cfg;
  memset(&rp, 0, sizeof(rp));
  rp.counts = d_counts;
  rp.M = c.num_slabs;
  rp.cap = c.slab_capacity;
  rp.K = c.top_k;
  rp.H = c.hidden;
  rp.e0 = c.expert_begin;
  rp.El = c.num_local_experts;
  rp.Eg = c.num_experts_global;
  rp.S = c.has_shared_expert;
  rp.G = P->G;
  rp.num_chunks = P->num_chunks;
  rp.rpad = P->rpad;
  rp.slab_base = P->slab_base;
  rp.info = P->info;
  rp.chunk_hist = P->chunk_hist;
  rp.chunk_off = P->chunk_off;
  rp.group_count = P->group_count;
  rp.group_off = P->group_off;
  rp.mtile_off = P->mtile_off;
  rp.scan_ticket = P->scan_ticket;
  rp.tiling = P->tiling;
  rp.tok_mt = P->tok_mt;
  rp.tok_need = P->tok_need;
  rp.pos = P->pos;
  rp.row_token = P->row_token;
  rp.row_mt = P->row_mt;
  rp.zero_y = P->external_acc ? 0 : 1;

  rp.row_k = P->row_k;
  rp.row_w = P->row_w;
  rp.a_perm = P->a_perm;
  rp.sa_t = P->sa_t;
  rp.status = P->status;
}

static void fill_gemm_params(afd_ffn_plan_t P, int epi, GemmParams& gp) {
  const afd_ffn_config_t& c = P->cfg;
  const bool small = P->num_chunks <= kSmallRouteChunks;
  memset(&gp, 0, sizeof(gp));
  gp.info = P->info;
  gp.group_off = P->group_off;
  gp.mtile_off = P->mtile_off;
  gp.G = P->G;
  gp.rpad = P->rpad;
  gp.I = c.intermediate;
  gp.H = c.hidden;
  gp.status = P->status;
  gp.wait_limit_ns = P->wait_limit_ns;
  gp.row_token = P->row_token;
  if (epi == EPI_SWIGLU) {
    gp.n_tiles = c.intermediate / 128;
    gp.num_kb = c.hidden / 128;
    gp.sa_t = P->sa_t;
    gp.w_scale = P->w.w13_scale;
    if (small && c.has_shared_expert) {
      // the shared expert's W13 (every token's), prefetched while the gather runs
      gp.pf_base = static_cast<const uint8_t*>(P->w.w13) + static_cast<size_t>(c.num_local_experts) * 2 * c.intermediate * c.hidden;
      gp.pf_bytes = static_cast<unsigned long long>(2) * c.intermediate * c.hidden;
    }
    gp.ws_rows = 2 * c.intermediate / 128;
    gp.hq = P->hq;
    gp.sh_t = P->sh_t;
    gp.inject_stall = P->inject_stall;
    gp.split_ok = 1;
    gp.g_ws = P->g_ws;
    gp.g_rows = P->g_rows;
    gp.g_cnt = P->g_cnt;
  } else {
    gp.n_tiles = c.hidden / 256;
    gp.num_kb = c.intermediate / 128;
    gp.sa_t = P->sh_t;
    gp.w_scale = P->w.w2_scale;
    if (small && c.has_shared_expert) {
      gp.pf_base = static_cast<const uint8_t*>(P->w.w2) + static_cast<size_t>(c.num_local_experts) * c.hidden * c.intermediate;
      gp.pf_bytes = static_cast<unsigned long long>(c.hidden) * c.intermediate;
    }
    gp.ws_rows = c.hidden / 128;
    gp.row_w = P->row_w;
    gp.row_mt = P->row_mt;
    gp.acc = P->external_acc ? P->ext_acc : P->own_acc;
    gp.slice_first = P->w2_slice_first;
    gp.split_ok = 1;
  }
}

afd_status_t afd_ffn_layer(afd_ffn_plan_t P, const afd_slab_t* slabs, const int32_t* d_counts,
                           afd_stream_t stream_) {
  if (!P || !slabs || !d_counts) return AFD_ERR_INVALID_ARGUMENT;
  {
    // the plan's workspace and tensor maps belong to the device it was built on
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != P->device) return AFD_ERR_INVALID_ARGUMENT;
  }
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const afd_ffn_config_t& c = P->cfg;
  SlabTable tab;
  YTable ytab;
  memset(&tab, 0, sizeof(tab));
  memset(&ytab, 0, sizeof(ytab));
  for (int m = 0; m < c.num_slabs; ++m) {
    const afd_slab_t& s = slabs[m];
    if (!s.x || !s.x_scale || !s.topk_ids || !s.topk_weights || !s.y) return AFD_ERR_INVALID_ARGUMENT;
    if (!aligned(s.x, 16) || !aligned(s.y, 16) || !aligned(s.x_scale, 4) || !aligned(s.topk_ids, 4) ||
        !aligned(s.topk_weights, 4))
      return AFD_ERR_INVALID_ARGUMENT;
    tab.x[m] = static_cast<const uint8_t*>(s.x);
    tab.xs[m] = s.x_scale;
    tab.ids[m] = s.topk_ids;
    tab.w[m] = s.topk_weights;
    tab.y[m] = static_cast<__nv_bfloat16*>(s.y);
    ytab.y[m] = static_cast<__nv_bfloat16*>(s.y);
  }
  const bool mx = P->tiling == 2;
  RouteParams rp;
  fill_route_params(P, d_counts, rp);
  GemmParams g13, g2;
  fill_gemm_params(P, EPI_SWIGLU, g13);
  fill_gemm_params(P, EPI_COMBINE, g2);
  P->inject_stall = 0;

  const bool tm = P->timing;
  if (tm) cudaEventRecord(P->ev[0], stream);
  if (P->num_chunks <= kSmallRouteChunks) {
    // small plans: count, scan and scatter in one block (the scan and scatter stage times
    // read as zero)
    route_small_kernel<<<1, kRouteThreads, P->scatter_smem, stream>>>(rp, tab);
    if (tm) cudaEventRecord(P->ev[1], stream);
    if (tm) cudaEventRecord(P->ev[2], stream);
  } else {
    // the routing scan runs in route_count's last block (its stage time reads as zero)
    route_count_kernel<<<P->num_chunks, kRouteThreads, sizeof(int32_t) * kChunkTokens * c.top_k, stream>>>(rp, tab);
    if (tm) cudaEventRecord(P->ev[1], stream);
    if (tm) cudaEventRecord(P->ev[2], stream);
    route_scatter_kernel<<<P->num_chunks, kRouteThreads, P->scatter_smem, stream>>>(rp, tab);
  }
  if (tm) cudaEventRecord(P->ev[3], stream);
  // one warp per token (gather) and per (token, 256 columns) (finalisation), grids no
  // larger than the plan's capacity needs, so that small plans do not launch idle blocks
  const int warps_per_block = kRouteThreads / 32;
  const int gather_grid = std::max(1, std::min(P->num_sms * 8, (P->Tmax + warps_per_block - 1) / warps_per_block));
  const int64_t fin_items = static_cast<int64_t>(P->Tmax) * (c.hidden / 256);
  const int fin_grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(P->num_sms * 4, (fin_items + warps_per_block - 1) / warps_per_block)));
  // Small plans (one routing chunk) chain the kernels after the routing with programmatic
  // dependent launch: each starts, sets itself up and waits on the device while its
  // predecessor drains, instead of paying a launch gap at every step (at a few tokens the
  // steps are a few microseconds each). Large plans launch in plain stream order: there
  // the early GEMM blocks would hold SMs the gather still needs.
  const bool pdl = P->num_chunks <= kSmallRouteChunks && !tm;
  launch(pdl, gather_rows_kernel, gather_grid, kRouteThreads, 0, stream, rp, tab);
  if (tm) cudaEventRecord(P->ev[4], stream);
  const int grid = P->num_sms;
  if (mx) {
    // factor images of this call's activation rows, then W13 on the block-scale path (the
    // W13 stage time includes the image kernel)
    mx_act_sf_kernel<<<P->num_sms * 4, 128, 0, stream>>>(P->mtile_off, P->group_off, P->G, P->sa_t,
                                                         P->rpad, c.hidden / 128, P->mx_sfa, P->status);
    launch(pdl, w13_mx_kernel, grid, kGemmThreads, mx_smem_bytes(), stream, g13, P->tm_a13, P->tm_w13,
           MxArgs{P->mx_sfa, P->mx_sfb});
  } else {
    launch(pdl, grouped_gemm_kernel<EPI_SWIGLU>, grid, kGemmThreads, gemm_smem_bytes<EPI_SWIGLU>(), stream,
           g13, P->tm_a13, P->tm_w13);
  }
  if (tm) cudaEventRecord(P->ev[5], stream);
  launch(pdl, grouped_gemm_kernel<EPI_COMBINE>, grid, kGemmThreads, gemm_smem_bytes<EPI_COMBINE>(), stream,
         g2, P->tm_a2, P->tm_w2);
  if (tm) cudaEventRecord(P->ev[6], stream);
  if (!P->external_acc)
    launch(pdl, combine_finalize_kernel, fin_grid, 256, 0, stream, static_cast<const int32_t*>(P->info),
           static_cast<const int32_t*>(P->tok_mt), P->own_acc, c.hidden, ytab);
  if (tm) cudaEventRecord(P->ev[7], stream);
  P->ev_valid = tm;
  if (cudaGetLastError() != cudaSuccess) return AFD_ERR_CUDA;
  return AFD_OK;
}

afd_status_t afd_ffn_get_status(afd_ffn_plan_t P, afd_stream_t stream, int32_t* word) {
  if (!P) return AFD_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return AFD_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, P->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return AFD_ERR_CUDA;
  if (cudaMemset(P->status, 0, sizeof(v)) != cudaSuccess) return AFD_ERR_CUDA;
  if (word) *word = v;
  if (v & AFD_STATUS_TIMEOUT) return AFD_ERR_TIMEOUT;
  if (v & (AFD_STATUS_BAD_ROUTING | AFD_STATUS_BAD_COUNT)) return AFD_ERR_BAD_ROUTING;
  if (v & AFD_STATUS_BAD_SCALE) return AFD_ERR_INVALID_ARGUMENT;
  return AFD_OK;
}

static afd_status_t d2h(void* dst, const void* src, size_t bytes) {
  if (!dst || bytes == 0) return AFD_OK;
  return cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost) == cudaSuccess ? AFD_OK : AFD_ERR_CUDA;
}

afd_status_t afd_ffn_read_routing(afd_ffn_plan_t P, afd_stream_t stream, int32_t* num_tokens,
                                  int32_t* num_rows, int32_t* counts, int32_t* offsets,
                                  int32_t* row_token, int32_t* row_k, float* row_weight,
                                  int32_t* pos) {
  if (!P) return AFD_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return AFD_ERR_CUDA;
  int32_t info[4];
  if (cudaMemcpy(info, P->info, sizeof(info), cudaMemcpyDeviceToHost) != cudaSuccess) return AFD_ERR_CUDA;
  const int T = info[0], R = info[1];
  if (num_tokens) *num_tokens = T;
  if (num_rows) *num_rows = R;
  afd_status_t s = AFD_OK;
  if (s == AFD_OK) s = d2h(counts, P->group_count, sizeof(int32_t) * P->G);
  if (s == AFD_OK) s = d2h(offsets, P->group_off, sizeof(int32_t) * (P->G + 1));
  if (s == AFD_OK) s = d2h(row_token, P->row_token, sizeof(int32_t) * R);
  if (s == AFD_OK) s = d2h(row_k, P->row_k, sizeof(int32_t) * R);
  if (s == AFD_OK) s = d2h(row_weight, P->row_w, sizeof(float) * R);
  if (s == AFD_OK) s = d2h(pos, P->pos, sizeof(int32_t) * static_cast<size_t>(T) * P->cfg.top_k);
  return s;
}

afd_status_t afd_ffn_read_intermediate(afd_ffn_plan_t P, afd_stream_t stream, uint8_t* h_codes,
                                       float* h_scales) {
  if (!P) return AFD_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return AFD_ERR_CUDA;
  int32_t info[4];
  if (cudaMemcpy(info, P->info, sizeof(info), cudaMemcpyDeviceToHost) != cudaSuccess) return AFD_ERR_CUDA;
  const int R = info[1];
  const int I = P->cfg.intermediate;
  afd_status_t s = d2h(h_codes, P->hq, static_cast<size_t>(R) * I);
  if (s == AFD_OK && h_scales && R > 0) {
    // stored transposed [I/128][rpad]; return row-major [R][I/128]
    const int nb = I / 128;
    float* tmp = static_cast<float*>(malloc(sizeof(float) * static_cast<size_t>(nb) * R));
    if (!tmp) return AFD_ERR_OUT_OF_MEMORY;
    for (int j = 0; j < nb && s == AFD_OK; ++j)
      s = d2h(tmp + static_cast<size_t>(j) * R, P->sh_t + static_cast<size_t>(j) * P->rpad,
              sizeof(float) * R);
    for (int r = 0; r < R; ++r)
      for (int j = 0; j < nb; ++j) h_scales[static_cast<size_t>(r) * nb + j] = tmp[static_cast<size_t>(j) * R + r];
    free(tmp);
  }
  return s;
}

afd_status_t afd_ffn_set_timing(afd_ffn_plan_t P, int32_t enable) {
  if (!P) return AFD_ERR_INVALID_ARGUMENT;
  P->timing = enable != 0;
  return AFD_OK;
}

afd_status_t afd_ffn_get_kernel_times(afd_ffn_plan_t P, float* ms) {
  if (!P || !ms) return AFD_ERR_INVALID_ARGUMENT;
  if (!P->ev_valid) return AFD_ERR_INVALID_ARGUMENT;
  if (cudaEventSynchronize(P->ev[AFD_NUM_KERNELS]) != cudaSuccess) return AFD_ERR_CUDA;
  for (int i = 0; i < AFD_NUM_KERNELS; ++i)
    if (cudaEventElapsedTime(&ms[i], P->ev[i], P->ev[i + 1]) != cudaSuccess) return AFD_ERR_CUDA;
  return AFD_OK;
}

afd_status_t afd_ffn_set_wait_limit(afd_ffn_plan_t P, int64_t limit_ns) {
  if (!P || limit_ns <= 0) return AFD_ERR_INVALID_ARGUMENT;
  P->wait_limit_ns = static_cast<unsigned long long>(limit_ns);
  return AFD_OK;
}

afd_status_t afd_ffn_set_tiling(afd_ffn_plan_t P, int32_t tiling) {
  if (!P || tiling < 0 || tiling > 2) return AFD_ERR_INVALID_ARGUMENT;
  if (tiling == 2 && !P->mx_sfb) {
    // the W13 factor images, once per plan (the weights are fixed for its lifetime)
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != P->device) return AFD_ERR_INVALID_ARGUMENT;
    const afd_ffn_config_t& c = P->cfg;
    const size_t n_img = static_cast<size_t>(P->G) * (2 * c.intermediate / 128) * (c.hidden / 128);
    if (n_img >= (size_t{1} << 31)) return AFD_ERR_UNSUPPORTED;
    // the images, then one word the check ORs AFD_STATUS_BAD_SCALE into (the plan's
    // status word is left alone: the weights are refused here, once, synchronously)
    uint8_t* img = nullptr;
    const size_t img_bytes = n_img * kSfImage;
    if (cudaMalloc(&img, img_bytes + 16) != cudaSuccess) {
      cudaGetLastError();
      return AFD_ERR_OUT_OF_MEMORY;
    }
    int* flag = reinterpret_cast<int*>(img + img_bytes);
    int bad = 0;
    if (cudaMemset(flag, 0, sizeof(int)) != cudaSuccess) {
      cudaFree(img);
      return AFD_ERR_CUDA;
    }
    mx_weight_sf_kernel<<<P->num_sms * 4, 256>>>(P->w.w13_scale, static_cast<int>(n_img), img, flag);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&bad, flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
      cudaFree(img);
      return AFD_ERR_CUDA;
    }
    if (bad & AFD_STATUS_BAD_SCALE) {
      cudaFree(img);
      return AFD_ERR_INVALID_ARGUMENT;
    }
    P->mx_sfb = img;
  }
  P->tiling = tiling;
  return AFD_OK;
}

afd_status_t afd_ffn_get_tiling(afd_ffn_plan_t P, afd_stream_t stream, int32_t* tiling) {
  if (!P || !tiling) return AFD_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return AFD_ERR_CUDA;
  if (cudaMemcpy(tiling, P->info + 3, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return AFD_ERR_CUDA;
  return AFD_OK;
}

afd_status_t afd_ffn_inject_stall(afd_ffn_plan_t P, int32_t enable) {
  if (!P) return AFD_ERR_INVALID_ARGUMENT;
  P->inject_stall = enable != 0;
  return AFD_OK;
}

afd_status_t afd_ffn_set_combine_targets(afd_ffn_plan_t P, float* const* acc_per_slab) {
  if (!P) return AFD_ERR_INVALID_ARGUMENT;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != P->device) return AFD_ERR_INVALID_ARGUMENT;
  if (!acc_per_slab) {
    P->external_acc = false;
    return AFD_OK;
  }
  AccTable t;
  memset(&t, 0, sizeof(t));
  for (int m = 0; m < P->cfg.num_slabs; ++m) {
    if (!acc_per_slab[m] || !aligned(acc_per_slab[m], 16)) return AFD_ERR_INVALID_ARGUMENT;
    t.a[m] = acc_per_slab[m];
  }
  P->ext_acc = t;
  P->external_acc = true;
  return AFD_OK;
}

afd_status_t afd_combine_finalize(const afd_slab_t* slabs, int32_t num_slabs, int32_t slab_capacity,
                                  int32_t hidden, const int32_t* d_counts, float* const* acc_per_slab,
                                  afd_stream_t stream_) {
  if (!slabs || !d_counts || !acc_per_slab) return AFD_ERR_INVALID_ARGUMENT;
  if (num_slabs < 1 || num_slabs > AFD_MAX_SLABS || slab_capacity < 1 || slab_capacity > (1 << 24) - 1 ||
      hidden < 256 || hidden % 256)
    return AFD_ERR_INVALID_ARGUMENT;
  AccTable acc;
  YTable ytab;
  memset(&acc, 0, sizeof(acc));
  memset(&ytab, 0, sizeof(ytab));
  for (int m = 0; m < num_slabs; ++m) {
    if (!slabs[m].y || !aligned(slabs[m].y, 16) || !acc_per_slab[m] || !aligned(acc_per_slab[m], 16))
      return AFD_ERR_INVALID_ARGUMENT;
    acc.a[m] = acc_per_slab[m];
    ytab.y[m] = static_cast<__nv_bfloat16*>(slabs[m].y);
  }
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // one warp per (token, 256 columns): enough blocks per slab to cover its capacity,
  // at most a few waves of the GPU over all slabs
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return AFD_ERR_CUDA;
  const int64_t items = static_cast<int64_t>(slab_capacity) * (hidden / 256);
  const int per_slab = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>((sms * 4 + num_slabs - 1) / num_slabs, (items + 7) / 8)));
  combine_finalize_slabs_kernel<<<dim3(per_slab, num_slabs), 256, 0, stream>>>(d_counts, slab_capacity, hidden,
                                                                               acc, ytab);
  if (cudaGetLastError() != cudaSuccess) return AFD_ERR_CUDA;
  return AFD_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Routing without allocation: the routing kernels run with their scratch in one
// file-scope device array instead of a plan workspace.
// ------------------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[AFD_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
uint8_t* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;   // guards g_noalloc_ptr and the set-up calls

// Once per device, with that device current: the array's device address (the host-side
// name of a __device__ array is only a stand-in) and the routing scatter's shared-memory
// limit. Host threads making their first call at the same time are serialised here; a
// failed set-up is retried by the next call.
afd_status_t noalloc_setup(int dev, uint8_t** out) {
  if (dev < 0 || dev >= kMaxDevices) return AFD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return AFD_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(route_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(scatter_smem_bytes(AFD_MAX_GROUPS, AFD_MAX_TOP_K))) !=
        cudaSuccess) {
      cudaGetLastError();
      return AFD_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return AFD_OK;
}

}  // namespace

extern "C" afd_status_t afd_ffn_route_noalloc(const afd_ffn_config_t* cfg, const afd_slab_t* slabs,
                                              const int32_t* d_counts, int32_t* d_sizes,
                                              int32_t* d_group_count, int32_t* d_group_offset,
                                              int32_t* d_row_token, int32_t* d_row_k,
                                              float* d_row_weight, int32_t* d_pos, int32_t* d_status,
                                              afd_stream_t stream_) {
  afd_status_t st = afd_ffn_check_config(cfg);
  if (st != AFD_OK) return st;
  if (!slabs || !d_counts || !d_sizes || !d_group_count || !d_group_offset || !d_row_token ||
      !d_row_k || !d_row_weight || !d_pos || !d_status)
    return AFD_ERR_INVALID_ARGUMENT;
  const afd_ffn_config_t& c = *cfg;
  SlabTable tab;
  memset(&tab, 0, sizeof(tab));
  for (int m = 0; m < c.num_slabs; ++m) {
    const afd_slab_t& s = slabs[m];
    if (!s.topk_ids || !s.topk_weights || !s.y) return AFD_ERR_INVALID_ARGUMENT;
    if (!aligned(s.y, 16) || !aligned(s.topk_ids, 4) || !aligned(s.topk_weights, 4))
      return AFD_ERR_INVALID_ARGUMENT;
    tab.ids[m] = s.topk_ids;
    tab.w[m] = s.topk_weights;
    tab.y[m] = static_cast<__nv_bfloat16*>(s.y);
  }
  // scratch layout (bytes), each region 256-byte aligned
  const int G = c.num_local_experts + c.has_shared_expert;
  const int El1 = std::max(c.num_local_experts, 1);
  const int64_t tmax = static_cast<int64_t>(c.num_slabs) * c.slab_capacity;
  const int64_t chunks = (tmax + kChunkTokens - 1) / kChunkTokens;
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    const int64_t o = off;
    off = (off + bytes + 255) / 256 * 256;
    return o;
  };
  const int64_t o_base = take(4 * (c.num_slabs + 1));
  const int64_t o_hist = take(4 * chunks * El1);
  const int64_t o_coff = take(4 * chunks * El1);
  const int64_t o_mtile = take(4 * (G + 1));
  const int64_t o_tmt = take(4 * tmax);
  const int64_t o_tneed = take(4 * tmax);
  if (off > static_cast<int64_t>(AFD_NOALLOC_SCRATCH_BYTES)) return AFD_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AFD_ERR_UNSUPPORTED;
  uint8_t* scratch = nullptr;
  st = noalloc_setup(dev, &scratch);
  if (st != AFD_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

  RouteParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.counts = d_counts;
  rp.M = c.num_slabs;
  rp.cap = c.slab_capacity;
  rp.K = c.top_k;
  rp.H = c.hidden;
  rp.e0 = c.expert_begin;
  rp.El = c.num_local_experts;
  rp.Eg = c.num_experts_global;
  rp.S = c.has_shared_expert;
  rp.G = G;
  rp.num_chunks = static_cast<int>(chunks);
  rp.slab_base = reinterpret_cast<int32_t*>(scratch + o_base);
  rp.info = d_sizes;
  rp.chunk_hist = reinterpret_cast<int32_t*>(scratch + o_hist);
  rp.chunk_off = reinterpret_cast<int32_t*>(scratch + o_coff);
  rp.group_count = d_group_count;
  rp.group_off = d_group_offset;
  rp.mtile_off = reinterpret_cast<int32_t*>(scratch + o_mtile);
  rp.tok_mt = reinterpret_cast<int32_t*>(scratch + o_tmt);
  rp.tok_need = reinterpret_cast<int32_t*>(scratch + o_tneed);
  rp.pos = d_pos;
  rp.row_token = d_row_token;
  rp.row_k = d_row_k;
  rp.row_w = d_row_weight;
  rp.status = d_status;
  rp.tiling = -1;           // routing only: d_sizes[3] = 0
  rp.zero_y = 1;
  // every scratch region is fully written before it is read; only the status starts at 0
  if (cudaMemsetAsync(d_status, 0, sizeof(int32_t), stream) != cudaSuccess) return AFD_ERR_CUDA;
  const size_t scatter_smem = scatter_smem_bytes(El1, c.top_k);
  route_count_kernel<<<static_cast<int>(chunks), kRouteThreads, sizeof(int32_t) * kChunkTokens * c.top_k, stream>>>(rp, tab);
  route_scan_kernel<<<1, 1024, 0, stream>>>(rp);
  route_scatter_kernel<<<static_cast<int>(chunks), kRouteThreads, scatter_smem, stream>>>(rp, tab);
  if (cudaGetLastError() != cudaSuccess) return AFD_ERR_CUDA;
  return AFD_OK;
}
