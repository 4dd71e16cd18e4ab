/*
 * afd_ffn.h -- C ABI of the FFN-pool expert layer of attention-FFN disaggregation (AFD).
 *
 * What the layer computes (FastAFD, "Methodology / System Design", items 1-3; vLLM AFD
 * plugin, "FFN service"): M attention ranks have published block-FP8 token activations
 * and their top-K routing (expert ids and combine weights) into M receive buffers
 * ("slabs") on this GPU. For every token the layer evaluates each routed expert that
 * this GPU holds, plus an optional shared expert, as
 *
 *     G = x . W13^T (block-FP8),  h = silu(G[:I]) * G[I:],  h -> e4m3 per (row, 128),
 *     Y = h . W2^T  (block-FP8),
 *
 * and writes  y = sum_k w_k * Y_k  (+ Y_shared)  as bf16 into the token's row of its slab.
 * Routing ids outside [expert_begin, expert_begin + num_local_experts) belong to other
 * FFN GPUs and are skipped, so y is this GPU's partial sum.
 *
 * Data formats (all device memory, row-major, caller-owned):
 *   e4m3      OCP FP8 E4M3 "fn" codes, one byte per element.
 *   W13       e4m3 [E][2I][H]: rows 0..I-1 are the gate projection, rows I..2I-1 the up
 *             projection. Scale fp32 [E][2I/128][H/128], one per 128x128 block.
 *   W2        e4m3 [E][H][I]. Scale fp32 [E][H/128][I/128].
 *             E = num_local_experts + has_shared_expert; the shared expert is index
 *             num_local_experts. Routing id i maps to weight index i - expert_begin.
 *   slab m    x e4m3 [cap][H], x_scale fp32 [cap][H/128] (one scale per token per 128
 *             channels), topk_ids int32 [cap][K] (global expert ids, -1 = empty slot),
 *             topk_weights fp32 [cap][K], y bf16 [cap][H] (output; rows < n_m written).
 *   counts    device int32 [M]: n_m, the number of valid rows of slab m (0 <= n_m <= cap).
 *
 * Routing rules: slot k of token t is used iff its id is in [0, E_g), not equal to an id
 * in an earlier slot of the same token, and local. An id that is neither -1 nor in
 * [0, E_g), or a repeated id, is skipped and sets AFD_STATUS_BAD_ROUTING in the plan's
 * device status word. Routed rows are grouped by expert in ascending (token, slot) order
 * with tokens numbered slab-major; this order is deterministic.
 *
 * Errors: functions return afd_status_t. Argument errors return before anything is
 * enqueued. Conditions detected on the device (bad routing ids, slab counts above the
 * capacity, a bounded wait that expired) are OR-ed into the plan's status word, read
 * with afd_ffn_get_status(); the kernels never trap.
 *
 * Threading: a plan is not thread-safe; calls on one plan must be serialised by the
 * caller, and layer calls on one plan must be ordered on the GPU (one stream, or
 * explicit events) because they share the plan's workspace.
 */
#ifndef AFD_FFN_H_
#define AFD_FFN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AFD_API __attribute__((visibility("default")))
#else
#define AFD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AFD_OK = 0,
  AFD_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size or shape; nothing was enqueued */
  AFD_ERR_UNSUPPORTED = 2,      /* no sm_100 device, or a shape outside the supported limits */
  AFD_ERR_OUT_OF_MEMORY = 3,    /* workspace allocation failed */
  AFD_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
  AFD_ERR_BAD_ROUTING = 5,      /* returned by afd_ffn_get_status when the device saw bad ids */
  AFD_ERR_TIMEOUT = 6           /* returned by afd_ffn_get_status when a device wait expired */
} afd_status_t;

/* Bits of the device status word. */
#define AFD_STATUS_BAD_ROUTING 0x1 /* id outside [0, E_g) and != -1, or repeated in a token */
#define AFD_STATUS_TIMEOUT 0x2     /* a bounded device wait expired; outputs are invalid */
#define AFD_STATUS_BAD_COUNT 0x4   /* some counts[m] < 0 or > slab_capacity; clamped */
#define AFD_STATUS_BAD_SCALE 0x8   /* tiling 2: an activation block scale of this call is not a
                                      positive normal power of two; outputs are invalid */

/* Limits. */
#define AFD_MAX_SLABS 128
#define AFD_MAX_TOP_K 32
#define AFD_MAX_GROUPS 1024 /* num_local_experts + has_shared_expert */
#define AFD_QBLOCK 128      /* quantisation block edge */
#define AFD_MAX_QBLOCKS 128 /* hidden and intermediate are at most 128 blocks (16384) */

/* Timed stages of one layer call, in launch order (for afd_ffn_get_kernel_times). One
 * kernel per stage, except that the routing scan runs in the last block of the route
 * count kernel (AFD_KERNEL_ROUTE_COUNT covers both and AFD_KERNEL_ROUTE_SCAN reads as
 * zero), and that a plan of at most 256 tokens (num_slabs * slab_capacity) routes in one
 * block (AFD_KERNEL_ROUTE_COUNT covers count, scan and scatter). The gather stage copies the routed FP8 rows and their scales into expert order. */
#define AFD_KERNEL_ROUTE_COUNT 0
#define AFD_KERNEL_ROUTE_SCAN 1
#define AFD_KERNEL_ROUTE_SCATTER 2
#define AFD_KERNEL_GATHER 3
#define AFD_KERNEL_GEMM13 4
#define AFD_KERNEL_GEMM2 5
#define AFD_KERNEL_FINALIZE 6
#define AFD_NUM_KERNELS 7

struct CUstream_st;
typedef struct CUstream_st* afd_stream_t; /* same type as cudaStream_t; NULL = legacy stream */

typedef struct afd_ffn_plan_s* afd_ffn_plan_t; /* opaque; owned by the library */

typedef struct {
  int32_t hidden;             /* H, multiple of 128; AFD_ERR_UNSUPPORTED unless a multiple
                                 of 256 (the down projection writes 256-column tiles) and
                                 at most 128 * AFD_MAX_QBLOCKS */
  int32_t intermediate;       /* I, multiple of 128; AFD_ERR_UNSUPPORTED above
                                 128 * AFD_MAX_QBLOCKS */
  int32_t num_experts_global; /* E_g >= 1: ids the router may emit are [0, E_g) */
  int32_t expert_begin;       /* e0 >= 0 */
  int32_t num_local_experts;  /* E_l >= 0, e0 + E_l <= E_g */
  int32_t has_shared_expert;  /* S in {0, 1}; E_l + S >= 1 */
  int32_t top_k;              /* K in [1, min(E_g, AFD_MAX_TOP_K)] */
  int32_t num_slabs;          /* M in [1, AFD_MAX_SLABS] */
  int32_t slab_capacity;      /* cap >= 1: rows allocated per slab */
} afd_ffn_config_t;

typedef struct {
  const void* w13;        /* e4m3 [E][2I][H], 16-byte aligned */
  const float* w13_scale; /* fp32 [E][2I/128][H/128] */
  const void* w2;         /* e4m3 [E][H][I], 16-byte aligned */
  const float* w2_scale;  /* fp32 [E][H/128][I/128] */
} afd_ffn_weights_t;

typedef struct {
  const void* x;              /* e4m3 [cap][H], 16-byte aligned */
  const float* x_scale;       /* fp32 [cap][H/128] */
  const int32_t* topk_ids;    /* int32 [cap][K] */
  const float* topk_weights;  /* fp32 [cap][K] */
  void* y;                    /* bf16 [cap][H], 16-byte aligned; rows < n_m are written */
} afd_slab_t;

/* Host-visible sizes of a plan (for sizing inspection buffers). */
typedef struct {
  int32_t num_groups;     /* G = E_l + S */
  int32_t max_tokens;     /* M * cap */
  int32_t max_rows;       /* M * cap * (min(K, E_l) + S): routed rows the workspace holds */
  int32_t num_sms;        /* grid of the persistent GEMM kernels */
  int64_t workspace_bytes;
} afd_ffn_plan_info_t;

/*
 * Validate a configuration without touching the GPU. AFD_OK or
 * AFD_ERR_INVALID_ARGUMENT (cfg NULL or a field out of range) or AFD_ERR_UNSUPPORTED
 * (a limit above is exceeded).
 */
AFD_API afd_status_t afd_ffn_check_config(const afd_ffn_config_t* cfg);

/*
 * Build a plan for one layer on the current CUDA device. The FFN GPUs hold expert weights
 * in block-FP8 and keep pre-allocated receive buffers for the tokens the attention GPUs
 * publish (FastAFD, "Methodology / System Design", items 1-2); the plan is the FFN side's
 * per-layer state: validates cfg and weights,
 * checks for an sm_100 device, allocates the workspace (cudaMalloc; freed by
 * afd_ffn_destroy), zeroes the combine accumulators and encodes the TMA descriptors of
 * the weights. The weights are read by every later layer call and must stay valid and
 * unchanged until afd_ffn_destroy. Synchronous. On error *out is set to NULL.
 */
AFD_API afd_status_t afd_ffn_plan(const afd_ffn_config_t* cfg, const afd_ffn_weights_t* weights,
                          afd_ffn_plan_t* out);

/*
 * Enqueue one layer evaluation on `stream`; never synchronises with the host. This is the
 * FFN service's compute step between receiving the activations with their routing and
 * returning the output (vLLM AFD plugin, "FFN service"), run as the FFN GPU's per-layer
 * work of pull, block-FP8 grouped GEMMs, activation and push-back (FastAFD, "Methodology /
 * System Design", item 3): routed rows are grouped by expert, W13 + SwiGLU and W2 run as
 * grouped GEMMs, and each token's top-K-weighted sum is written as bf16 into its slab row.
 * slabs: host array of num_slabs descriptors (read during the call only; the device
 * buffers they point to must stay valid until the stream reaches the work).
 * d_counts: device int32 [num_slabs]. Returns AFD_ERR_INVALID_ARGUMENT for NULL
 * arguments, misaligned slab pointers or a current CUDA device other than the plan's
 * (nothing enqueued) and AFD_ERR_CUDA if a launch fails.
 */
AFD_API afd_status_t afd_ffn_layer(afd_ffn_plan_t plan, const afd_slab_t* slabs, const int32_t* d_counts,
                           afd_stream_t stream);

/* Free the plan and its workspace (the FFN side's per-layer state built by afd_ffn_plan;
 * FastAFD, "Methodology / System Design", item 2: the receive buffers are pre-allocated and
 * live as long as the serving instance). NULL is a no-op. Synchronises the device. */
AFD_API void afd_ffn_destroy(afd_ffn_plan_t plan);

/* Sizes of a plan. */
AFD_API afd_status_t afd_ffn_get_info(afd_ffn_plan_t plan, afd_ffn_plan_info_t* info);

/*
 * Synchronise `stream`, read the device status word into *status_word (may be NULL),
 * and clear it. Returns AFD_ERR_TIMEOUT if the TIMEOUT bit was set, else
 * AFD_ERR_BAD_ROUTING if BAD_ROUTING or BAD_COUNT was set, else AFD_ERR_INVALID_ARGUMENT
 * if BAD_SCALE was set, else AFD_OK.
 */
AFD_API afd_status_t afd_ffn_get_status(afd_ffn_plan_t plan, afd_stream_t stream, int32_t* status_word);

/*
 * Copy the routing of the last layer call to HOST buffers after synchronising `stream`.
 * Any pointer may be NULL to skip that array. Sizes: counts [G], offsets [G+1],
 * row_token / row_k / row_weight [max_rows] (first num_rows valid), pos [max_tokens*K]
 * (first num_tokens*K valid). row_k is -1 for shared-expert rows; pos is -1 for slots
 * that are not local.
 */
AFD_API afd_status_t afd_ffn_read_routing(afd_ffn_plan_t plan, afd_stream_t stream, int32_t* num_tokens,
                                  int32_t* num_rows, int32_t* counts, int32_t* offsets,
                                  int32_t* row_token, int32_t* row_k, float* row_weight,
                                  int32_t* pos);

/*
 * Copy the intermediate of the last layer call to HOST buffers after synchronising
 * `stream`: h_codes e4m3 [max_rows][I] and h_scales fp32 [max_rows][I/128]
 * (first num_rows rows valid). Either pointer may be NULL.
 */
AFD_API afd_status_t afd_ffn_read_intermediate(afd_ffn_plan_t plan, afd_stream_t stream,
                                       uint8_t* h_codes, float* h_scales);

/*
 * Per-kernel timing. When enabled, layer calls record CUDA events around each kernel
 * on the launch stream. afd_ffn_get_kernel_times waits for the last call's events and
 * writes AFD_NUM_KERNELS durations in milliseconds (index = AFD_KERNEL_*).
 */
AFD_API afd_status_t afd_ffn_set_timing(afd_ffn_plan_t plan, int32_t enable);
AFD_API afd_status_t afd_ffn_get_kernel_times(afd_ffn_plan_t plan, float* ms);

/*
 * Tiling of the two grouped GEMMs, chosen on the host for the following calls.
 * 0 (default) or 1: one CTA per 128-row x 256-column tile; every 128-wide K block is a
 *    separate tensor-core partial product that the epilogue scales by (activation block
 *    scale x weight block scale) and accumulates in fp32 registers, so any positive fp32
 *    block scales are exact.
 * 2: as 1, but W13 runs on the tensor core's block-scale path (kind::mxf8f6f4 with UE8M0
 *    factors): TMEM accumulates a tile's whole K loop and the epilogue runs once per
 *    tile. Only for inputs whose activation and W13 block scales are all positive normal
 *    powers of two (each is then exactly its UE8M0 factor). The first selection on a plan
 *    allocates the W13 factor images (E * 2I/128 * H/128 * 512 bytes), builds them with
 *    one kernel launch and a device synchronisation, and checks every W13 scale: if one is
 *    not a positive normal power of two it frees the images, keeps the previous tiling and
 *    returns AFD_ERR_INVALID_ARGUMENT (AFD_ERR_OUT_OF_MEMORY / AFD_ERR_CUDA on failure; call
 *    it on the plan's device). Each layer call then adds one launch (the activation factor
 *    images), which checks that call's activation scales: any other scale sets
 *    AFD_STATUS_BAD_SCALE, on every such call, and afd_ffn_get_status then returns
 *    AFD_ERR_INVALID_ARGUMENT.
 * Results are the same within rounding. Returns AFD_ERR_INVALID_ARGUMENT outside 0..2.
 */
#define AFD_TILING_DEFAULT 1
#define AFD_TILING_BLOCK_SCALE 2
AFD_API afd_status_t afd_ffn_set_tiling(afd_ffn_plan_t plan, int32_t tiling);

/* Synchronise `stream` and report the tiling (1 or 2) the last layer call used. */
AFD_API afd_status_t afd_ffn_get_tiling(afd_ffn_plan_t plan, afd_stream_t stream, int32_t* tiling);

/*
 * Limit, in nanoseconds, of every bounded device wait (default 1e9). Used by tests to
 * make an injected stall expire quickly.
 */
AFD_API afd_status_t afd_ffn_set_wait_limit(afd_ffn_plan_t plan, int64_t limit_ns);

/*
 * Test hook: when `enable` is non-zero, the next layer call's W13 producer skips one
 * stage so that the consumer's bounded wait expires and sets AFD_STATUS_TIMEOUT.
 * The layer's outputs are then invalid. Host-side fault injection only; it does not
 * fault the GPU.
 */
AFD_API afd_status_t afd_ffn_inject_stall(afd_ffn_plan_t plan, int32_t enable);

/*
 * Routing without any allocation, for callers that cannot call cudaMalloc.
 *
 * The pages have no counterpart for this entry point; it exists for integrations where
 * allocating at call time is not possible: a serving engine that has already reserved
 * nearly all of HBM for its KV-cache pool, a step loop that must not stall on a
 * synchronous allocation, or code running inside another library's callback where
 * allocation is forbidden. It runs the routing stage of afd_ffn_layer (slab intake,
 * histogram, scan, stable permutation) and writes the same routing arrays to caller
 * buffers. Its scratch lives in one file-scope device array of AFD_NOALLOC_SCRATCH_BYTES
 * bytes that every GPU which loads the library holds until the process exits.
 *
 * cfg, slabs (host array [num_slabs]) and d_counts: as for afd_ffn_plan/afd_ffn_layer
 * (only topk_ids, topk_weights and y of each slab are used; y rows of tokens that receive
 * no contribution are set to zero, as afd_ffn_layer does). Outputs, all caller-owned
 * device memory: d_sizes int32[4] = {T, R, m-tiles, 0} (T tokens, R routed rows, the
 * number of 128-row GEMM tiles over all groups, and 0); d_group_count int32[G];
 * d_group_offset int32[G+1]; d_row_token, d_row_k int32[max_rows] and d_row_weight
 * fp32[max_rows] (max_rows = M*cap*(min(K,E_l)+S)); d_pos int32[M*cap*K];
 * d_status int32[1] (cleared, then OR-ed with AFD_STATUS_* bits).
 *
 * Returns AFD_ERR_INVALID_ARGUMENT for bad arguments, AFD_ERR_UNSUPPORTED when the
 * configuration needs more scratch than AFD_NOALLOC_SCRATCH_BYTES, AFD_ERR_CUDA if a
 * set-up call or launch fails. The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture. Every call shares the array and it keeps the last call's contents,
 * so calls whose work overlaps on the GPU (different streams, or several host threads)
 * race: order them. No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define AFD_NOALLOC_SCRATCH_BYTES (2u << 20)
AFD_API afd_status_t afd_ffn_route_noalloc(const afd_ffn_config_t* cfg, const afd_slab_t* slabs,
                                           const int32_t* d_counts, int32_t* d_sizes,
                                           int32_t* d_group_count, int32_t* d_group_offset,
                                           int32_t* d_row_token, int32_t* d_row_k,
                                           float* d_row_weight, int32_t* d_pos, int32_t* d_status,
                                           afd_stream_t stream);

/*
 * Expert-parallel return path. With the experts sharded over several FFN GPUs, each one
 * computes a partial output for every token it received, and a token's result is the sum
 * of the partials of all FFN GPUs, pushed back to the attention rank that owns the token
 * (FastAFD, "Methodology / System Design", item 3, push-back M2N; items 2-3 for the
 * receive buffers that the attention ranks write into).
 *
 * afd_ffn_set_combine_targets: from the next afd_ffn_layer call on, the down projection
 * of this plan adds each token's weighted expert rows (fp32, one reduction per element)
 * into acc_per_slab[m] + t * hidden for token t of received slab m, instead of into the
 * plan's own accumulators, and the layer call stops there: no finalisation launch, and
 * no slab y row is written. acc_per_slab: HOST array of num_slabs device pointers to fp32
 * [slab_capacity][hidden] buffers, 16-byte aligned; they may be other GPUs' memory mapped
 * into this device's address space (peer pointers), and several plans, on this or other
 * GPUs, may add into the same buffers at the same time. The buffers must hold zeros where
 * rows will be added before the first such call (afd_combine_finalize leaves them zero).
 * NULL restores the plan's own accumulators and the bf16 slab outputs. The plan keeps a
 * copy of the table and passes it with every down-projection launch (nothing is written
 * to the device; the host array may be freed after the call). AFD_ERR_INVALID_ARGUMENT
 * for a NULL plan, a NULL or misaligned entry, or a current device other than the plan's.
 *
 * afd_combine_finalize: on the GPU of the owning attention rank, once every FFN GPU's
 * additions have completed: for each of num_slabs slabs and t < counts[m], writes
 * y[m][t] = bf16(acc_per_slab[m][t]) (round to nearest even) and clears that accumulator
 * row. slabs: host array (only y is used); d_counts: device int32 [num_slabs], clamped
 * to [0, slab_capacity] on the device; acc_per_slab: host array of device pointers as
 * above. Enqueued on `stream`, never synchronises. AFD_ERR_INVALID_ARGUMENT for NULL or
 * misaligned pointers or sizes out of range (num_slabs 1..AFD_MAX_SLABS, hidden a positive
 * multiple of 256), AFD_ERR_CUDA if the launch fails.
 */
AFD_API afd_status_t afd_ffn_set_combine_targets(afd_ffn_plan_t plan, float* const* acc_per_slab);
AFD_API afd_status_t afd_combine_finalize(const afd_slab_t* slabs, int32_t num_slabs, int32_t slab_capacity,
                                          int32_t hidden, const int32_t* d_counts,
                                          float* const* acc_per_slab, afd_stream_t stream);

/* Number of this library's kernel launches one afd_ffn_layer call of this plan makes with
 * its current tiling: 6, or 5 when num_slabs * slab_capacity <= 256 (the routing runs in
 * one block), one more with tiling 2, one fewer with combine targets set (no
 * finalisation). -1 for NULL. */
AFD_API int32_t afd_ffn_kernels_per_layer(afd_ffn_plan_t plan);

/* Human-readable name of a status code. */
AFD_API const char* afd_status_string(afd_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* AFD_FFN_H_ */
