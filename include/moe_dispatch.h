/*
 * moe_dispatch.h -- C ABI of the single-GPU MoE token dispatch / combine
 * library for NVIDIA B200 (sm_100a).
 *
 * The operations and where they are defined:
 *   [ASC]   Huawei torch_npu "npu_moe_distribute_combine" API reference:
 *           function description (combine = the dispatch path walked back,
 *           expert outputs multiplied by their weights and summed, plus the
 *           shared expert) and the parameters expert_ids, expand_x,
 *           expand_idx, ep_send_counts, expert_scales, shared_expert_x,
 *           moe_expert_num, H, BS, K.
 *   [DEP]   DeepEP pull request "Intra-node compute compensation + overlap
 *           robustness (CUDA719 fix)", section "Kernel / host": the fused
 *           unzip that scatters token rows and the mapping table into expert
 *           buffers, its chunk-completion counter updated with
 *           atom.acq_rel.gpu, one acquire per chunk on the consumer side, and
 *           bounds guards on every write.
 *   [TEMPO] TEMPO summary (makespan-aware expert load balancing), section 1:
 *           grouped GEMMs round each expert's tokens up to 128-token M-tiles.
 *
 * Notation: T tokens, H hidden size, E routed experts, K experts per token,
 * R logical expert-parallel ranks (expert e belongs to rank e / (E/R)),
 * c_e = number of (t, k) slots routed to expert e, offsets are exclusive
 * prefix sums of 128 * ceil(c_e / 128), P = offsets[E] <= P_cap.
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer; the library allocates no memory and keeps no state besides
 *     cached per-device launch settings (and the fixed scratch array of
 *     moe_dispatch_layout_static, part of the loaded library image).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued on it; no call synchronises the host.
 *   - bf16 = IEEE bfloat16 (2 bytes), E4M3 = OCP 8-bit float E4M3 (1 byte).
 *   - Row-major layouts; "[A, B]" = A rows of B elements.
 *   - Empty batch (T = 0): the layout writes zero counts and offsets; every
 *     other call returns MOE_OK without a launch.  Buffers that have no rows
 *     in that case (x, xp, xp_scales, grad_y, out, ...) may be NULL.
 *   - Return value: MOE_OK if the work was enqueued.  Argument errors that
 *     the host can see (NULL where not allowed, sizes out of range, bad
 *     alignment, E % R != 0, capacity too small) return at once and launch
 *     nothing.  MOE_ERR_CUDA if a launch failed.
 *   - `d_status`: device int32, set to 0 by the caller before a sequence of
 *     calls.  Errors that depend on data (an expert id out of range, a
 *     repeated id, a row index outside the buffers, a timed-out wait) are
 *     written there with first-writer-wins semantics; the kernel then skips
 *     the offending writes instead of trapping.  Read it after the stream
 *     has been synchronised.  Outputs are unspecified (but every write stays
 *     inside the buffers) when it is non-zero.
 *   - After MOE_ERR_TIMEOUT (a device-side wait gave up after its bound) the
 *     call's outputs are undefined, and so is the device state it leaves:
 *     a kernel that gave up waits, again bounded, for the copies it issued
 *     and then exits, and a bulk load that has still not landed by then may
 *     complete later into shared memory that a later CTA on that SM owns.
 *     A timeout means the GPU stalled for seconds; the caller should
 *     synchronise the device, treat every output of the calls since the
 *     status was last clear as garbage, and re-run them (or restart the
 *     process, if the stall recurs).
 */
#ifndef MOE_DISPATCH_H_
#define MOE_DISPATCH_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_TILE_M 128 /* rows per M-tile ([TEMPO] section 1) */
#define MOE_MAX_EXPERTS 512 /* [ASC] moe_expert_num in [1, 512] */
#define MOE_MAX_TOPK 16     /* [ASC] K <= 16 */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,      /* host-side argument check failed */
  MOE_ERR_EXPERT_RANGE = 2,     /* an expert id outside [0, E) */
  MOE_ERR_DUPLICATE_EXPERT = 3, /* an expert id repeated within a token's row */
  MOE_ERR_CAPACITY = 4,         /* P_cap below moe_padded_capacity(T, K, E) */
  MOE_ERR_TIMEOUT = 5,          /* a bounded device-side wait gave up */
  MOE_ERR_CUDA = 6,             /* a CUDA launch or attribute call failed */
  MOE_ERR_UNSUPPORTED = 7,      /* dtype or device not supported */
  MOE_ERR_BOUNDS = 8            /* a row index pointed outside its buffer */
} moe_status_t;

typedef enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_E4M3 = 1 } moe_dtype_t;

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(int status);

/* Library ABI version (major * 100 + minor). */
MOE_API int moe_version(void);

/*
 * Upper bound on the padded row count P for T tokens, K slots per token and
 * E experts, rounded up to a multiple of 128:  T*K + 127*min(E, T*K).
 * Every expert-major buffer (xp, y, grad_y) needs at least this many rows.
 * Returns -1 if an argument is out of range.
 */
MOE_API int64_t moe_padded_capacity(int64_t T, int K, int E);

/* Bytes of device scratch that moe_dispatch_layout needs (256-byte aligned
 * start).  0 is never returned for valid sizes; -1 cast to size_t on bad
 * arguments. */
MOE_API size_t moe_layout_workspace_bytes(int64_t T, int K, int E);

/*
 * Dispatch layout.  [ASC] expert_ids (validation), expand_idx and
 * ep_send_counts (counts in prefix-sum form); [TEMPO] 128-row padding;
 * [DEP] the mapping table written by the fused unzip.
 *
 * In:
 *   topk_idx      int32 [T, K], contiguous; ids in [0, E), distinct per row.
 *   T >= 0, 1 <= K <= 16, 1 <= E <= 512, 1 <= R <= E with E % R == 0,
 *   T*K <= 2^31 - 1, P_cap >= moe_padded_capacity(T, K, E), P_cap < 2^31.
 * Out:
 *   expert_counts  int32 [E]     c_e
 *   expert_offsets int32 [E+1]   exclusive prefix sum of 128*ceil(c_e/128);
 *                                expert_offsets[E] = P
 *   rank_counts    int32 [R]     sum of c_e over the experts of rank r
 *   rank_offsets   int32 [R+1]   expert_offsets[r*E/R]; rank_offsets[R] = P
 *   dst_row        int32 [T*K]   row of slot (t,k) in the expert-major
 *                                buffer: expert_offsets[e] + number of
 *                                earlier tokens routed to e (stable, token
 *                                order); -1 for an out-of-range id
 *   row_src        int32 [P_cap] (nullable) slot t*K+k stored in each row,
 *                                -1 for padding rows and rows >= P
 *   tile_ready     uint32 [ceil(P_cap/128)] (nullable) chunk-completion
 *                                counters, all set to 0 here
 * Scratch: workspace of workspace_bytes >= moe_layout_workspace_bytes(),
 *   256-byte aligned; its contents need no initialisation.  Integer arrays
 *   must be 4-byte aligned (else MOE_ERR_INVALID_ARG).
 * Data errors: MOE_ERR_EXPERT_RANGE (that slot is not placed),
 *   MOE_ERR_DUPLICATE_EXPERT (both slots are still placed).
 * Results are bit-exact and independent of launch configuration.
 */
MOE_API int moe_dispatch_layout(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                        int32_t* expert_counts, int32_t* expert_offsets,
                        int32_t* rank_counts, int32_t* rank_offsets, int32_t* dst_row,
                        int32_t* row_src, uint32_t* tile_ready, int64_t P_cap,
                        int32_t* d_status, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * Allocation-free form of moe_dispatch_layout.  The pages have no
 * counterpart; this exists for callers that cannot allocate device memory
 * when they call: engines whose device memory is planned once at start-up
 * and may not grow, foreign-language callers with no device allocator at
 * hand, and hot paths that must not pay for cudaMalloc, which can
 * synchronise the whole device.
 *
 * Same arguments, outputs and results as moe_dispatch_layout, minus the
 * workspace: the scratch lives in a static device array of
 * MOE_LAYOUT_STATIC_SCRATCH_BYTES that is part of the library image, so every
 * GPU that loads the library holds it until the process exits.  The call
 * makes no allocation of any kind.
 *   - Sizes: accepted while moe_layout_workspace_bytes(T, K, E) is at most
 *     MOE_LAYOUT_STATIC_SCRATCH_BYTES (for E=256, K=8: up to 116480 tokens);
 *     larger sizes return MOE_ERR_UNSUPPORTED before anything is launched.
 *   - Set-up: the first call on each device looks up that device's address
 *     of the array (cudaGetSymbolAddress, with the device current); make
 *     that first call before any stream capture.  A failed lookup returns
 *     MOE_ERR_CUDA.  The address is kept for the life of the process, so a
 *     device reset (cudaDeviceReset, or anything that destroys the primary
 *     context) between calls is not supported: the array may move and the
 *     kept address would then be stale.
 *   - Sharing: all calls on a device use the same array, which keeps the last
 *     call's contents.  Nothing in it needs to start at zero (every word the
 *     kernels read is written earlier in the same call), but calls that may
 *     overlap on the GPU (different streams without ordering between them)
 *     race on it; order them, or use moe_dispatch_layout with separate
 *     workspaces.
 */
#define MOE_LAYOUT_STATIC_SCRATCH_BYTES (4u << 20)
MOE_API int moe_dispatch_layout_static(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                                       int32_t* expert_counts, int32_t* expert_offsets,
                                       int32_t* rank_counts, int32_t* rank_offsets,
                                       int32_t* dst_row, int32_t* row_src,
                                       uint32_t* tile_ready, int64_t P_cap, int32_t* d_status,
                                       void* stream);

/*
 * Dispatch permute (the fused unzip of [DEP]; produces [ASC] expand_x).
 *   xp[dst_row[t*K+k]] = x[t]  for every placed slot, byte for byte;
 *   padding rows [offsets[e] + counts[e], offsets[e+1]) = 0 (E4M3: code
 *   0x00 and scale 0.0f); rows >= P untouched.
 *
 * In:
 *   x        [T, H] of `dtype`, row stride x_row_stride elements (>= H);
 *            16-byte aligned base, row bytes and stride multiples of 16
 *            (bf16: H % 8 == 0; E4M3: H % 128 == 0).
 *   x_scales fp32 [T, H/128], row stride x_scales_row_stride (E4M3 only;
 *            NULL for bf16).
 *   dst_row, expert_counts, expert_offsets: as produced by the layout call.
 * Out:
 *   xp        [P_cap, H] of `dtype`, contiguous, 16-byte aligned.
 *   xp_scales fp32 [P_cap, H/128] (E4M3 only; NULL for bf16).
 *   tile_ready (nullable) counters zeroed by the layout call; every row
 *            written adds 1 to tile_ready[row/128] once its bytes (and
 *            scales) are globally visible, behind a gpu-scope release
 *            (fence.acq_rel.gpu, then relaxed atomic adds), so a tile whose
 *            counter reads 128 with an ld.acquire.gpu is complete.  Each
 *            CTA counts its rows per tile and adds them when all of its rows
 *            have landed (with more than 8192 tiles: in batches as it goes);
 *            a tile's rows come from tokens across the whole batch, so tiles
 *            complete near the end of the launch either way.
 * Scheduling words:
 *   work     device uint32 [2], 4-byte aligned, non-NULL: the claim counter
 *            through which the copy pipelines take tokens and padding rows as
 *            they go (so pipelines on faster SMs take more of the work), and
 *            a count of finished pipelines.  They must be zero before the
 *            first call that uses them; every completed call returns them to
 *            zero.  Calls that share the same words must not overlap on the
 *            GPU (order them on one stream, or give each its own words).
 * Data errors: MOE_ERR_BOUNDS if a dst_row entry or offset leaves
 *   [0, P_cap) (that write is skipped); MOE_ERR_TIMEOUT if a staged load
 *   did not land within about 2 s (outputs and device state are then
 *   undefined: see the conventions above).
 */
MOE_API int moe_dispatch_permute(const void* x, int dtype, int64_t T, int H, int64_t x_row_stride,
                         const float* x_scales, int64_t x_scales_row_stride,
                         const int32_t* dst_row, int K, const int32_t* expert_counts,
                         const int32_t* expert_offsets, int E, void* xp, float* xp_scales,
                         int64_t P_cap, uint32_t* tile_ready, uint32_t* work,
                         int32_t* d_status, void* stream);

/*
 * Dispatch in one call ([DEP] fused unzip; [ASC] expand_x, expand_idx,
 * ep_send_counts): moe_dispatch_layout followed by moe_dispatch_permute, with
 * the same arguments, outputs, errors and results as those two calls made
 * back to back on `stream` (x, dtype, H, x_row_stride, x_scales,
 * x_scales_row_stride, xp, xp_scales and work as in moe_dispatch_permute;
 * the rest as in moe_dispatch_layout; counters are always maintained when
 * tile_ready is given).  In one call the permute's first row loads overlap
 * the layout, so x (and x_scales) must not overlap any buffer the call
 * writes; like every input, x must be complete in stream order when the call
 * is enqueued.  Every argument is checked before anything is launched.
 */
MOE_API int moe_dispatch(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                         const void* x, int dtype, int H, int64_t x_row_stride,
                         const float* x_scales, int64_t x_scales_row_stride,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                         int32_t* rank_offsets, int32_t* dst_row, int32_t* row_src,
                         uint32_t* tile_ready, int64_t P_cap, void* workspace,
                         size_t workspace_bytes, void* xp, float* xp_scales, uint32_t* work,
                         int32_t* d_status, void* stream);

/*
 * Counter-driven overlap: the dispatch permute and a consumer of its
 * chunk-completion counters in ONE cooperative launch ([DEP]: a consumer
 * acquires each chunk once and must then see all of it).  Warp 0 of every
 * CTA is a tile-ordered copy pipeline: the padded rows are cut into 16-row
 * items dealt round-robin to the CTAs, each filled row by row (source rows
 * found through row_src) and added to its tile's counter as it lands, so
 * tiles complete roughly in index order while the copy runs.  Warps 1..3
 * are the CTA's consumer group: for each of the same items it waits until
 * the item's tile counter reads 128 (ld.acquire.gpu), reads the item and
 * adds its share of the tile's checksum, as moe_wait_tiles_checksum defines
 * it (an expert stand-in that reads every byte, scales included; partial
 * sums add mod 2^32, so their order does not matter).  The cooperative
 * launch keeps all CTAs resident, so no consumer waits on a producer that
 * cannot run.
 * Arguments: as moe_dispatch_permute, plus row_src from the layout call
 * (required), tile_ready (required, zeroed by the layout call), checksums
 * uint32 [ceil(P_cap/128)] (no initialisation needed; each tile's entry is
 * cleared before its first item is published) and timeout_ns, the longest
 * wait for one tile; xp_scales, when given, 16-byte aligned.  A wait that
 * runs out sets MOE_ERR_TIMEOUT (that tile's checksum is then incomplete);
 * MOE_ERR_UNSUPPORTED if the device cannot hold the cooperative grid.  xp,
 * xp_scales and the counters end as after moe_dispatch_permute.
 */
MOE_API int moe_dispatch_permute_consume(const void* x, int dtype, int64_t T, int H,
                                         int64_t x_row_stride, const float* x_scales,
                                         int64_t x_scales_row_stride, const int32_t* dst_row,
                                         int K, const int32_t* expert_counts,
                                         const int32_t* expert_offsets, int E,
                                         const int32_t* row_src, void* xp, float* xp_scales,
                                         int64_t P_cap, uint32_t* tile_ready,
                                         uint32_t* checksums, int64_t timeout_ns,
                                         int32_t* d_status, void* stream);

/*
 * Fused quantise-on-dispatch (the FP8 dispatch of [DEP] Testing, with the
 * codes and scales of moe_quantize_e4m3 written straight into the
 * expert-major buffer).  Byte for byte the same as moe_quantize_e4m3
 * followed by moe_dispatch_permute(MOE_DTYPE_E4M3), without the
 * intermediate code buffer:
 *   per token t and 128-channel block b: s = amax|x| / 448 (fp32; 1 if the
 *   block is zero), q = E4M3(x / s) (fp32 division, nearest-even,
 *   saturating); xp[dst_row[t*K+k]] = q[t], xp_scales[dst_row[t*K+k]] = s[t];
 *   padding rows: code 0x00, scale 0.0f; rows >= P untouched.
 * In:  x bf16 [T, H], row stride x_row_stride elements (multiple of 8),
 *      16-byte aligned; H % 128 == 0.
 * Out: xp uint8 [P_cap, H] (16-byte aligned); xp_scales fp32 [P_cap, H/128]
 *      (4-byte aligned; with 16-byte alignment and H % 512 == 0 the scales
 *      are bulk-stored with the codes); tile_ready (nullable) and work
 *      (scheduling words, uint32 [2], zero between calls) as in
 *      moe_dispatch_permute.
 * Data errors: MOE_ERR_BOUNDS as in moe_dispatch_permute.
 */
MOE_API int moe_dispatch_permute_quant(const void* x, int64_t T, int H, int64_t x_row_stride,
                                       const int32_t* dst_row, int K,
                                       const int32_t* expert_counts,
                                       const int32_t* expert_offsets, int E, void* xp,
                                       float* xp_scales, int64_t P_cap, uint32_t* tile_ready,
                                       uint32_t* work, int32_t* d_status, void* stream);

/*
 * Combine ([ASC] function description, expert_scales, shared_expert_x):
 *   out[t] = bf16( sum_{k=0..K-1} scales[t,k] * y[dst_row[t*K+k]] + shared_x[t] )
 * computed per element in fp32: acc = 0; acc = fma(scales[t,k], y, acc) for
 * k = 0, 1, ..., K-1 in that order; acc = acc + shared_x; one round-to-
 * nearest-even to bf16.  The shared-expert term has no weight.
 *
 * In:  y bf16 [P_cap, H] contiguous; scales fp32 [T, K]; dst_row int32 [T*K];
 *      shared_x bf16 [T, H] or NULL (no shared expert).
 * Out: out bf16 [T, H] contiguous.
 * H % 8 == 0; y, shared_x, out 16-byte aligned.
 * Slots with dst_row == -1 add nothing; other out-of-range rows set
 * MOE_ERR_BOUNDS and add nothing.
 */
MOE_API int moe_combine(const void* y, const int32_t* dst_row, const float* scales,
                const void* shared_x, int64_t T, int K, int H, int64_t P_cap, void* out,
                int32_t* d_status, void* stream);

/*
 * Backward of combine (out is linear in y and in scales):
 *   grad_y[dst_row[t*K+k]] = bf16( scales[t,k] * grad_out[t] )   (the exact
 *                            product, rounded once to nearest-even)
 *   grad_scales[t*K+k]     = sum_h grad_out[t,h] * y[dst_row[t*K+k], h]
 *                            (fp32, fixed order for a given H)
 *   padding rows of grad_y below P are set to 0; rows >= P untouched.
 * In:  grad_out bf16 [T, H]; y bf16 [P_cap, H]; scales fp32 [T, K];
 *      dst_row, expert_counts, expert_offsets from the layout call.
 * Out: grad_y bf16 [P_cap, H]; grad_scales fp32 [T, K].
 */
MOE_API int moe_combine_bwd(const void* grad_out, const void* y, const float* scales,
                    const int32_t* dst_row, const int32_t* expert_counts,
                    const int32_t* expert_offsets, int E, int64_t T, int K, int H,
                    int64_t P_cap, void* grad_y, float* grad_scales, int32_t* d_status,
                    void* stream);

/*
 * Backward of dispatch (the permute copies x[t] into K rows; its adjoint
 * adds them back):
 *   grad_x[t] = bf16( sum_{k in order} grad_xp[dst_row[t*K+k]] )   (fp32 adds)
 * In:  grad_xp bf16 [P_cap, H]; dst_row int32 [T*K].   Out: grad_x bf16 [T, H].
 */
MOE_API int moe_dispatch_bwd(const void* grad_xp, const int32_t* dst_row, int64_t T, int K, int H,
                     int64_t P_cap, void* grad_x, int32_t* d_status, void* stream);

/*
 * E4M3 quantisation with one fp32 scale per 128 channels (the FP8 dispatch
 * input: codes plus scales carried alongside).  Per token t and block b:
 *   s = amax|x| / 448 in fp32 (1 if amax == 0);
 *   q = E4M3(x / s) with fp32 division, round-to-nearest-even, saturating
 *       at +-448.
 * In:  x bf16 [T, H], row stride x_row_stride elements (multiple of 8),
 *      16-byte aligned (32-byte aligned x with a stride that is a multiple of
 *      16 is read 32 bytes per load); H % 128 == 0.
 * Out: q uint8 [T, H] contiguous, 8-byte aligned (16-byte aligned q is
 *      written with 16-byte stores); q_scales fp32 [T, H/128] contiguous.
 */
MOE_API int moe_quantize_e4m3(const void* x, int64_t T, int H, int64_t x_row_stride, void* q,
                      float* q_scales, int32_t* d_status, void* stream);

/*
 * Reference consumer of the chunk-completion counters ([DEP]: one acquire
 * per chunk).  For every tile j < P/128 (P = expert_offsets[E]) it polls
 * tile_ready[j] with ld.acquire.gpu until it reads 128, at most timeout_ns
 * nanoseconds, then reads the tile and writes
 *   checksums[j] = sum_i w_i * (2i + 1)  mod 2^32
 * over the tile's 32-bit words w_i (128 rows of row_bytes, then, when
 * xp_scales is given, 128 scale rows of 4*scale_cols bytes).  A wait that
 * runs out sets MOE_ERR_TIMEOUT and leaves checksums[j] unwritten; once the
 * status is non-zero no further wait is started.
 * row_bytes % 4 == 0; checksums uint32 [ceil(P_cap/128)].
 */
MOE_API int moe_wait_tiles_checksum(const uint32_t* tile_ready, const int32_t* expert_offsets, int E,
                            const void* xp, int64_t row_bytes, const float* xp_scales,
                            int scale_cols, int64_t P_cap, uint32_t* checksums,
                            int64_t timeout_ns, int32_t* d_status, void* stream);

/*
 * Host balance planner over the layout's per-expert counts (host memory;
 * copy expert_counts back first).  Sources: the DeepEP pull request's
 * water-filling chunk-migration planner (expert-affinity batching, makespan
 * guard, cost-aware no-op, 128-aligned fine-balance pass; section "Python")
 * and TEMPO's max-affine cost (summary, section 2): a logical rank's time is
 *   t_r = max(a + b*G + b2*(tiles - G), c + beta*N) + mig * (tokens moved in)
 * with G the experts that have tokens on r, N its tokens and tiles the sum of
 * their ceil(n / 128).  Rank r starts with the experts [r*E/R, (r+1)*E/R).
 * Each step pairs the most expensive rank (src, lowest index on ties) with
 * the cheapest (dst) and moves 128-token chunks (the remainder when fewer
 * are left) of one expert: experts already on dst first, then most tokens
 * on src, then lower id.  Pass 1 moves the most whole chunks that keep dst
 * no costlier than src (at least one); pass 2 moves one chunk.  A move is
 * kept only if it lowers the makespan by more than min_gain (>= 0); a pass
 * ends when no candidate helps or max_moves moves exist.  Costs are double,
 * evaluated in the order written, so plans are reproducible bit for bit.
 * Out: moves[0..*n_moves) in the order made, makespans before and after
 * (either pointer may be NULL).  No GPU work; returns MOE_ERR_INVALID_ARG
 * on bad sizes (E % R != 0, E > 512, negative counts).
 */
typedef struct {
  int32_t expert, src_rank, dst_rank, tokens;
} moe_move_t;

typedef struct {
  double a, b, b2, c, beta, mig;
} moe_cost_model_t;

MOE_API int moe_plan_balance(const int32_t* expert_counts, int E, int R,
                             const moe_cost_model_t* cost, double min_gain, int max_moves,
                             moe_move_t* moves, int* n_moves, double* makespan_before,
                             double* makespan_after);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DISPATCH_H_ */
