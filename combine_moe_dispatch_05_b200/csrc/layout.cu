// Dispatch layout: validation, per-expert counting, padded prefix sums and the
// stable slot -> row map.
//
// Defined by: torch_npu "npu_moe_distribute_combine" API reference
// (expert_ids: ids in [0, moe_expert_num), no repeats in a row; expand_idx and
// ep_send_counts: per-expert counts, prefix-sum form), the TEMPO summary,
// section 1 (128-token M-tiles), and the DeepEP fused-unzip mapping table
// (PR "Intra-node compute compensation + overlap robustness", Kernel / host).
//
// Three launches, all deterministic (positions come from ordered scans, never
// from the order in which atomics arrive):
//   1. count:  each block owns a contiguous run of whole tokens (<= 512 slots).
//      Warp w walks its 64-slot segment 32 slots at a time; __match_any_sync
//      groups lanes with the same expert, the popcount of the lower lanes is
//      the rank inside the group, and a per-warp shared histogram carries the
//      running count.  A scan over the 8 warps turns those into ranks inside
//      the block (written to scratch) and the block's per-expert totals.
//      Also validates the ids and resets row_src / tile_ready.
//   2. scan:   one warp per expert scans the block totals in block order ->
//      each block's base inside the expert, and c_e.
//   3. assign: every block rebuilds the padded expert offsets from c_e with a
//      block scan (E <= 512), block 0 publishes offsets and the per-rank
//      sums, and each slot gets row = offset_e + block base + rank.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kSlotsPerBlock = 512;
constexpr int kItersPerWarp = kSlotsPerBlock / kLayoutThreads;  // 2

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(kLayoutThreads)
layout_count_kernel(const int32_t* __restrict__ ids, int64_t T, int K, int E,
                    int tokens_per_block, int32_t* __restrict__ block_counts,
                    int32_t* __restrict__ slot_rank, int32_t* __restrict__ row_src,
                    int64_t P_cap, uint32_t* __restrict__ tile_ready, int64_t n_tiles,
                    int32_t* status) {
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;                      // [kLayoutWarps][E]
  int32_t* s_ids = smem + kLayoutWarps * E;  // [kSlotsPerBlock]

  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)b * tokens_per_block;
  const int nt = (int)max((int64_t)0, min((int64_t)tokens_per_block, T - t0));
  const int n_b = nt * K;
  const int64_t s0 = t0 * K;

  // reset the inverse map and the chunk counters (grid-stride)
  {
    const int64_t gt = (int64_t)b * kLayoutThreads + tid;
    const int64_t gs = (int64_t)gridDim.x * kLayoutThreads;
    if (row_src)
      for (int64_t p = gt; p < P_cap; p += gs) row_src[p] = -1;
    if (tile_ready)
      for (int64_t j = gt; j < n_tiles; j += gs) tile_ready[j] = 0u;
  }

  for (int i = tid; i < kLayoutWarps * E; i += kLayoutThreads) hist[i] = 0;
  for (int i = tid; i < n_b; i += kLayoutThreads) s_ids[i] = ids[s0 + i];
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  int my_e[kItersPerWarp], my_r[kItersPerWarp];
  int err = 0;
#pragma unroll
  for (int it = 0; it < kItersPerWarp; ++it) {
    const int rel = warp * (kItersPerWarp * 32) + it * 32 + lane;
    int e = -1;
    if (rel < n_b) {
      const int v = s_ids[rel];
      if (v < 0 || v >= E) {
        if (!err) err = MOE_ERR_EXPERT_RANGE;
      } else {
        e = v;
        const int k = rel % K;
        const int base = rel - k;
        for (int j = 0; j < k; ++j)
          if (s_ids[base + j] == v && !err) err = MOE_ERR_DUPLICATE_EXPERT;
      }
    }
    const int key = e >= 0 ? e : -(lane + 1);  // invalid slots match nobody
    const unsigned grp = __match_any_sync(0xffffffffu, key);
    int prev = 0;
    if (e >= 0) prev = hist[warp * E + e];
    __syncwarp();
    if (e >= 0 && lane == __ffs(grp) - 1) hist[warp * E + e] = prev + __popc(grp);
    __syncwarp();
    my_e[it] = e;
    my_r[it] = e >= 0 ? prev + __popc(grp & lanemask_lt()) : -1;
  }
  if (err) record_error(status, err);
  __syncthreads();

  // exclusive scan over warps per expert -> warp bases; block totals out
  for (int e = tid; e < E; e += kLayoutThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kLayoutWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    block_counts[(int64_t)b * E + e] = run;
  }
  __syncthreads();

#pragma unroll
  for (int it = 0; it < kItersPerWarp; ++it) {
    const int rel = warp * (kItersPerWarp * 32) + it * 32 + lane;
    if (rel < n_b)
      slot_rank[s0 + rel] = my_e[it] >= 0 ? hist[warp * E + my_e[it]] + my_r[it] : -1;
  }
}

// One warp per expert: exclusive scan of the per-block counts in block order.
__global__ void __launch_bounds__(256)
layout_scan_kernel(int32_t* __restrict__ block_counts, int nb, int E,
                   int32_t* __restrict__ expert_counts) {
  const int e = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= E) return;  // whole warp exits together
  const int chunk = (nb + 31) / 32;
  const int b0 = min(nb, lane * chunk), b1 = min(nb, b0 + chunk);
  int sum = 0;
  for (int b = b0; b < b1; ++b) sum += block_counts[(int64_t)b * E + e];
  const int incl = warp_inclusive_scan(sum);
  int run = incl - sum;
  for (int b = b0; b < b1; ++b) {
    const int c = block_counts[(int64_t)b * E + e];
    block_counts[(int64_t)b * E + e] = run;
    run += c;
  }
  if (lane == 31) expert_counts[e] = incl;
}

// Block-wide exclusive scan of 128*ceil(c_e/128) over E <= 512 experts into
// s_off[0..E] (s_off[E] = total).  Every thread of the block must call it.
__device__ void padded_offsets_block(const int32_t* __restrict__ counts, int E, int32_t* s_off,
                                     int32_t* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e0 = 2 * tid, e1 = 2 * tid + 1;
  const int p0 = e0 < E ? (counts[e0] + kTile - 1) / kTile * kTile : 0;
  const int p1 = e1 < E ? (counts[e1] + kTile - 1) / kTile * kTile : 0;
  const int local = p0 + p1;
  const int incl = warp_inclusive_scan(local);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
    const int wi = warp_inclusive_scan(v);
    if (lane < (int)(blockDim.x >> 5)) s_warp[lane] = wi - v;
  }
  __syncthreads();
  const int excl = s_warp[warp] + incl - local;
  if (e0 < E) s_off[e0] = excl;
  if (e1 < E) s_off[e1] = excl + p0;
  if (e1 == E - 1 || e0 == E - 1) s_off[E] = excl + local;
  __syncthreads();
}

__global__ void __launch_bounds__(kLayoutThreads)
layout_assign_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ slot_rank,
                     const int32_t* __restrict__ block_bases,
                     const int32_t* __restrict__ expert_counts, int64_t T, int K, int E, int R,
                     int tokens_per_block, int32_t* __restrict__ expert_offsets,
                     int32_t* __restrict__ rank_counts, int32_t* __restrict__ rank_offsets,
                     int32_t* __restrict__ dst_row, int32_t* __restrict__ row_src,
                     int64_t P_cap, int32_t* status) {
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_warp[kLayoutWarps];
  padded_offsets_block(expert_counts, E, s_off, s_warp);

  const int b = blockIdx.x, tid = threadIdx.x;
  if (b == 0) {
    for (int e = tid; e <= E; e += kLayoutThreads) expert_offsets[e] = s_off[e];
    const int El = E / R;
    for (int r = tid; r < R; r += kLayoutThreads) {
      int s = 0;
      for (int e = r * El; e < (r + 1) * El; ++e) s += expert_counts[e];
      rank_counts[r] = s;
      rank_offsets[r] = s_off[r * El];
    }
    if (tid == 0) rank_offsets[R] = s_off[E];
  }

  const int64_t t0 = (int64_t)b * tokens_per_block;
  const int nt = (int)max((int64_t)0, min((int64_t)tokens_per_block, T - t0));
  const int n_b = nt * K;
  const int64_t s0 = t0 * K;
  for (int i = tid; i < n_b; i += kLayoutThreads) {
    const int64_t slot = s0 + i;
    const int r = slot_rank[slot];
    if (r < 0) {
      dst_row[slot] = -1;
      continue;
    }
    const int e = ids[slot];
    const int64_t row = (int64_t)s_off[e] + block_bases[(int64_t)b * E + e] + r;
    if (row < 0 || row >= P_cap) {  // unreachable when P_cap passed the host check
      record_error(status, MOE_ERR_BOUNDS);
      dst_row[slot] = -1;
      continue;
    }
    dst_row[slot] = (int32_t)row;
    if (row_src) row_src[row] = (int32_t)slot;
  }
}

inline int tokens_per_block_for(int K) { return kSlotsPerBlock / K; }

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace moe

extern "C" size_t moe_layout_workspace_bytes(int64_t T, int K, int E) {
  if (T < 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 || E > MOE_MAX_EXPERTS) return (size_t)-1;
  const int tpb = moe::tokens_per_block_for(K);
  const int64_t nb = T > 0 ? (T + tpb - 1) / tpb : 1;
  return moe::align256((size_t)nb * E * sizeof(int32_t)) +
         moe::align256((size_t)T * K * sizeof(int32_t));
}

extern "C" int moe_dispatch_layout(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                                   int32_t* expert_counts, int32_t* expert_offsets,
                                   int32_t* rank_counts, int32_t* rank_offsets,
                                   int32_t* dst_row, int32_t* row_src, uint32_t* tile_ready,
                                   int64_t P_cap, int32_t* d_status, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  using namespace moe;
  if (T < 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 || E > MOE_MAX_EXPERTS || R < 1 || R > E ||
      E % R != 0)
    return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)K > (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  const int64_t need = moe_padded_capacity(T, K, E);
  if (P_cap > (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (P_cap < need) return MOE_ERR_CAPACITY;
  if (!expert_counts || !expert_offsets || !rank_counts || !rank_offsets || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !dst_row)) return MOE_ERR_INVALID_ARG;
  if (!moe_host::aligned16(workspace)) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe_layout_workspace_bytes(T, K, E)) return MOE_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int tpb = tokens_per_block_for(K);
  const int nb = T > 0 ? (int)((T + tpb - 1) / tpb) : 1;
  int32_t* block_counts = static_cast<int32_t*>(workspace);
  int32_t* slot_rank = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                                  align256((size_t)nb * E * sizeof(int32_t)));
  const int64_t n_tiles = (P_cap + kTile - 1) / kTile;
  const size_t smem1 = (size_t)(kLayoutWarps * E + kSlotsPerBlock) * sizeof(int32_t);

  layout_count_kernel<<<nb, kLayoutThreads, smem1, s>>>(topk_idx, T, K, E, tpb, block_counts,
                                                        slot_rank, row_src, P_cap, tile_ready,
                                                        n_tiles, d_status);
  const int scan_blocks = (E * 32 + 255) / 256;
  layout_scan_kernel<<<scan_blocks, 256, 0, s>>>(block_counts, nb, E, expert_counts);
  layout_assign_kernel<<<nb, kLayoutThreads, 0, s>>>(
      topk_idx, slot_rank, block_counts, expert_counts, T, K, E, R, tpb, expert_offsets,
      rank_counts, rank_offsets, dst_row, row_src, P_cap, d_status);
  return moe_host::launch_status();
}
