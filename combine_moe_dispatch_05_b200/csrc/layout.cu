// Dispatch layout: validation, per-expert counting, padded prefix sums and the
// stable slot -> row map.
//
// Defined by: torch_npu "npu_moe_distribute_combine" API reference
// (expert_ids: ids in [0, moe_expert_num), no repeats in a row; expand_idx and
// ep_send_counts: per-expert counts, prefix-sum form), the TEMPO summary,
// section 1 (128-token M-tiles), and the DeepEP fused-unzip mapping table
// (PR "Intra-node compute compensation + overlap robustness", Kernel / host).
//
// Two launches, deterministic by construction (positions come from ordered
// scans, never from the order in which atomics arrive):
//   1. count:  each 1024-thread block owns a contiguous run of whole tokens
//      (<= 1024 slots up to 65536 slots in all, else <= 2048).  Warp w walks
//      its 32- or 64-slot segment 32 slots at a time;
//      ballots over the id bits group the lanes holding the same expert, the
//      popcount of the lower lanes is the rank inside the group, and a
//      per-warp 16-bit shared histogram carries the running count.  A scan
//      over the 32 warps turns these into each slot's rank inside the block
//      (written to scratch) and the block's per-expert totals.  The same
//      pass validates the ids and resets row_src and tile_ready.
//   2. assign: each block sums the per-block totals column by column (all
//      blocks -> c_e; blocks before it -> its base inside each expert),
//      rebuilds the padded offsets with a block scan over E <= 512 experts,
//      and gives every slot row = offset_e + base_e + rank.  Block 0
//      publishes counts, offsets and the per-rank sums.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kLayoutThreads = 1024;
constexpr int kLayoutWarps = kLayoutThreads / 32;
// A block owns kIters x 1024 slots (kIters 32-slot steps per warp): 1024 when
// the batch has at most kSmallLayoutSlots slots, where more, shorter blocks
// finish sooner; 2048 above, where the assign kernel's column sums over the
// per-block totals would grow with the block count instead.
constexpr int64_t kSmallLayoutSlots = 65536;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Lanes of this warp holding the same valid expert id as this lane (itself
// included); an invalid lane matches nobody.  One ballot per bit of the id
// (nbits = bits of E-1, at most 9): two lanes agree on every bit exactly when
// they hold the same id.
__device__ __forceinline__ unsigned match_peers(int e, bool valid, int nbits, int lane) {
  unsigned peers = __ballot_sync(0xffffffffu, valid);
#pragma unroll
  for (int b = 0; b < 9; ++b) {
    if (b < nbits) {
      const bool bit = (e >> b) & 1;
      const unsigned m = __ballot_sync(0xffffffffu, bit);
      peers &= bit ? m : ~m;
    }
  }
  return valid ? peers : (1u << lane);
}

// One 32-slot step of the count.  rel: the slot's index in the block's run
// (n_b slots, starting at a token boundary; the warp's steps start at
// multiples of 32); v: its id.  Validates the id, finds the slot's rank among
// the earlier slots of the same expert in this warp's segment from the
// warp's running histogram h, and advances h.  Duplicates inside a token are
// found from the match when K is a power of two (the token's K slots are one
// aligned group of K lanes), else by comparing with the token's earlier ids.
__device__ __forceinline__ void count_step(int rel, int n_b, int v, int K, int E, int nbits,
                                           const int32_t* s_ids, uint16_t* h, int lane,
                                           int& err, int& e_out, int& r_out) {
  const bool k_pow2 = (K & (K - 1)) == 0;
  int e = -1;
  if (rel < n_b) {
    if (v < 0 || v >= E) {
      if (!err) err = MOE_ERR_EXPERT_RANGE;
    } else {
      e = v;
      if (!k_pow2) {
        const int k = rel % K;
        const int base = rel - k;
        for (int j = 0; j < k; ++j)
          if (s_ids[base + j] == v && !err) err = MOE_ERR_DUPLICATE_EXPERT;
      }
    }
  }
  const unsigned peers = match_peers(e, e >= 0, nbits, lane);
  if (k_pow2 && e >= 0) {
    const unsigned tok = ((1u << K) - 1u) << (lane & ~(K - 1));  // K <= 16
    if ((peers & tok & lanemask_lt()) && !err) err = MOE_ERR_DUPLICATE_EXPERT;
  }
  int prev = 0;
  if (e >= 0) prev = h[e];
  __syncwarp();
  if (e >= 0 && lane == __ffs(peers) - 1) h[e] = (uint16_t)(prev + __popc(peers));
  __syncwarp();
  e_out = e;
  r_out = e >= 0 ? prev + __popc(peers & lanemask_lt()) : -1;
}

__device__ __forceinline__ int id_bits(int E) { return E > 1 ? 32 - __clz(E - 1) : 0; }

// dst[0..n) = value, by the threads gt = 0..gs-1: scalar words up to the first
// 16-byte boundary, 16-byte stores over the body, scalar words after it
__device__ __forceinline__ void fill_words(uint32_t* dst, int64_t n, uint32_t value, int64_t gt,
                                           int64_t gs) {
  int64_t head = (int64_t)((16 - (reinterpret_cast<uintptr_t>(dst) & 15)) & 15) / 4;
  if (head > n) head = n;
  if (gt < head) dst[gt] = value;
  const int64_t nv = (n - head) / 4;
  uint4* body = reinterpret_cast<uint4*>(dst + head);
  const uint4 v4 = make_uint4(value, value, value, value);
  for (int64_t i = gt; i < nv; i += gs) body[i] = v4;
  const int64_t tail0 = head + nv * 4;
  if (gt < n - tail0) dst[tail0 + gt] = value;
}

template <int kIters>
__global__ void __launch_bounds__(kLayoutThreads)
layout_count_kernel(const int32_t* __restrict__ ids, int64_t T, int K, int E,
                    int tokens_per_block, int32_t* __restrict__ block_counts,
                    int32_t* __restrict__ slot_rank, int32_t* __restrict__ row_src,
                    int64_t P_cap, uint32_t* __restrict__ tile_ready, int64_t n_tiles,
                    int32_t* status, int trigger) {
  pdl_begin();
  if (trigger) pdl_trigger();
  __shared__ __align__(16) uint16_t hist[kLayoutWarps * MOE_MAX_EXPERTS];  // [warp][E]
  __shared__ int32_t s_ids[kIters * kLayoutThreads];

  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)b * tokens_per_block;
  const int nt = (int)max((int64_t)0, min((int64_t)tokens_per_block, T - t0));
  const int n_b = nt * K;
  const int64_t s0 = t0 * K;

  for (int i = tid; i < n_b; i += kLayoutThreads) s_ids[i] = __ldg(ids + s0 + i);
  const int Es = (E + 7) & ~7;  // row pitch of hist: whole 16-byte rows
  {
    uint4* h4 = reinterpret_cast<uint4*>(hist);
    const int n4 = kLayoutWarps * Es * 2 / 16;
    for (int i = tid; i < n4; i += kLayoutThreads) h4[i] = make_uint4(0, 0, 0, 0);
  }
  // reset the inverse map and the chunk counters (grid-stride)
  {
    const int64_t gt = (int64_t)b * kLayoutThreads + tid;
    const int64_t gs = (int64_t)gridDim.x * kLayoutThreads;
    if (row_src)
      fill_words(reinterpret_cast<uint32_t*>(row_src), P_cap, 0xFFFFFFFFu, gt, gs);
    if (tile_ready)
      fill_words(tile_ready, n_tiles, 0u, gt, gs);
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  uint16_t* my_hist = hist + warp * Es;
  int my_e[kIters], my_r[kIters];
  int err = 0;
  const int nbits = id_bits(E);
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int rel = warp * (kIters * 32) + it * 32 + lane;
    count_step(rel, n_b, rel < n_b ? s_ids[rel] : -1, K, E, nbits, s_ids, my_hist, lane, err,
               my_e[it], my_r[it]);
  }
  if (err) record_error(status, err);
  __syncthreads();

  // exclusive scan over warps per expert -> warp bases; block totals out
  for (int e = tid; e < E; e += kLayoutThreads) {
    int run = 0;
#pragma unroll 8
    for (int w = 0; w < kLayoutWarps; ++w) {
      const int c = hist[w * Es + e];
      hist[w * Es + e] = (uint16_t)run;
      run += c;
    }
    block_counts[(int64_t)b * E + e] = run;
  }
  __syncthreads();

#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int rel = warp * (kIters * 32) + it * 32 + lane;
    if (rel < n_b) slot_rank[s0 + rel] = my_e[it] >= 0 ? my_hist[my_e[it]] + my_r[it] : -1;
  }
}

template <int kIters>
__global__ void __launch_bounds__(kLayoutThreads)
layout_assign_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ slot_rank,
                     const int32_t* __restrict__ block_counts, int nb, int64_t T, int K, int E,
                     int R, int tokens_per_block, int32_t* __restrict__ expert_counts,
                     int32_t* __restrict__ expert_offsets, int32_t* __restrict__ rank_counts,
                     int32_t* __restrict__ rank_offsets, int32_t* __restrict__ dst_row,
                     int32_t* __restrict__ row_src, int64_t P_cap, int32_t* status,
                     int trigger) {
  pdl_begin();
  if (trigger) pdl_trigger();
  __shared__ int32_t s_pre[kLayoutThreads];   // [group][E] partial sums of earlier blocks
  __shared__ int32_t s_tot[kLayoutThreads];   // [group][E] partial sums of all blocks
  __shared__ int32_t s_base[MOE_MAX_EXPERTS];
  __shared__ int32_t s_cnt[MOE_MAX_EXPERTS];
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_warp[kLayoutWarps];

  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // this block's slots: their ranks and ids are fetched first, so those loads
  // are in flight while the column sums below are formed
  const int64_t t0 = (int64_t)b * tokens_per_block;
  const int nt = (int)max((int64_t)0, min((int64_t)tokens_per_block, T - t0));
  const int n_b = nt * K;
  const int64_t s0 = t0 * K;
  int my_rank[kIters], my_id[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = tid + it * kLayoutThreads;
    my_rank[it] = i < n_b ? slot_rank[s0 + i] : -1;
    my_id[it] = i < n_b ? __ldg(ids + s0 + i) : 0;
  }

  // 1. column sums of the per-block totals, split into ng interleaved groups
  const int ng = kLayoutThreads / E;  // >= 2 since E <= 512
  if (tid < ng * E) {
    const int e = tid % E, g = tid / E;
    int pre = 0, tot = 0;
    int r = g;
    for (; r + 3 * ng < nb; r += 4 * ng) {  // four independent loads in flight
      const int c0 = __ldg(block_counts + (int64_t)r * E + e);
      const int c1 = __ldg(block_counts + (int64_t)(r + ng) * E + e);
      const int c2 = __ldg(block_counts + (int64_t)(r + 2 * ng) * E + e);
      const int c3 = __ldg(block_counts + (int64_t)(r + 3 * ng) * E + e);
      tot += c0 + c1 + c2 + c3;
      pre += (r < b ? c0 : 0) + (r + ng < b ? c1 : 0) + (r + 2 * ng < b ? c2 : 0) +
             (r + 3 * ng < b ? c3 : 0);
    }
    for (; r < nb; r += ng) {
      const int c = __ldg(block_counts + (int64_t)r * E + e);
      tot += c;
      if (r < b) pre += c;
    }
    s_pre[tid] = pre;
    s_tot[tid] = tot;
  }
  __syncthreads();
  int padded = 0;
  if (tid < E) {
    int pre = 0, tot = 0;
    for (int g = 0; g < ng; ++g) {
      pre += s_pre[g * E + tid];
      tot += s_tot[g * E + tid];
    }
    s_base[tid] = pre;
    s_cnt[tid] = tot;
    padded = (tot + kTile - 1) / kTile * kTile;
  }

  // 2. exclusive block scan of the padded counts -> s_off[0..E]
  const int incl = warp_inclusive_scan(padded);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = s_warp[lane];
    const int wi = warp_inclusive_scan(v);
    s_warp[lane] = wi - v;
  }
  __syncthreads();
  if (tid < E) s_off[tid] = s_warp[warp] + incl - padded;
  if (tid == E - 1) s_off[E] = s_warp[warp] + incl;
  __syncthreads();

  if (b == 0) {
    for (int e = tid; e < E; e += kLayoutThreads) expert_counts[e] = s_cnt[e];
    for (int e = tid; e <= E; e += kLayoutThreads) expert_offsets[e] = s_off[e];
    const int El = E / R;
    for (int r = tid; r < R; r += kLayoutThreads) {
      int s = 0;
      for (int e = r * El; e < (r + 1) * El; ++e) s += s_cnt[e];
      rank_counts[r] = s;
      rank_offsets[r] = s_off[r * El];
    }
    if (tid == 0) rank_offsets[R] = s_off[E];
  }

  // 3. rows of this block's slots
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int i = tid + it * kLayoutThreads;
    if (i >= n_b) continue;
    const int64_t slot = s0 + i;
    const int r = my_rank[it];
    if (r < 0) {
      dst_row[slot] = -1;
      continue;
    }
    const int e = my_id[it];
    const int64_t row = (int64_t)s_off[e] + s_base[e] + r;
    if (row < 0 || row >= P_cap) {  // unreachable when P_cap passed the host check
      record_error(status, MOE_ERR_BOUNDS);
      dst_row[slot] = -1;
      continue;
    }
    dst_row[slot] = (int32_t)row;
    if (row_src) row_src[row] = (int32_t)slot;
  }
}

inline int layout_iters(int64_t T, int K) { return T * K <= kSmallLayoutSlots ? 1 : 2; }
inline int tokens_per_block_for(int64_t T, int K) {
  return layout_iters(T, K) * kLayoutThreads / K;
}

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace moe

extern "C" size_t moe_layout_workspace_bytes(int64_t T, int K, int E) {
  if (T < 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 || E > MOE_MAX_EXPERTS) return (size_t)-1;
  const int tpb = moe::tokens_per_block_for(T, K);
  const int64_t nb = T > 0 ? (T + tpb - 1) / tpb : 1;
  return moe::align256((size_t)nb * E * sizeof(int32_t)) +
         moe::align256((size_t)(T > 0 ? T : 1) * K * sizeof(int32_t));
}

namespace moe {
// The layout's checks and launches (see moe_dispatch_layout).  With dry_run
// the checks run and nothing is launched; with trigger both kernels let the
// next kernel in the stream launch right after their own grid wait.
int layout_launch(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                  int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                  int32_t* rank_offsets, int32_t* dst_row, int32_t* row_src,
                  uint32_t* tile_ready, int64_t P_cap, int32_t* d_status, void* workspace,
                  size_t workspace_bytes, cudaStream_t s, int trigger, int dry_run) {
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
  for (const void* q : {(const void*)topk_idx, (const void*)expert_counts,
                        (const void*)expert_offsets, (const void*)rank_counts,
                        (const void*)rank_offsets, (const void*)dst_row, (const void*)row_src,
                        (const void*)tile_ready})
    if (!moe_host::aligned4(q)) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe_layout_workspace_bytes(T, K, E)) return MOE_ERR_INVALID_ARG;
  if (dry_run) return MOE_OK;

  const int64_t n_tiles = (P_cap + kTile - 1) / kTile;
  const int tpb = tokens_per_block_for(T, K);
  const int nb = T > 0 ? (int)((T + tpb - 1) / tpb) : 1;
  int32_t* block_counts = static_cast<int32_t*>(workspace);
  int32_t* slot_rank = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                                  align256((size_t)nb * E * sizeof(int32_t)));

  const bool small = layout_iters(T, K) == 1;
  int st = moe_host::launch(small ? layout_count_kernel<1> : layout_count_kernel<2>, dim3(nb),
                            dim3(kLayoutThreads), 0, s, topk_idx, T, K, E, tpb, block_counts,
                            slot_rank, row_src, P_cap, tile_ready, n_tiles, d_status, trigger);
  if (st != MOE_OK) return st;
  return moe_host::launch(small ? layout_assign_kernel<1> : layout_assign_kernel<2>, dim3(nb),
                          dim3(kLayoutThreads), 0, s, topk_idx, (const int32_t*)slot_rank,
                          (const int32_t*)block_counts, nb, T, K, E, R, tpb, expert_counts,
                          expert_offsets, rank_counts, rank_offsets, dst_row, row_src, P_cap,
                          d_status, trigger);
}
}  // namespace moe

extern "C" int moe_dispatch_layout(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                                   int32_t* expert_counts, int32_t* expert_offsets,
                                   int32_t* rank_counts, int32_t* rank_offsets,
                                   int32_t* dst_row, int32_t* row_src, uint32_t* tile_ready,
                                   int64_t P_cap, int32_t* d_status, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return moe::layout_launch(topk_idx, T, K, E, R, expert_counts, expert_offsets, rank_counts,
                            rank_offsets, dst_row, row_src, tile_ready, P_cap, d_status,
                            workspace, workspace_bytes, static_cast<cudaStream_t>(stream), 0, 0);
}

// ---------------------------------------------------------------------------
// Allocation-free layout: the same two kernels, with their scratch in a
// file-scope device array instead of a caller-provided workspace.  Callers
// that cannot allocate device memory at call time use this one (see the
// header).  In host code the array's name is only a host-side stand-in, so
// each device's real address is looked up once, with that device current.
// ---------------------------------------------------------------------------
#include <mutex>

static __device__ __align__(256) unsigned char g_layout_scratch[MOE_LAYOUT_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_layout_scratch_mu;
void* g_layout_scratch_ptr[64] = {};
}  // namespace

extern "C" int moe_dispatch_layout_static(const int32_t* topk_idx, int64_t T, int K, int E,
                                          int R, int32_t* expert_counts,
                                          int32_t* expert_offsets, int32_t* rank_counts,
                                          int32_t* rank_offsets, int32_t* dst_row,
                                          int32_t* row_src, uint32_t* tile_ready,
                                          int64_t P_cap, int32_t* d_status, void* stream) {
  const size_t need = moe_layout_workspace_bytes(T, K, E);
  if (need == (size_t)-1) return MOE_ERR_INVALID_ARG;
  if (need > (size_t)MOE_LAYOUT_STATIC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_layout_scratch_mu);
    if (g_layout_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      g_layout_scratch_ptr[dev] = p;
    }
    scratch = g_layout_scratch_ptr[dev];
  }
  return moe_dispatch_layout(topk_idx, T, K, E, R, expert_counts, expert_offsets, rank_counts,
                             rank_offsets, dst_row, row_src, tile_ready, P_cap, d_status,
                             scratch, (size_t)MOE_LAYOUT_STATIC_SCRATCH_BYTES, stream);
}
