// Reference consumer of the chunk-completion counters (DeepEP pull request
// "Intra-node compute compensation + overlap robustness (CUDA719 fix)",
// Kernel / host: a consumer acquires "ready" once per chunk and must then see
// the whole chunk).  A chunk here is one 128-row M-tile of the expert-major
// buffer.
//
// One thread per CTA polls the tile's counter with ld.acquire.gpu (bounded by
// a caller-given timeout); the CTA barrier then orders that acquire before
// every thread's reads of the tile, which bypass L1 (ld.global.cg).  The tile
// is summarised by sum_i w_i * (2i + 1) mod 2^32 over its 32-bit words, which
// is order-independent to compute and changes if two unequal words swap.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kConsThreads = 256;

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_cg_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(kConsThreads)
tile_checksum_kernel(const uint32_t* tile_ready, const int32_t* __restrict__ offsets, int E,
                     const uint8_t* xp, int64_t row_bytes, const float* xs, int scale_cols,
                     int64_t P_cap, uint32_t* __restrict__ checksums, int64_t timeout_ns,
                     int vec16, int32_t* status) {
  pdl_begin();
  __shared__ int s_ok;
  __shared__ uint32_t s_red[kConsThreads / 32];
  const int tid = threadIdx.x;
  const int64_t P = __ldg(offsets + E);
  if (P < 0 || P > P_cap) {
    if (tid == 0 && blockIdx.x == 0) record_error(status, MOE_ERR_BOUNDS);
    return;
  }
  const int64_t n_tiles = P / kTile;
  const int64_t data_words = (int64_t)kTile * row_bytes / 4;
  const int64_t scale_words = xs ? (int64_t)kTile * scale_cols : 0;

  for (int64_t j = blockIdx.x; j < n_tiles; j += gridDim.x) {
    if (tid == 0) {
      int ok = 0;
      if (read_status(status) == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (true) {
          if (ld_acquire_gpu(tile_ready + j) == (uint32_t)kTile) {
            ok = 1;
            break;
          }
          if ((int64_t)(globaltimer_ns() - t0) > timeout_ns) break;
          __nanosleep(256);
        }
        if (!ok) record_error(status, MOE_ERR_TIMEOUT);
      }
      s_ok = ok;
    }
    __syncthreads();
    if (s_ok) {
      uint32_t acc = 0;
      if (vec16) {
        // 16-byte loads: word i = 4v + q gets weight 2i + 1
        const uint4* d4 = reinterpret_cast<const uint4*>(xp + j * kTile * row_bytes);
        const int64_t n4 = data_words / 4;
#pragma unroll 8
        for (int64_t v = tid; v < n4; v += kConsThreads) {
          const uint4 w = ld_cg_v4(d4 + v);
          const uint32_t i = 4u * (uint32_t)v;
          acc += w.x * (2u * i + 1u) + w.y * (2u * i + 3u) + w.z * (2u * i + 5u) +
                 w.w * (2u * i + 7u);
        }
        if (scale_words) {
          const uint4* s4 = reinterpret_cast<const uint4*>(xs + j * kTile * scale_cols);
          const int64_t m4 = scale_words / 4;
          for (int64_t v = tid; v < m4; v += kConsThreads) {
            const uint4 w = ld_cg_v4(s4 + v);
            const uint32_t i = (uint32_t)data_words + 4u * (uint32_t)v;
            acc += w.x * (2u * i + 1u) + w.y * (2u * i + 3u) + w.z * (2u * i + 5u) +
                   w.w * (2u * i + 7u);
          }
        }
      } else {
        const uint32_t* dw = reinterpret_cast<const uint32_t*>(xp + j * kTile * row_bytes);
        for (int64_t i = tid; i < data_words; i += kConsThreads)
          acc += ld_cg_u32(dw + i) * (uint32_t)(2 * i + 1);
        if (scale_words) {
          const uint32_t* sw = reinterpret_cast<const uint32_t*>(xs + j * kTile * scale_cols);
          for (int64_t i = tid; i < scale_words; i += kConsThreads)
            acc += ld_cg_u32(sw + i) * (uint32_t)(2 * (data_words + i) + 1);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if ((tid & 31) == 0) s_red[tid >> 5] = acc;
      __syncthreads();
      if (tid == 0) {
        uint32_t sum = 0;
        for (int w = 0; w < kConsThreads / 32; ++w) sum += s_red[w];
        checksums[j] = sum;
      }
    }
    __syncthreads();
  }
}

}  // namespace
}  // namespace moe

extern "C" int moe_wait_tiles_checksum(const uint32_t* tile_ready, const int32_t* expert_offsets,
                                       int E, const void* xp, int64_t row_bytes,
                                       const float* xp_scales, int scale_cols, int64_t P_cap,
                                       uint32_t* checksums, int64_t timeout_ns,
                                       int32_t* d_status, void* stream) {
  if (!tile_ready || !expert_offsets || !xp || !checksums || E < 1 || E > MOE_MAX_EXPERTS)
    return MOE_ERR_INVALID_ARG;
  if (row_bytes <= 0 || row_bytes % 4 != 0 || P_cap < 0 || timeout_ns < 0 ||
      (xp_scales && scale_cols <= 0) || !moe_host::aligned4(xp))
    return MOE_ERR_INVALID_ARG;
  const int dev = moe_host::current_device();
  const int64_t max_tiles = (P_cap + moe::kTile - 1) / moe::kTile;
  int64_t grid = (int64_t)moe_host::sm_count(dev) * 4;
  if (grid > max_tiles) grid = max_tiles;
  if (grid < 1) grid = 1;
  // 16-byte loads when every tile (and scale tile) starts on a 16-byte boundary
  const int vec16 = moe_host::aligned16(xp) && row_bytes % 16 == 0 &&
                    (!xp_scales || (moe_host::aligned16(xp_scales) &&
                                    ((int64_t)moe::kTile * scale_cols) % 4 == 0));
  return moe_host::launch(moe::tile_checksum_kernel, dim3((unsigned)grid), dim3(moe::kConsThreads),
                          0, static_cast<cudaStream_t>(stream), tile_ready, expert_offsets, E,
                          static_cast<const uint8_t*>(xp), row_bytes, xp_scales, scale_cols, P_cap,
                          checksums, timeout_ns, vec16, d_status);
}
