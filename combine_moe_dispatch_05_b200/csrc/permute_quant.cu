// Fused quantise-on-dispatch: bf16 token rows are quantised to E4M3 with one
// fp32 scale per 128 channels and the codes and scales are written straight
// into the expert-major buffer (the FP8 dispatch path of the DeepEP pull
// request "Intra-node compute compensation + overlap robustness (CUDA719
// fix)", Testing: FP8 dispatch; layout as in the torch_npu
// "npu_moe_distribute_combine" API's expand_x; 128-row M-tile padding from the
// TEMPO summary, section 1).  The result equals quantise-then-permute byte for
// byte, but x is read once and the intermediate codes never touch HBM.
//
// A 128-thread CTA owns a token: thread i holds 16-byte vectors i, i+128, ...
// of the bf16 row, four at a time with all four loads issued before any
// math; the 16 threads of a half-warp share one 128-channel block,
// reduce its amax with shuffles, divide by s = amax/448 in fp32 and convert
// with saturating round-to-nearest-even.  Pairs of lanes merge their 8 codes
// into one 16-byte store per destination row.  The next token's row indices
// are prefetched into shared memory while the current one is processed.
// Padding rows get code 0x00 and scale 0.  Each token's K rows are released
// on the chunk-completion counters after a CTA barrier and one
// fence.acq_rel.gpu.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQpThreads = 128;
constexpr int kQpU = 4;  // columns per thread per batch

struct QuantPermArgs {
  const uint16_t* x;
  int64_t x_stride;  // elements
  int64_t T;
  int H;
  int K;
  const int32_t* dst_row;
  const int32_t* counts;
  const int32_t* offsets;
  int E;
  uint8_t* xp;
  float* xp_scales;
  int64_t P_cap;
  uint32_t* tile_ready;
  int32_t* status;
};

__global__ void __launch_bounds__(kQpThreads) permute_quant_kernel(const QuantPermArgs a) {
  pdl_begin();
  __shared__ int32_t s_row[2][MOE_MAX_TOPK];
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_cnt[MOE_MAX_EXPERTS];
  __shared__ int32_t s_pad[MOE_MAX_EXPERTS];
  __shared__ int32_t s_padpref[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_warp[kQpThreads / 32];
  __shared__ int s_bad;

  const int tid = threadIdx.x, lane = tid & 31;
  const int E = a.E, K = a.K, H = a.H;
  const int V = H >> 3;        // 16-byte bf16 vectors per row
  const int nb = H >> 7;       // 128-channel blocks per row
  const unsigned half_mask = 0xFFFFu << (lane & 16);

  if (tid == 0) s_bad = 0;
  for (int e = tid; e <= E; e += kQpThreads) s_off[e] = __ldg(a.offsets + e);
  for (int e = tid; e < E; e += kQpThreads) s_cnt[e] = __ldg(a.counts + e);
  __syncthreads();
  for (int e = tid; e < E; e += kQpThreads) {
    const int pad = (s_off[e + 1] - s_off[e]) - s_cnt[e];
    const bool ok = pad >= 0 && pad < kTile && s_cnt[e] >= 0;
    if (!ok) s_bad = 1;
    s_pad[e] = ok ? pad : 0;
  }
  __syncthreads();
  block_exclusive_scan(s_pad, E, s_padpref, s_warp);
  if (s_bad || (int64_t)s_off[E] > a.P_cap || s_off[0] != 0) {
    if (tid == 0) record_error(a.status, MOE_ERR_BOUNDS);
    return;
  }

  auto fetch = [&](int64_t t, int buf) {
    if (tid < K && t < a.T) {
      int r = __ldg(a.dst_row + t * K + tid);
      if (r != -1 && (r < 0 || (int64_t)r >= a.P_cap)) {
        record_error(a.status, MOE_ERR_BOUNDS);
        r = -1;
      }
      s_row[buf][tid] = r;
    }
  };
  int buf = 0;
  fetch(blockIdx.x, 0);
  __syncthreads();
  for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
    fetch(t + gridDim.x, buf ^ 1);
    const uint16_t* xr = a.x + t * a.x_stride;
    // kQpU columns per thread per batch, all loads issued before any math;
    // a half-warp's 16 lanes share one 128-channel block in every column
    for (int vb = tid; vb < V; vb += kQpThreads * kQpU) {  // V % 16 == 0: half-warps stay whole
      uint4 d[kQpU];
#pragma unroll
      for (int i = 0; i < kQpU; ++i) {
        const int v = vb + i * kQpThreads;
        d[i] = v < V ? ld_nc_v4(xr + (int64_t)v * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kQpU; ++i) {
        const int v = vb + i * kQpThreads;
        if (v >= V) break;  // uniform across the half-warp
        const uint32_t w[4] = {d[i].x, d[i].y, d[i].z, d[i].w};
        float f[8];
        float amax = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          f[2 * q] = bf16_lo(w[q]);
          f[2 * q + 1] = bf16_hi(w[q]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(half_mask, amax, o, 16));
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint32_t c[2] = {0u, 0u};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 pr = make_float2(__fdiv_rn(f[2 * q], s), __fdiv_rn(f[2 * q + 1], s));
          const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
          c[q >> 1] |= c2 << (16 * (q & 1));
        }
        // even lanes store 16 codes: their own 8 and their odd neighbour's 8
        const uint32_t n0 = __shfl_down_sync(half_mask, c[0], 1, 16);
        const uint32_t n1 = __shfl_down_sync(half_mask, c[1], 1, 16);
        const int blk = v >> 4;
        for (int k = 0; k < K; ++k) {
          const int r = s_row[buf][k];
          if (r < 0) continue;
          if ((lane & 1) == 0)
            st_v4(a.xp + (int64_t)r * H + (int64_t)v * 8, make_uint4(c[0], c[1], n0, n1));
          if ((lane & 15) == 0) a.xp_scales[(int64_t)r * nb + blk] = s;
        }
      }
    }
    // thread 0 keeps its own copy of token t's rows: other threads may refill
    // s_row[buf] for a later token as soon as they pass the barrier
    int rel[MOE_MAX_TOPK];
    if (a.tile_ready && tid == 0) {
#pragma unroll
      for (int k = 0; k < MOE_MAX_TOPK; ++k) rel[k] = k < K ? s_row[buf][k] : -1;
    }
    __syncthreads();  // every row of token t is written (and s_row[buf ^ 1] is filled)
    if (a.tile_ready && tid == 0) {
      fence_acq_rel_gpu();
#pragma unroll
      for (int k = 0; k < MOE_MAX_TOPK; ++k)
        if (rel[k] >= 0) atomic_add_relaxed_gpu(a.tile_ready + rel[k] / kTile, 1u);
    }
    buf ^= 1;
  }

  // ---- padding rows: code 0x00, scale 0 ----
  const int pad_total = s_padpref[E];
  const int Vc = H >> 4;  // 16-byte code vectors per row
  auto pad_row = [&](int q) -> int64_t {
    int lo = 0, hi = E - 1;  // last expert with padpref <= q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_padpref[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return (int64_t)s_off[lo] + s_cnt[lo] + (q - s_padpref[lo]);
  };
  for (int q = blockIdx.x; q < pad_total; q += gridDim.x) {
    const int64_t r = pad_row(q);
    for (int v = tid; v < Vc; v += kQpThreads) st_v4(a.xp + r * H + (int64_t)v * 16, make_uint4(0, 0, 0, 0));
    for (int b = tid; b < nb; b += kQpThreads) a.xp_scales[r * nb + b] = 0.0f;
  }
  if (a.tile_ready && (int)blockIdx.x < pad_total) {
    __syncthreads();  // all of this CTA's padding rows are written
    if (tid == 0) {
      fence_acq_rel_gpu();
      for (int q = blockIdx.x; q < pad_total; q += gridDim.x)
        atomic_add_relaxed_gpu(a.tile_ready + pad_row(q) / kTile, 1u);
    }
  }
}

std::atomic<int> g_occ_qp[moe_host::kMaxCachedDevices];

}  // namespace
}  // namespace moe

extern "C" int moe_dispatch_permute_quant(const void* x, int64_t T, int H, int64_t x_row_stride,
                                          const int32_t* dst_row, int K,
                                          const int32_t* expert_counts,
                                          const int32_t* expert_offsets, int E, void* xp,
                                          float* xp_scales, int64_t P_cap, uint32_t* tile_ready,
                                          int32_t* d_status, void* stream) {
  using namespace moe;
  if (T < 0 || H <= 0 || H % 128 != 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 ||
      E > MOE_MAX_EXPERTS || x_row_stride < H || x_row_stride % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)K > (int64_t)INT32_MAX || P_cap > (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (P_cap < moe_padded_capacity(T, K, E)) return MOE_ERR_CAPACITY;
  if (!xp || !xp_scales || !expert_counts || !expert_offsets || (T > 0 && (!x || !dst_row)))
    return MOE_ERR_INVALID_ARG;
  if (!moe_host::aligned16(xp) || (x && !moe_host::aligned16(x)) || !moe_host::aligned4(xp_scales))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  QuantPermArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.x_stride = x_row_stride;
  a.T = T;
  a.H = H;
  a.K = K;
  a.dst_row = dst_row;
  a.counts = expert_counts;
  a.offsets = expert_offsets;
  a.E = E;
  a.xp = static_cast<uint8_t*>(xp);
  a.xp_scales = xp_scales;
  a.P_cap = P_cap;
  a.tile_ready = tile_ready;
  a.status = d_status;
  const int dev = moe_host::current_device();
  const int bps = moe_host::blocks_per_sm(permute_quant_kernel, kQpThreads, 0, dev, g_occ_qp);
  int64_t grid = (int64_t)moe_host::sm_count(dev) * bps;
  const int64_t need = T + (int64_t)(kTile - 1) * E;
  if (grid > need) grid = need;
  return moe_host::launch(permute_quant_kernel, dim3((unsigned)grid), dim3(kQpThreads), 0,
                          static_cast<cudaStream_t>(stream), a);
}
