// E4M3 quantisation with one fp32 scale per 128 channels: the input side of
// the FP8 dispatch (codes travel with their per-block scales; DeepEP pull
// request "Intra-node compute compensation ...", Testing: the FP8 dispatch
// path).  s = amax / 448 in fp32 (1 when the block is all zero), codes =
// E4M3(x / s) with IEEE fp32 division, round to nearest even, saturating.
//
// A half-warp owns one (token, 128-channel) block: 16 lanes x 8 bf16 = one
// 256-byte row segment read with 16-byte loads, amax reduced by shuffles,
// 8 codes per lane written as one 8-byte store, one scale per block.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQThreads = 256;

__global__ void __launch_bounds__(kQThreads)
quantize_e4m3_kernel(const uint16_t* __restrict__ x, int64_t T, int H, int64_t stride,
                     uint8_t* __restrict__ q, float* __restrict__ qs) {
  pdl_begin();
  const int nb = H / 128;
  const int64_t n_units = T * nb;
  const int lane = threadIdx.x & 31, sub = lane & 15;
  const int64_t hw0 = ((int64_t)blockIdx.x * kQThreads + threadIdx.x) >> 4;  // half-warp id
  const int64_t n_hw = ((int64_t)gridDim.x * kQThreads) >> 4;
  // both half-warps of a warp run the same number of iterations (shuffles use the full mask)
  const int64_t hw_even = hw0 & ~(int64_t)1;
  for (int64_t base = hw_even; base < n_units; base += n_hw) {
    const int64_t u = base + (hw0 & 1);
    const bool active = u < n_units;
    float f[8];
    float amax = 0.0f;
    int64_t t = 0, b = 0;
    if (active) {
      t = u / nb;
      b = u - t * nb;
      const uint4 v = ld_nc_v4(x + t * stride + b * 128 + sub * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o, 16));
    if (!active) continue;
    const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 pr = make_float2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
      const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
      if (i < 2) lo |= c2 << (16 * i);
      else hi |= c2 << (16 * (i - 2));
    }
    *reinterpret_cast<uint2*>(q + t * H + b * 128 + sub * 8) = make_uint2(lo, hi);
    if (sub == 0) qs[t * nb + b] = s;
  }
}

}  // namespace
}  // namespace moe

extern "C" int moe_quantize_e4m3(const void* x, int64_t T, int H, int64_t x_row_stride, void* q,
                                 float* q_scales, int32_t* d_status, void* stream) {
  (void)d_status;
  if (T < 0 || H <= 0 || H % 128 != 0 || x_row_stride < H || x_row_stride % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !q || !q_scales)) return MOE_ERR_INVALID_ARG;
  if ((x && !moe_host::aligned16(x)) || (q && (reinterpret_cast<uintptr_t>(q) & 7u)) ||
      (q_scales && !moe_host::aligned4(q_scales)))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const int dev = moe_host::current_device();
  const int64_t units = T * (H / 128);
  int64_t grid = (units * 16 + moe::kQThreads - 1) / moe::kQThreads;
  const int64_t cap = (int64_t)moe_host::sm_count(dev) * 8;
  if (grid > cap) grid = cap;
  return moe_host::launch(moe::quantize_e4m3_kernel, dim3((unsigned)grid), dim3(moe::kQThreads), 0,
                          static_cast<cudaStream_t>(stream), static_cast<const uint16_t*>(x), T, H,
                          x_row_stride, static_cast<uint8_t*>(q), q_scales);
}
