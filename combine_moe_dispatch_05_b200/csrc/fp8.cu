// E4M3 quantisation with one fp32 scale per 128 channels: the input side of
// the FP8 dispatch (codes travel with their per-block scales; DeepEP pull
// request "Intra-node compute compensation ...", Testing: the FP8 dispatch
// path).  s = amax / 448 in fp32 (1 when the block is all zero), codes =
// E4M3(x / s) with the fp32 quotient rounded to nearest even (the IEEE
// division's result, formed with one reciprocal per block and Markstein's
// correction step: div8_by_scale), converted with round to nearest even,
// saturating.
//
// A 256-thread CTA owns a token row (grid-stride over tokens): thread i holds
// 16-byte vectors i, i+256, ... of the bf16 row, four at a time with all four
// loads issued before any math.  The 16 lanes of a half-warp cover one
// 128-channel block, reduce its amax with shuffles and convert their 8
// channels each; pairs of lanes merge their codes into one 16-byte store when
// q is 16-byte aligned (else each lane stores its 8 codes), and one lane per
// block writes the scale.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQThreads = 256;
constexpr int kQU = 4;  // columns per thread per batch

// x / s rounded to nearest even, for a divisor s shared by many x (one
// 128-channel block's scale).  r must be the correctly rounded reciprocal
// RN(1/s) (the __frcp_rn intrinsic), computed once per block.  Markstein's
// theorem (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also Muller et
// al., Handbook of Floating-Point Arithmetic, the section on division with
// an FMA): if r is within half an ulp of 1/s and q0 = RN(x*r) within one ulp
// of x/s, then with the exact residual e = x - s*q0 (one FMA), RN(q0 + e*r)
// is RN(x/s).  It needs the operands and the residual away from underflow,
// which div8_by_scale arranges.  A zero residual returns q0 as it is, which
// keeps the sign of a zero quotient.
__device__ __forceinline__ float div_by_shared(float x, float s, float r) {
  const float q0 = __fmul_rn(x, r);
  const float e = __fmaf_rn(-q0, s, x);
  return e == 0.0f ? q0 : __fmaf_rn(e, r, q0);
}

// The eight quotients f[k] / s of one 16-byte bf16 vector, each rounded to
// nearest even as an IEEE division would round it, for a block scale
// s = amax / 448 with |f[k]| <= amax.  A scale below 2^-100 is first
// multiplied, with the f[k], by 2^64: exact (powers of two, no overflow since
// |f| <= 448 s), and the quotients are unchanged.  Then s >= 2^-85, so every
// quotient that an E4M3 code can tell apart (above 2^-24) has an operand,
// product and residual in the normal range, where Markstein's step holds.
__device__ __forceinline__ void div8_by_scale(const float* f, float s, float* out) {
  const float m = s < 0x1p-100f ? 0x1p64f : 1.0f;
  const float ss = __fmul_rn(s, m);
  const float r = __frcp_rn(ss);
#pragma unroll
  for (int k = 0; k < 8; ++k) out[k] = div_by_shared(__fmul_rn(f[k], m), ss, r);
}

__global__ void __launch_bounds__(kQThreads)
quantize_e4m3_kernel(const uint16_t* __restrict__ x, int64_t T, int H, int64_t stride,
                     uint8_t* __restrict__ q, float* __restrict__ qs, int vec16) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const unsigned half_mask = 0xFFFFu << (lane & 16);
  const int V = H >> 3;   // 16-byte bf16 vectors per row
  const int nb = H >> 7;  // 128-channel blocks per row
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t* xr = x + t * stride;
    uint8_t* qr = q + t * H;
    for (int vb = threadIdx.x; vb < V; vb += kQThreads * kQU) {  // V % 16 == 0: half-warps stay whole
      uint4 d[kQU];
#pragma unroll
      for (int i = 0; i < kQU; ++i) {
        const int v = vb + i * kQThreads;
        d[i] = v < V ? ld_nc_v4(xr + (int64_t)v * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kQU; ++i) {
        const int v = vb + i * kQThreads;
        if (v >= V) break;  // uniform across the half-warp
        const uint32_t w[4] = {d[i].x, d[i].y, d[i].z, d[i].w};
        float f[8];
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          f[2 * k] = bf16_lo(w[k]);
          f[2 * k + 1] = bf16_hi(w[k]);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(f[k]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(half_mask, amax, o, 16));
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        float qf[8];
        div8_by_scale(f, s, qf);
        uint32_t c[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 pr = make_float2(qf[2 * k], qf[2 * k + 1]);
          const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
          c[k >> 1] |= c2 << (16 * (k & 1));
        }
        if (vec16) {
          const uint32_t n0 = __shfl_down_sync(half_mask, c[0], 1, 16);
          const uint32_t n1 = __shfl_down_sync(half_mask, c[1], 1, 16);
          if ((lane & 1) == 0) st_v4(qr + (int64_t)v * 8, make_uint4(c[0], c[1], n0, n1));
        } else {
          *reinterpret_cast<uint2*>(qr + (int64_t)v * 8) = make_uint2(c[0], c[1]);
        }
        if ((lane & 15) == 0) qs[t * nb + (v >> 4)] = s;
      }
    }
  }
}

std::atomic<int> g_occ_q[moe_host::kMaxCachedDevices];

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
  const int bps =
      moe_host::blocks_per_sm(moe::quantize_e4m3_kernel, moe::kQThreads, 0, dev, moe::g_occ_q);
  int64_t grid = (int64_t)moe_host::sm_count(dev) * bps;
  if (grid > T) grid = T;
  const int vec16 = moe_host::aligned16(q) ? 1 : 0;
  return moe_host::launch(moe::quantize_e4m3_kernel, dim3((unsigned)grid), dim3(moe::kQThreads), 0,
                          static_cast<cudaStream_t>(stream), static_cast<const uint16_t*>(x), T, H,
                          x_row_stride, static_cast<uint8_t*>(q), q_scales, vec16);
}
