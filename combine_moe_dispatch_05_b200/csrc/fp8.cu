// E4M3 quantisation with one fp32 scale per 128 channels: the input side of
// the FP8 dispatch (codes travel with their per-block scales; DeepEP pull
// request "Intra-node compute compensation ...", Testing: the FP8 dispatch
// path).  s = amax / 448 in fp32 (1 when the block is all zero), codes =
// E4M3(x / s) with the fp32 quotient rounded to nearest even (the IEEE
// division's result, formed with one reciprocal per block and Markstein's
// correction step on packed pairs: quotient_pair), converted with round to
// nearest even, saturating.
//
// A 256-thread CTA owns a token row (grid-stride over tokens): thread i holds
// 32-byte units i, i+256, ... of the bf16 row (16 channels each, one 256-bit
// load, or two 16-byte loads when x is not 32-byte aligned), two at a time
// with both loads issued before any math.  The 8 lanes of a group cover one
// 128-channel block, reduce its amax with shuffles and convert their 16
// channels each, so the block's scale and reciprocal are formed once per 16
// channels; each lane stores its 16 codes (one 16-byte store when q is
// 16-byte aligned, else two 8-byte stores), and one lane per block writes the
// scale.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQThreads = 256;
constexpr int kQU = 2;  // 32-byte units per thread per batch

// Pairs of fp32 values in one 64-bit register pair, for the sm_100 packed
// arithmetic (mul/fma .rn.f32x2: two IEEE operations, each rounded to
// nearest, in one instruction).
__device__ __forceinline__ uint64_t pack_f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ void unpack_f2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

__device__ __forceinline__ uint64_t mul_f2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Quotients x / s rounded to nearest even, for a divisor s shared by a
// 128-channel block, two at a time.  Markstein's theorem (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; also Muller et al., Handbook of
// Floating-Point Arithmetic, the section on division with an FMA): with r
// the correctly rounded reciprocal RN(1/s) and q0 = RN(x*r), the residual
// x - s*q0 is exact in one FMA and RN(q0 + (x - s*q0)*r) is RN(x/s), given
// operands and residual away from underflow.  The pair holds -x (not x) and
// nr = -r: q0 = RN((-x)*(-r)) is the same product, the FMA forms the
// negated residual s*q0 - x, and adding it times -r gives the same sum;
// written this way a zero x keeps its sign (the last addition is -0 + -0
// for x = -0) with no compare or select.  A scale below 2^-100 is first
// multiplied, with the x, by m = 2^64: exact (powers of two, no overflow
// since |x| <= 448 s), and the quotients are unchanged; then s >= 2^-85, so
// every quotient that an E4M3 code can tell apart (above 2^-24) has
// operands, product and residual in the normal range.
__device__ __forceinline__ void quotient_pair(float nx0, float nx1, uint64_t m2, uint64_t s2,
                                              uint64_t nr2, float& q0, float& q1) {
  const uint64_t x2 = mul_f2(pack_f2(nx0, nx1), m2);    // -x * m
  const uint64_t p2 = mul_f2(x2, nr2);                  // RN(x * r)
  const uint64_t e2 = fma_f2(p2, s2, x2);               // s*p - x, exact
  unpack_f2(fma_f2(e2, nr2, p2), q0, q1);               // RN(p + (x - s*p) * r)
}

// 32 bytes of global memory in one load (sm_100: 256-bit loads), through
// the non-coherent path without allocating in L1
__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&w)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                 "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}

__global__ void __launch_bounds__(kQThreads)
quantize_e4m3_kernel(const uint16_t* __restrict__ x, int64_t T, int H, int64_t stride,
                     uint8_t* __restrict__ q, float* __restrict__ qs, int vec16, int x32) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const unsigned grp_mask = 0xFFu << (lane & 24);  // the 8 lanes of one 128-channel block
  const int U = H >> 4;   // 32-byte units (16 channels) per row
  const int nb = H >> 7;  // 128-channel blocks per row
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t* xr = x + t * stride;
    uint8_t* qr = q + t * H;
    for (int ub = threadIdx.x; ub < U; ub += kQThreads * kQU) {  // U % 8 == 0: groups stay whole
      uint32_t d[kQU][8];
#pragma unroll
      for (int i = 0; i < kQU; ++i) {
        const int u = ub + i * kQThreads;
        if (u < U) {
          if (x32) {
            ld_nc_v8(xr + (int64_t)u * 16, d[i]);
          } else {
            const uint4 a = ld_nc_v4(xr + (int64_t)u * 16);
            const uint4 b = ld_nc_v4(xr + (int64_t)u * 16 + 8);
            d[i][0] = a.x; d[i][1] = a.y; d[i][2] = a.z; d[i][3] = a.w;
            d[i][4] = b.x; d[i][5] = b.y; d[i][6] = b.z; d[i][7] = b.w;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kQU; ++i) {
        const int u = ub + i * kQThreads;
        if (u >= U) break;  // uniform across each 8-lane group
        // the negated values: |-x| gives amax, and the quotient step takes -x
        float f[16];
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t w = d[i][k] ^ 0x80008000u;
          f[2 * k] = bf16_lo(w);
          f[2 * k + 1] = bf16_hi(w);
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(f[k]));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(grp_mask, amax, o, 8));
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        const float m = s < 0x1p-100f ? 0x1p64f : 1.0f;
        const float sm = __fmul_rn(s, m);
        const float nr = -__frcp_rn(sm);
        const uint64_t m2 = pack_f2(m, m), s2 = pack_f2(sm, sm), nr2 = pack_f2(nr, nr);
        uint32_t c[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float2 pr;
          quotient_pair(f[2 * k], f[2 * k + 1], m2, s2, nr2, pr.x, pr.y);
          const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
          c[k >> 1] |= c2 << (16 * (k & 1));
        }
        if (vec16) {
          st_v4(qr + (int64_t)u * 16, make_uint4(c[0], c[1], c[2], c[3]));
        } else {
          *reinterpret_cast<uint2*>(qr + (int64_t)u * 16) = make_uint2(c[0], c[1]);
          *reinterpret_cast<uint2*>(qr + (int64_t)u * 16 + 8) = make_uint2(c[2], c[3]);
        }
        if ((lane & 7) == 0) qs[t * nb + (u >> 3)] = s;
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
  const int x32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && x_row_stride % 16 == 0 ? 1 : 0;
  return moe_host::launch(moe::quantize_e4m3_kernel, dim3((unsigned)grid), dim3(moe::kQThreads), 0,
                          static_cast<cudaStream_t>(stream), static_cast<const uint16_t*>(x), T, H,
                          x_row_stride, static_cast<uint8_t*>(q), q_scales, vec16, x32);
}
