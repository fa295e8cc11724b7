// Combine and the two backward calls.
//
// Combine is defined by the torch_npu "npu_moe_distribute_combine" API
// reference (function description): the expert outputs are brought back along
// the dispatch path, multiplied by their expert_scales and summed, and the
// shared-expert output is added without a weight (parameter expert_scales).
// Here the "way back" is the dispatch map itself: out[t] gathers the K rows
// dst_row[t*K + k] of the expert-major buffer.
//
// combine_bwd and dispatch_bwd are the adjoints of the two linear maps
// (combine in y and in the scales; permute = copy of x[t] to K rows).
//
// B200 design.  All three are HBM-bound gathers / scatters of 16-byte
// vectors; there is no contraction to put on tensor cores.
//   * combine / dispatch_bwd: a 256-thread CTA owns a token row; threads
//     0..K-1 fetch the next token's row indices and scales into a second
//     shared buffer while the CTA works on the current one, so index latency
//     stays off the critical path.  Each thread issues all K 16-byte gathers
//     of its column (K*16 bytes in flight per thread) before reducing.  The
//     fp32 reduction runs k = 0..K-1 in order with fma, then adds the shared
//     row, then rounds once.
//   * combine_bwd: a 128-thread CTA owns a token row: it reads grad_out[t]
//     once, gathers the K rows of y, writes the K scaled rows of grad_y
//     (each element the exact product rounded once to bf16) and
//     reduces the K dot products across the CTA in a fixed order
//     (deterministic).  The same CTAs then zero the padding rows of grad_y.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kKBatch = 8;       // gathers issued before reducing

#ifndef MOE_GATHER_CTA_THREADS
#define MOE_GATHER_CTA_THREADS 256
#endif
// resident 256-thread CTAs per SM asked of the register allocator, per
// column and row batch: 4 (64 registers) for one column, fewer as the batch
// holds more loads; a batch of fewer than kKBatch loads (few slots per
// token) leaves registers for 4 CTAs up to two columns, 2 at four
constexpr int gather_min_blocks(int u, int kb) {
  return u * kb < kKBatch ? (u <= 2 ? 4 : 2) : u == 1 ? 4 : u == 2 ? 3 : u == 4 ? 2 : 1;
}
constexpr int kCtaThreads = MOE_GATHER_CTA_THREADS;

// CTA-per-token reduction: threads 0..K-1 fetch the next token's row indices
// and scales while the CTA works on the current token (double-buffered in
// shared memory), so index latency stays off the critical path.  Each thread
// handles kU columns at a time and issues kU * min(K, 8 / kU) 16-byte gathers
// before reducing, so about eight loads are in flight per thread whatever K
// is (kU = 8 / K rounded down to a power of two).  A batch holds kKB rows:
// 8 / kU, or fewer when the token has fewer slots (K itself with one column
// per thread, K rounded up to a power of two with more), so that short
// tokens do not hold registers for rows they lack.
template <bool kScaled, bool kShared, int kU, int kKB>
__global__ void __launch_bounds__(kCtaThreads, gather_min_blocks(kU, kKB))
gather_reduce_cta_kernel(const uint16_t* __restrict__ y, const int32_t* __restrict__ dst_row,
                         const float* __restrict__ scales, const uint16_t* __restrict__ shared,
                         int64_t T, int K, int H, int64_t P_cap, uint16_t* __restrict__ out,
                         int32_t* status) {
  pdl_begin();
  __shared__ int32_t s_row[2][MOE_MAX_TOPK];
  __shared__ float s_sc[2][MOE_MAX_TOPK];
  const int tid = threadIdx.x;
  const int V = H >> 3;
  auto fetch = [&](int64_t t, int buf) {
    if (tid < K && t < T) {
      int r = __ldg(dst_row + t * K + tid);
      if (r != -1 && (r < 0 || (int64_t)r >= P_cap)) {
        record_error(status, MOE_ERR_BOUNDS);
        r = -1;
      }
      s_row[buf][tid] = r;
      s_sc[buf][tid] = kScaled ? __ldg(scales + t * K + tid) : 1.0f;
    }
  };
  int buf = 0;
  fetch(blockIdx.x, 0);
  __syncthreads();
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    fetch(t + gridDim.x, buf ^ 1);
    for (int vb = tid; vb < V; vb += kCtaThreads * kU) {
      float acc[kU][8];
#pragma unroll
      for (int i = 0; i < kU; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.0f;
      // when the row batch leaves registers free, the shared term's vectors
      // go out with the first batch of gathers (they are added after the k
      // loop either way, as the definition orders them)
      constexpr bool kEarlyShared = kShared && kU * kKB < kKBatch;
      uint4 sv[kEarlyShared ? kU : 1];
#pragma unroll
      for (int i = 0; i < (kEarlyShared ? kU : 1); ++i) {
        const int vec = vb + i * kCtaThreads;
        sv[i] = (kEarlyShared && vec < V) ? ld_nc_v4(shared + t * H + (int64_t)vec * 8)
                                          : make_uint4(0, 0, 0, 0);
      }
      for (int kb = 0; kb < K; kb += kKB) {
        uint4 v[kKB][kU];
#pragma unroll
        for (int j = 0; j < kKB; ++j) {
          const int k = kb + j;
          const int r = k < K ? s_row[buf][k] : -1;
#pragma unroll
          for (int i = 0; i < kU; ++i) {
            const int vec = vb + i * kCtaThreads;
            v[j][i] = (r >= 0 && vec < V) ? ld_nc_v4(y + (int64_t)r * H + (int64_t)vec * 8)
                                          : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int j = 0; j < kKB; ++j) {
          const int k = kb + j;
          const int r = k < K ? s_row[buf][k] : -1;
          if (r < 0) continue;  // an unplaced slot contributes nothing
          const float sk = s_sc[buf][k];
#pragma unroll
          for (int i = 0; i < kU; ++i) {
            const uint32_t w[4] = {v[j][i].x, v[j][i].y, v[j][i].z, v[j][i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (kScaled) {
                acc[i][2 * q] = fmaf(sk, bf16_lo(w[q]), acc[i][2 * q]);
                acc[i][2 * q + 1] = fmaf(sk, bf16_hi(w[q]), acc[i][2 * q + 1]);
              } else {
                acc[i][2 * q] = __fadd_rn(acc[i][2 * q], bf16_lo(w[q]));
                acc[i][2 * q + 1] = __fadd_rn(acc[i][2 * q + 1], bf16_hi(w[q]));
              }
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kU; ++i) {
        const int vec = vb + i * kCtaThreads;
        if (vec >= V) continue;
        if (kShared) {
          const uint4 sh = kEarlyShared ? sv[kEarlyShared ? i : 0]
                                        : ld_nc_v4(shared + t * H + (int64_t)vec * 8);
          const uint32_t w[4] = {sh.x, sh.y, sh.z, sh.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[i][2 * q] = __fadd_rn(acc[i][2 * q], bf16_lo(w[q]));
            acc[i][2 * q + 1] = __fadd_rn(acc[i][2 * q + 1], bf16_hi(w[q]));
          }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[i][0], acc[i][1]);
        o.y = pack_bf16x2(acc[i][2], acc[i][3]);
        o.z = pack_bf16x2(acc[i][4], acc[i][5]);
        o.w = pack_bf16x2(acc[i][6], acc[i][7]);
        st_v4(out + t * H + (int64_t)vec * 8, o);
      }
    }
    __syncthreads();
    buf ^= 1;
  }
}

// s * g as an fp32 value whose round-to-nearest-even bf16 conversion equals
// the conversion of the exact product (one rounding, as the definition of
// grad_y asks).  The fp32 product p = RN32(s * g) is rounded the same way as
// the exact product unless p sits exactly on a midpoint between two bf16
// values (low 16 bits 0x8000): RN32 is monotone and every bf16 midpoint is an
// fp32 value, so otherwise p and the exact product lie on the same side of
// every midpoint.  On a midpoint reached by rounding, the exact product
// (24 + 8 significant bits, so exact in fp64) tells on which side it lies
// and p moves one fp32 ulp toward it, off the tie.  The caller tests eight
// products at once and calls this only for a vector that holds a midpoint
// (for random data about one vector in 8192).
__device__ __forceinline__ float scaled_for_bf16(float s, float g) {
  const float p = __fmul_rn(s, g);
  const uint32_t b = __float_as_uint(p);
  if ((b & 0xFFFFu) != 0x8000u) return p;
  const double v = (double)s * (double)g;
  const double pd = (double)p;
  if (v == pd) return p;
  return __uint_as_float(fabs(v) > fabs(pd) ? b + 1u : b - 1u);
}

#ifndef MOE_BWD_THREADS
#define MOE_BWD_THREADS 128
#endif
constexpr int kBwdThreads = MOE_BWD_THREADS;
constexpr int kBwdWarps = kBwdThreads / 32;

// resident CTAs per SM asked of the register allocator, per column batch
constexpr int bwd_min_blocks(int u) { return u == 8 ? 3 : u == 2 ? 4 : 5; }
// most slots a token can have for a column batch: the launch picks kU >= 2
// only when K <= 8 / kU (gather_u), so the dot products need no more
__host__ __device__ constexpr int bwd_max_k(int u) { return u == 1 ? MOE_MAX_TOPK : 8 / u; }

template <int kU>
__global__ void __launch_bounds__(kBwdThreads, bwd_min_blocks(kU))
combine_bwd_kernel(const uint16_t* __restrict__ g, const uint16_t* __restrict__ y,
                   const float* __restrict__ scales, const int32_t* __restrict__ dst_row,
                   const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                   int E, int64_t T, int K, int H, int64_t P_cap,
                   uint16_t* __restrict__ grad_y, float* __restrict__ grad_s,
                   int32_t* status) {
  pdl_begin();
  constexpr int kKB = kKBatch / kU;  // rows per batch
  __shared__ int32_t s_row[2][MOE_MAX_TOPK];
  __shared__ float s_sc[2][MOE_MAX_TOPK];
  __shared__ float s_part[kBwdWarps][MOE_MAX_TOPK];
  __shared__ int32_t s_padpref[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_pad_base[MOE_MAX_EXPERTS];
  __shared__ int32_t s_pad[MOE_MAX_EXPERTS];
  __shared__ int32_t s_warp[kBwdWarps];
  __shared__ int s_bad;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int V = H >> 3;
  auto fetch = [&](int64_t t, int buf) {
    if (tid < K && t < T) {
      int r = __ldg(dst_row + t * K + tid);
      if (r != -1 && (r < 0 || (int64_t)r >= P_cap)) {
        record_error(status, MOE_ERR_BOUNDS);
        r = -1;
      }
      s_row[buf][tid] = r;
      s_sc[buf][tid] = __ldg(scales + t * K + tid);
    }
  };
  int buf = 0;
  fetch(blockIdx.x, 0);
  __syncthreads();

  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    fetch(t + gridDim.x, buf ^ 1);
    const int* rows = s_row[buf];
    const float* scs = s_sc[buf];
    constexpr int kMaxK = bwd_max_k(kU);
    float dot[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) dot[k] = 0.0f;

    for (int vb = tid; vb < V; vb += kBwdThreads * kU) {
      float gf[kU][8];
#pragma unroll
      for (int i = 0; i < kU; ++i) {
        const int vec = vb + i * kBwdThreads;
        const uint4 gv = vec < V ? ld_nc_v4(g + t * H + (int64_t)vec * 8) : make_uint4(0, 0, 0, 0);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          gf[i][2 * q] = bf16_lo(gw[q]);
          gf[i][2 * q + 1] = bf16_hi(gw[q]);
        }
      }
#pragma unroll
      for (int kb = 0; kb < kMaxK; kb += kKB) {
        if (kb >= K) break;
        uint4 yv[kKB][kU];
#pragma unroll
        for (int j = 0; j < kKB; ++j) {
          const int k = kb + j;
          const int r = k < K ? rows[k] : -1;
#pragma unroll
          for (int i = 0; i < kU; ++i) {
            const int vec = vb + i * kBwdThreads;
            yv[j][i] = (r >= 0 && vec < V) ? ld_nc_v4(y + (int64_t)r * H + (int64_t)vec * 8)
                                           : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int j = 0; j < kKB; ++j) {
          const int k = kb + j;
          const int r = k < K ? rows[k] : -1;
          if (r < 0) continue;
          const float sk = scs[k];
          float d = dot[k];
#pragma unroll
          for (int i = 0; i < kU; ++i) {
            const int vec = vb + i * kBwdThreads;
            if (vec >= V) continue;
            const uint32_t yw[4] = {yv[j][i].x, yv[j][i].y, yv[j][i].z, yv[j][i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              d = fmaf(gf[i][2 * q], bf16_lo(yw[q]), d);
              d = fmaf(gf[i][2 * q + 1], bf16_hi(yw[q]), d);
            }
            float pr[8];
            bool tie = false;  // an fp32 product on a bf16 midpoint: about 1 vector in 8192
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              pr[q] = __fmul_rn(sk, gf[i][q]);
              tie |= (__float_as_uint(pr[q]) & 0xFFFFu) == 0x8000u;
            }
            if (tie) {
#pragma unroll
              for (int q = 0; q < 8; ++q) pr[q] = scaled_for_bf16(sk, gf[i][q]);
            }
            uint4 o;
            o.x = pack_bf16x2(pr[0], pr[1]);
            o.y = pack_bf16x2(pr[2], pr[3]);
            o.z = pack_bf16x2(pr[4], pr[5]);
            o.w = pack_bf16x2(pr[6], pr[7]);
            st_v4(grad_y + (int64_t)r * H + (int64_t)vec * 8, o);
          }
          dot[k] = d;
        }
      }
    }

    // fixed-order reduction of the K dot products over the CTA
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
      if (k >= K) break;
      float d = dot[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      if (lane == 0) s_part[warp][k] = d;
    }
    __syncthreads();  // partial sums ready; s_row[buf ^ 1] filled
    if (tid < K) {
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kBwdWarps; ++w) sum += s_part[w][tid];
      grad_s[t * K + tid] = rows[tid] >= 0 ? sum : 0.0f;
    }
    __syncthreads();  // s_part and s_row[buf] free for reuse
    buf ^= 1;
  }

  // ---- zero the padding rows (below P) of grad_y ----
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int e = tid; e < E; e += kBwdThreads) {
    const int c = __ldg(counts + e);
    const int pad = (__ldg(offsets + e + 1) - __ldg(offsets + e)) - c;
    const bool ok = pad >= 0 && pad < kTile && c >= 0;
    if (!ok) s_bad = 1;
    s_pad_base[e] = __ldg(offsets + e) + c;
    s_pad[e] = ok ? pad : 0;
  }
  __syncthreads();
  block_exclusive_scan(s_pad, E, s_padpref, s_warp);
  if (s_bad || (int64_t)__ldg(offsets + E) > P_cap) {
    if (tid == 0) record_error(status, MOE_ERR_BOUNDS);
    return;
  }
  const int pad_total = s_padpref[E];
  for (int q = blockIdx.x; q < pad_total; q += gridDim.x) {
    int lo = 0, hi = E - 1;  // last expert with padpref <= q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_padpref[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int64_t r = (int64_t)s_pad_base[lo] + (q - s_padpref[lo]);
    for (int vec = tid; vec < V; vec += kBwdThreads)
      st_v4(grad_y + r * H + (int64_t)vec * 8, make_uint4(0, 0, 0, 0));
  }
}

// occupancy cache per (caller, kU, kKB): caller * 40 + log2(kU) * 10 + kKB
std::atomic<int> g_occ_comb[120][moe_host::kMaxCachedDevices];
std::atomic<int> g_occ_bwd[4][moe_host::kMaxCachedDevices];

// kU = columns per thread per batch: 8 / K rounded down to a power of two,
// and no more than the row has columns for the CTA (V / threads).
inline int gather_u(int K, int V, int threads) {
  int u = K <= 1 ? 8 : K == 2 ? 4 : K <= 4 ? 2 : 1;
  while (u > 1 && u * threads > V) u >>= 1;
  return u;
}

constexpr int log2_small(int v) { return v >= 8 ? 3 : v >= 4 ? 2 : v >= 2 ? 1 : 0; }

template <bool kScaled, bool kShared, int kU, int kKB>
int launch_gather_u(int caller, const uint16_t* y, const int32_t* dst_row, const float* scales,
                    const uint16_t* shared, int64_t T, int K, int H, int64_t P_cap,
                    uint16_t* out, int32_t* status, cudaStream_t s) {
  const int dev = moe_host::current_device();
  auto kern = gather_reduce_cta_kernel<kScaled, kShared, kU, kKB>;
  const int slot = caller * 40 + log2_small(kU) * 10 + kKB;
  const int bps = moe_host::blocks_per_sm(kern, kCtaThreads, 0, dev, g_occ_comb[slot]);
  int64_t grid = (int64_t)moe_host::sm_count(dev) * bps;
  if (grid > T) grid = T;
  if (grid < 1) grid = 1;
  return moe_host::launch(kern, dim3((unsigned)grid), dim3(kCtaThreads), 0, s, y, dst_row, scales,
                          shared, T, K, H, P_cap, out, status);
}

// the row batch: 8 / kU rows, or fewer when K is smaller: K itself for one
// column per thread, K rounded up to a power of two for more
template <bool kScaled, bool kShared, int kU>
int launch_gather_rows(int caller, const uint16_t* y, const int32_t* dst_row,
                       const float* scales, const uint16_t* shared, int64_t T, int K, int H,
                       int64_t P_cap, uint16_t* out, int32_t* status, cudaStream_t s) {
  constexpr int kFull = kKBatch / kU;
  if constexpr (kU == 1) {
    switch (K < kFull ? K : kFull) {
      case 7:
        return launch_gather_u<kScaled, kShared, 1, 7>(caller, y, dst_row, scales, shared, T, K,
                                                       H, P_cap, out, status, s);
      case 6:
        return launch_gather_u<kScaled, kShared, 1, 6>(caller, y, dst_row, scales, shared, T, K,
                                                       H, P_cap, out, status, s);
      case 5:
        return launch_gather_u<kScaled, kShared, 1, 5>(caller, y, dst_row, scales, shared, T, K,
                                                       H, P_cap, out, status, s);
      case 3:
        return launch_gather_u<kScaled, kShared, 1, 3>(caller, y, dst_row, scales, shared, T, K,
                                                       H, P_cap, out, status, s);
      default:
        break;  // 1, 2, 4 and 8 below
    }
  }
  int kb = 1;
  while (kb < K && kb < kFull) kb <<= 1;
  if constexpr (kFull >= 8) {
    if (kb == 4)
      return launch_gather_u<kScaled, kShared, kU, 4>(caller, y, dst_row, scales, shared, T, K, H,
                                                      P_cap, out, status, s);
  }
  if constexpr (kFull >= 4) {
    if (kb == 2)
      return launch_gather_u<kScaled, kShared, kU, 2>(caller, y, dst_row, scales, shared, T, K, H,
                                                      P_cap, out, status, s);
  }
  if constexpr (kFull >= 2) {
    if (kb == 1)
      return launch_gather_u<kScaled, kShared, kU, 1>(caller, y, dst_row, scales, shared, T, K, H,
                                                      P_cap, out, status, s);
  }
  return launch_gather_u<kScaled, kShared, kU, kFull>(caller, y, dst_row, scales, shared, T, K, H,
                                                      P_cap, out, status, s);
}

template <bool kScaled, bool kShared>
int launch_gather(int caller, const uint16_t* y, const int32_t* dst_row, const float* scales,
                  const uint16_t* shared, int64_t T, int K, int H, int64_t P_cap, uint16_t* out,
                  int32_t* status, cudaStream_t s) {
  switch (gather_u(K, H >> 3, kCtaThreads)) {
    case 8:
      return launch_gather_rows<kScaled, kShared, 8>(caller, y, dst_row, scales, shared, T, K, H,
                                                     P_cap, out, status, s);
    case 4:
      return launch_gather_rows<kScaled, kShared, 4>(caller, y, dst_row, scales, shared, T, K, H,
                                                     P_cap, out, status, s);
    case 2:
      return launch_gather_rows<kScaled, kShared, 2>(caller, y, dst_row, scales, shared, T, K, H,
                                                     P_cap, out, status, s);
    default:
      return launch_gather_rows<kScaled, kShared, 1>(caller, y, dst_row, scales, shared, T, K, H,
                                                     P_cap, out, status, s);
  }
}

template <int kU>
int launch_bwd(int slot, const uint16_t* g, const uint16_t* y, const float* scales,
               const int32_t* dst_row, const int32_t* counts, const int32_t* offsets, int E,
               int64_t T, int K, int H, int64_t P_cap, uint16_t* grad_y, float* grad_s,
               int32_t* status, cudaStream_t s) {
  const int dev = moe_host::current_device();
  auto kern = combine_bwd_kernel<kU>;
  const int bps = moe_host::blocks_per_sm(kern, kBwdThreads, 0, dev, g_occ_bwd[slot]);
  int64_t grid = (int64_t)moe_host::sm_count(dev) * bps;
  const int64_t need = T + (int64_t)(kTile - 1) * E;
  if (grid > need) grid = need;
  return moe_host::launch(kern, dim3((unsigned)grid), dim3(kBwdThreads), 0, s, g, y, scales,
                          dst_row, counts, offsets, E, T, K, H, P_cap, grad_y, grad_s, status);
}

int check_rows_args(const void* y, const int32_t* dst_row, int64_t T, int K, int H,
                    int64_t P_cap, const void* out) {
  if (T < 0 || K < 1 || K > MOE_MAX_TOPK || H <= 0 || H % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)K > (int64_t)INT32_MAX || P_cap < 0 || P_cap > (int64_t)INT32_MAX)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!y || !dst_row || !out)) return MOE_ERR_INVALID_ARG;
  if ((y && !moe_host::aligned16(y)) || (out && !moe_host::aligned16(out)))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" int moe_combine(const void* y, const int32_t* dst_row, const float* scales,
                           const void* shared_x, int64_t T, int K, int H, int64_t P_cap,
                           void* out, int32_t* d_status, void* stream) {
  using namespace moe;
  int st = check_rows_args(y, dst_row, T, K, H, P_cap, out);
  if (st != MOE_OK) return st;
  if (T > 0 && !scales) return MOE_ERR_INVALID_ARG;
  if (shared_x && !moe_host::aligned16(shared_x)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t* yy = static_cast<const uint16_t*>(y);
  uint16_t* o = static_cast<uint16_t*>(out);
  if (shared_x)
    return launch_gather<true, true>(0, yy, dst_row, scales,
                                     static_cast<const uint16_t*>(shared_x), T, K, H, P_cap, o,
                                     d_status, s);
  return launch_gather<true, false>(1, yy, dst_row, scales, nullptr, T, K, H, P_cap, o,
                                    d_status, s);
}

extern "C" int moe_dispatch_bwd(const void* grad_xp, const int32_t* dst_row, int64_t T, int K,
                                int H, int64_t P_cap, void* grad_x, int32_t* d_status,
                                void* stream) {
  using namespace moe;
  int st = check_rows_args(grad_xp, dst_row, T, K, H, P_cap, grad_x);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  return launch_gather<false, false>(2, static_cast<const uint16_t*>(grad_xp), dst_row, nullptr,
                                     nullptr, T, K, H, P_cap, static_cast<uint16_t*>(grad_x),
                                     d_status, static_cast<cudaStream_t>(stream));
}

extern "C" int moe_combine_bwd(const void* grad_out, const void* y, const float* scales,
                               const int32_t* dst_row, const int32_t* expert_counts,
                               const int32_t* expert_offsets, int E, int64_t T, int K, int H,
                               int64_t P_cap, void* grad_y, float* grad_scales,
                               int32_t* d_status, void* stream) {
  using namespace moe;
  int st = check_rows_args(y, dst_row, T, K, H, P_cap, grad_y);
  if (st != MOE_OK) return st;
  if (E < 1 || E > MOE_MAX_EXPERTS || !expert_counts || !expert_offsets ||
      (P_cap > 0 && !grad_y))
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!grad_out || !scales || !grad_scales)) return MOE_ERR_INVALID_ARG;
  if (grad_out && !moe_host::aligned16(grad_out)) return MOE_ERR_INVALID_ARG;
  if (!moe_host::aligned16(grad_y)) return MOE_ERR_INVALID_ARG;
  if (P_cap < moe_padded_capacity(T, K, E)) return MOE_ERR_CAPACITY;
  if (T == 0) return MOE_OK;  // P = 0: no rows to write
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t* go = static_cast<const uint16_t*>(grad_out);
  const uint16_t* yy = static_cast<const uint16_t*>(y);
  uint16_t* gy = static_cast<uint16_t*>(grad_y);
  switch (gather_u(K, H >> 3, kBwdThreads)) {
    case 8:
      return launch_bwd<8>(0, go, yy, scales, dst_row, expert_counts, expert_offsets, E, T, K, H,
                           P_cap, gy, grad_scales, d_status, s);
    case 4:
      return launch_bwd<4>(1, go, yy, scales, dst_row, expert_counts, expert_offsets, E, T, K, H,
                           P_cap, gy, grad_scales, d_status, s);
    case 2:
      return launch_bwd<2>(2, go, yy, scales, dst_row, expert_counts, expert_offsets, E, T, K, H,
                           P_cap, gy, grad_scales, d_status, s);
    default:
      return launch_bwd<1>(3, go, yy, scales, dst_row, expert_counts, expert_offsets, E, T, K, H,
                           P_cap, gy, grad_scales, d_status, s);
  }
}
