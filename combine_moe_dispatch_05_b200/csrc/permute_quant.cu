// Fused quantise-on-dispatch: bf16 token rows are quantised to E4M3 with one
// fp32 scale per 128 channels and the codes and scales are written straight
// into the expert-major buffer (the FP8 dispatch path of the DeepEP pull
// request "Intra-node compute compensation + overlap robustness (CUDA719
// fix)", Testing: FP8 dispatch; layout as in the torch_npu
// "npu_moe_distribute_combine" API's expand_x; 128-row M-tile padding from the
// TEMPO summary, section 1).  The result equals quantise-then-permute byte for
// byte, but x is read once and the intermediate codes never touch HBM.
//
// A 128-thread CTA owns a token and works through its row in units of at
// most 8192 channels: thread i holds 16-byte vectors i, i+128, ... of the
// unit's bf16 slice, four at a time with all four loads issued before any
// math; the 16 threads of a half-warp share one 128-channel block, reduce its
// amax with shuffles, divide by s = amax/448 in fp32 and convert with
// saturating round-to-nearest-even.  Codes and scales are staged once in
// shared memory and thread 0 sends them to the K destination rows with bulk
// stores (cp.async.bulk, no multicast), so the K-fold write fan-out costs the
// SM's threads nothing.  Two stage buffers alternate; a stage is rewritten
// only after the stores that read it have finished reading.  A token's rows
// are released on the chunk-completion counters one unit later, once its
// bulk group has completed.  Padding rows get code 0x00 and scale 0.  Where
// a row's scales are not 16-byte aligned (H not a multiple of 512) the
// scales are written with plain stores instead.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQpThreads = 128;
constexpr int kQpU = 4;          // columns per thread per batch
constexpr int kQpChunk = 8192;   // channels per unit (a multiple of 512)
constexpr int kQpStages = 2;     // stage buffers per CTA

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
  int chunk;          // channels per unit: H, or kQpChunk when H is larger
  int stage_bytes;    // chunk codes + chunk/128 scales, rounded up to 16
  int bulk_scales;    // scales go out by bulk store (H % 512 == 0, aligned base)
  uint32_t* work;     // [2] claim counter and done count
  int64_t tokens_per_ticket;
  int64_t pad_per_ticket;
};

__host__ __device__ constexpr int qp_stage_bytes(int chunk) {
  return (chunk + chunk / 32 + 15) / 16 * 16;
}

// Work claiming (TicketStream, first batch of one ticket) and releases, as in
// the token-ordered permute: tickets [0, n_tok) name tpt tokens each, tickets
// [n_tok, n_tok + n_pad) name ppt padding rows each.
// Thread 0 resolves the token after next while the CTA works on the current
// one, so the claim's latency is hidden.  Rows are released in batches: once
// kQRelLag + kQRelBatch bulk groups are unreleased, one completion wait and
// one gpu-scope fence release all but the newest kQRelLag.  The last CTA out
// returns work[0..1] to zero.
constexpr int kQRing = 16;       // tokens whose rows are held (until released)
constexpr int kQRelLag = 4;      // bulk groups left in flight at a release
constexpr int kQRelBatch = 8;    // groups released per completion wait
static_assert(kQRing > kQRelLag + kQRelBatch + 2, "token ring too small for the release lag");

__global__ void __launch_bounds__(kQpThreads, 8) permute_quant_kernel(const QuantPermArgs a) {
  pdl_begin();
  extern __shared__ __align__(128) uint8_t qp_stage[];
  __shared__ int32_t s_row[kQRing][MOE_MAX_TOPK];
  __shared__ int64_t s_tok[kQRing];   // token of local sequence number j % kQRing, -1 = none
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_cnt[MOE_MAX_EXPERTS];
  __shared__ int32_t s_pad[MOE_MAX_EXPERTS];
  __shared__ int32_t s_padpref[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_warp[kQpThreads / 32];
  __shared__ int64_t s_padq;          // padding ticket being processed, -1 = none
  __shared__ int32_t s_rec[kQRelLag + kQRelBatch];  // per unreleased group: its token's slot or -1
  __shared__ int s_bad;

  const int tid = threadIdx.x, lane = tid & 31;
  const int E = a.E, K = a.K, H = a.H;
  const int nb = H >> 7;       // 128-channel blocks per row
  const int CH = a.chunk;
  const int nch = (H + CH - 1) / CH;
  const unsigned half_mask = 0xFFFFu << (lane & 16);
  const int64_t tpt = a.tokens_per_ticket, ppt = a.pad_per_ticket;
  const int64_t n_tok = (a.T + tpt - 1) / tpt;

  __shared__ TicketStream tk;  // used by thread 0 only
  if (tid == 0) {
    s_bad = 0;
    tk.init(a.work, 1);
  }
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
  const bool bad = s_bad || (int64_t)s_off[E] > a.P_cap || s_off[0] != 0;
  if (bad && tid == 0) record_error(a.status, MOE_ERR_BOUNDS);
  const int pad_total = s_padpref[E];
  const int64_t n_tickets = n_tok + ((int64_t)pad_total + ppt - 1) / ppt;

  // ---- thread 0's ticket stream ----
  int64_t tok_cur = 0, tok_end = 0;
  int64_t first_pad_ticket = -1;  // the ticket that ended the token phase
  bool tokens_done = false;
  auto take_ticket = [&]() -> int64_t { return tk.take(n_tickets); };  // thread 0
  auto next_token = [&]() -> int64_t {  // thread 0; -1 when the token tickets are used up
    while (!tokens_done) {
      if (tok_cur < tok_end) return tok_cur++;
      const int64_t k = take_ticket();
      if (k < n_tok) {
        tok_cur = k * tpt;
        tok_end = min(a.T, tok_cur + tpt);
      } else {
        tokens_done = true;
        first_pad_ticket = k;
      }
    }
    return -1;
  };
  if (tid == 0) {
    s_tok[0] = bad ? -1 : next_token();
    s_tok[1] = (bad || s_tok[0] < 0) ? -1 : next_token();
  }
  __syncthreads();

  auto fetch = [&](int64_t t, int slot) {
    if (tid < K && t >= 0) {
      int r = __ldg(a.dst_row + t * K + tid);
      if (r != -1 && (r < 0 || (int64_t)r >= a.P_cap)) {
        record_error(a.status, MOE_ERR_BOUNDS);
        r = -1;
      }
      s_row[slot][tid] = r;
    }
  };
  // thread 0: group bookkeeping for batched releases
  uint32_t n_commit = 0, n_rel = 0;
  auto release_batch = [&](uint32_t keep) {  // thread 0: release all groups but the newest `keep`
    if (keep == 0) bulk_wait_all<0>(); else bulk_wait_all<kQRelLag>();
    fence_proxy_async_global();
    fence_acq_rel_gpu();
    while (n_commit - n_rel > keep) {
      const int32_t slot = s_rec[n_rel % (kQRelLag + kQRelBatch)];
      if (slot >= 0)
        for (int k = 0; k < K; ++k) {
          const int32_t r = s_row[slot][k];
          if (r >= 0) atomic_add_relaxed_gpu(a.tile_ready + r / kTile, 1u);
        }
      ++n_rel;
    }
  };

  fetch(s_tok[0], 0);
  __syncthreads();
  int64_t u = 0;  // units issued by this CTA
  for (int64_t j = 0;; ++j) {
    const int64_t t = s_tok[j % kQRing];
    if (t < 0) break;
    const int slot = (int)(j % kQRing);
    fetch(s_tok[(j + 1) % kQRing], (int)((j + 1) % kQRing));
    if (tid == 0) {  // the token after next
      const int64_t t1 = s_tok[(j + 1) % kQRing];
      s_tok[(j + 2) % kQRing] = t1 < 0 ? -1 : next_token();
    }
    const int32_t* rows = s_row[slot];
    const uint16_t* xr = a.x + t * a.x_stride;
    for (int c = 0; c < nch; ++c, ++u) {
      const int c0 = c * CH;
      const int cl = min(CH, H - c0);
      const int Vn = cl >> 3;  // bf16 vectors in the unit, a multiple of 16
      uint8_t* st_codes = qp_stage + (int)(u % kQpStages) * a.stage_bytes;
      float* st_scl = reinterpret_cast<float*>(st_codes + CH);
      const uint16_t* xc = xr + c0;
      // a half-warp's 16 lanes share one 128-channel block in every column
      for (int vb = tid; vb < Vn; vb += kQpThreads * kQpU) {
        uint4 d[kQpU];
#pragma unroll
        for (int i = 0; i < kQpU; ++i) {
          const int v = vb + i * kQpThreads;
          d[i] = v < Vn ? ld_nc_v4(xc + (int64_t)v * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kQpU; ++i) {
          const int v = vb + i * kQpThreads;
          if (v >= Vn) break;  // uniform across the half-warp
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
          uint32_t cw[2] = {0u, 0u};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 pr = make_float2(__fdiv_rn(f[2 * q], s), __fdiv_rn(f[2 * q + 1], s));
            const uint32_t c2 = (uint32_t)__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
            cw[q >> 1] |= c2 << (16 * (q & 1));
          }
          *reinterpret_cast<uint2*>(st_codes + v * 8) = make_uint2(cw[0], cw[1]);
          if ((lane & 15) == 0) {
            if (a.bulk_scales) {
              st_scl[v >> 4] = s;
            } else {
              for (int k = 0; k < K; ++k)
                if (rows[k] >= 0) a.xp_scales[(int64_t)rows[k] * nb + ((c0 + v * 8) >> 7)] = s;
            }
          }
        }
      }
      fence_proxy_async_shared();  // this thread's stage writes precede the bulk reads
      if (tid == 0) bulk_wait_read<kQpStages - 2>();  // the next unit's stage is free
      __syncthreads();
      if (tid == 0) {
        for (int k = 0; k < K; ++k) {
          const int64_t r = rows[k];
          if (r < 0) continue;
          bulk_store_s2g(a.xp + r * H + c0, st_codes, (uint32_t)cl);
          if (a.bulk_scales)
            bulk_store_s2g(a.xp_scales + r * nb + (c0 >> 7), st_scl, (uint32_t)(cl >> 5));
        }
        bulk_commit();
        s_rec[n_commit % (kQRelLag + kQRelBatch)] = c == nch - 1 ? slot : -1;
        ++n_commit;
        if (a.tile_ready && n_commit - n_rel == (uint32_t)(kQRelLag + kQRelBatch))
          release_batch(kQRelLag);
      }
    }
  }
  if (tid == 0) {
    if (a.tile_ready) release_batch(0);  // the last tokens' rows: written, then released
    else bulk_wait_all<0>();             // stages stay alive until read; rows written
  }

  // ---- padding rows: code 0x00, scale 0, claimed ppt rows at a time ----
  const int Vc = H >> 4;  // 16-byte code vectors per row
  auto pad_row = [&](int q) -> int64_t {
    int lo = 0, hi = E - 1;  // last expert with padpref <= q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_padpref[mid] <= q) lo = mid; else hi = mid - 1;
    }
    return (int64_t)s_off[lo] + s_cnt[lo] + (q - s_padpref[lo]);
  };
  if (tid == 0) s_padq = (!bad && first_pad_ticket >= n_tok && first_pad_ticket < n_tickets)
                             ? first_pad_ticket - n_tok : -1;
  __syncthreads();
  while (true) {
    const int64_t pq = s_padq;
    if (pq < 0) break;
    const int q0 = (int)(pq * ppt), q1 = (int)min((int64_t)pad_total, (pq + 1) * ppt);
    for (int q = q0; q < q1; ++q) {
      const int64_t r = pad_row(q);
      for (int v = tid; v < Vc; v += kQpThreads) st_v4(a.xp + r * H + (int64_t)v * 16, make_uint4(0, 0, 0, 0));
      for (int b = tid; b < nb; b += kQpThreads) a.xp_scales[r * nb + b] = 0.0f;
    }
    __syncthreads();  // every row of the ticket is written (and s_padq read by all)
    if (tid == 0) {
      if (a.tile_ready) {
        fence_acq_rel_gpu();
        for (int q = q0; q < q1;) {  // one add per run inside one expert
          const int64_t r = pad_row(q);
          int lo = 0, hi = E - 1;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_padpref[mid] <= q) lo = mid; else hi = mid - 1;
          }
          const int qe = min(q1, s_padpref[lo + 1]);
          atomic_add_relaxed_gpu(a.tile_ready + r / kTile, (uint32_t)(qe - q));
          q = qe;
        }
      }
      const int64_t k = take_ticket();
      s_padq = (k >= n_tok && k < n_tickets) ? k - n_tok : -1;
    }
    __syncthreads();
  }

  if (tid == 0) finish_claims(a.work);  // the last CTA out returns both words to zero
}

std::atomic<int> g_occ_qp[moe_host::kMaxCachedDevices];

}  // namespace
}  // namespace moe

extern "C" int moe_dispatch_permute_quant(const void* x, int64_t T, int H, int64_t x_row_stride,
                                          const int32_t* dst_row, int K,
                                          const int32_t* expert_counts,
                                          const int32_t* expert_offsets, int E, void* xp,
                                          float* xp_scales, int64_t P_cap, uint32_t* tile_ready,
                                          uint32_t* work, int32_t* d_status, void* stream) {
  using namespace moe;
  if (T < 0 || H <= 0 || H % 128 != 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 ||
      E > MOE_MAX_EXPERTS || x_row_stride < H || x_row_stride % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)K > (int64_t)INT32_MAX || P_cap > (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (P_cap < moe_padded_capacity(T, K, E)) return MOE_ERR_CAPACITY;
  // an empty batch (P_cap = 0) may pass null row buffers
  if ((P_cap > 0 && (!xp || !xp_scales)) || !expert_counts || !expert_offsets ||
      (T > 0 && (!x || !dst_row)))
    return MOE_ERR_INVALID_ARG;
  if (!moe_host::aligned16(xp) || (x && !moe_host::aligned16(x)) || !moe_host::aligned4(xp_scales))
    return MOE_ERR_INVALID_ARG;
  if (!work || !moe_host::aligned4(work)) return MOE_ERR_INVALID_ARG;
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
  a.chunk = H < kQpChunk ? H : kQpChunk;
  a.stage_bytes = qp_stage_bytes(a.chunk);
  a.bulk_scales = (H % 512 == 0 && moe_host::aligned16(xp_scales)) ? 1 : 0;
  a.work = work;
  // a token ticket names about 32 KiB of code writes; a padding ticket 32 rows
  const int64_t tok_bytes = (int64_t)K * H;
  a.tokens_per_ticket = (32768 + tok_bytes - 1) / tok_bytes;
  if (a.tokens_per_ticket > 64) a.tokens_per_ticket = 64;
  a.pad_per_ticket = 32;
  const size_t dyn = (size_t)kQpStages * a.stage_bytes;
  // occupancy at the largest stage size, so one cached figure holds for every H
  const size_t dyn_max = (size_t)kQpStages * qp_stage_bytes(kQpChunk);
  const int dev = moe_host::current_device();
  const int bps = moe_host::blocks_per_sm(permute_quant_kernel, kQpThreads, dyn_max, dev, g_occ_qp);
  int64_t grid = (int64_t)moe_host::sm_count(dev) * bps;
  const int64_t need = T + (int64_t)(kTile - 1) * E;
  if (grid > need) grid = need;
  return moe_host::launch(permute_quant_kernel, dim3((unsigned)grid), dim3(kQpThreads), dyn,
                          static_cast<cudaStream_t>(stream), a);
}
