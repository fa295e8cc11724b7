// Dispatch permute: the "fused unzip" of the DeepEP pull request "Intra-node
// compute compensation + overlap robustness (CUDA719 fix)" (Kernel / host),
// for one GPU: every token row is scattered into its K expert rows of the
// expert-major buffer (expand_x of the torch_npu npu_moe_distribute_combine
// API), padding rows of each expert's last 128-row M-tile (TEMPO summary,
// section 1) are zero-filled, and each finished row bumps its tile's
// chunk-completion counter behind a gpu-scope release.
//
// B200 design.  The work is pure data movement, so it is written as a bulk
// copy engine rather than as threads moving registers:
//   * one warp per CTA (2 CTAs per SM for rows over 8 KiB, else 4); lane 0
//     drives the SM's bulk-copy (TMA) unit: a non-multicast cp.async.bulk
//     global -> shared load of each token row (or 16 KiB column chunk) into
//     an S-stage ring, completed on an mbarrier, then K cp.async.bulk
//     shared -> global stores of the same bytes, one per destination row.
//     The row is read from HBM once and never passes through registers; the
//     token's destination rows (and E4M3 scales) arrive by cp.async on the
//     same mbarrier phase.
//   * padding rows are bulk-stored from a zero-filled shared chunk.
//   * work is claimed dynamically: tokens, then padding rows, as tickets
//     from a claim counter, so CTAs on faster SMs take more of it and all
//     finish together (see the token-ordered pipeline below).
//   * counters: a row's +1 is released only after its bulk-store group has
//     completed (cp.async.bulk.wait_group), behind a proxy fence and a
//     fence.acq_rel.gpu, with relaxed adds (the pull request's
//     atom.acq_rel.gpu on every add is a full fence per row).  Each CTA
//     counts its rows per 128-row tile in a shared-memory table and adds
//     the counts when all of its stores have completed, so no completion
//     wait stalls the copy loop; with too many tiles for the table it
//     releases in batches as it goes.  FP8 scale rows are copied by the 32
//     lanes with plain stores before the same release.
//   * the tile-ordered pipeline for the counter-driven overlap (at the end of
//     this file) fills 16-row items in tile order and releases each as it
//     lands.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

#ifndef MOE_PERM_MAX_CHUNK
#define MOE_PERM_MAX_CHUNK 16384
#endif
#ifndef MOE_PERM_REL_LAG
#define MOE_PERM_REL_LAG 4
#endif
#ifndef MOE_PERM_REL_BATCH
#define MOE_PERM_REL_BATCH 8
#endif
#ifndef MOE_PERM_CTAS_PER_SM
#define MOE_PERM_CTAS_PER_SM 0  // 0: chosen from the row size
#endif
#ifndef MOE_PERM_READ_LAG
#define MOE_PERM_READ_LAG 1
#endif
constexpr uint32_t kMaxChunk = MOE_PERM_MAX_CHUNK;  // bytes per bulk copy
constexpr int kMaxStages = 16;
constexpr int kRelLag = MOE_PERM_REL_LAG;          // bulk groups in flight before a release
constexpr int kReadLag = MOE_PERM_READ_LAG;        // bulk groups still reading before a refill
// Copy pipelines (CTAs) per SM.  Short rows mean more per-row bookkeeping on
// the one issuing lane (waits, fences, counter adds) per byte moved, so they
// get more pipelines per SM to hide it; long rows get deeper rings instead.
inline int perm_ctas_per_sm(int64_t row_bytes) {
  if (MOE_PERM_CTAS_PER_SM > 0) return MOE_PERM_CTAS_PER_SM;
  return row_bytes <= 8192 ? 4 : 2;
}

struct PermArgs {
  const uint8_t* x;
  int64_t x_stride_bytes;
  int64_t row_bytes;
  const float* x_scales;
  int64_t xs_stride;   // elements
  int scale_cols;      // H/128 on the E4M3 path, 0 otherwise
  const int32_t* dst_row;
  int64_t T;
  int K;
  const int32_t* counts;
  const int32_t* offsets;
  int E;
  uint8_t* xp;
  float* xp_scales;
  int64_t P_cap;
  uint32_t* tile_ready;
  int32_t* status;
  uint32_t chunk_cap;   // bytes per chunk (multiple of 16)
  uint32_t stage_bytes; // chunk_cap rounded up to 128
  int n_chunks;
  int stages;
  uint32_t* work;            // [2] claim counter and done count (token-ordered pipeline)
  int64_t tokens_per_ticket; // tokens named by one token ticket
  int64_t pad_per_ticket;    // padding rows named by one padding ticket
  int first_tickets;         // tickets each CTA claims at once to fill its ring
  int early_x;               // issue the first batch's x loads before the grid wait
  int tile_table;            // tiles counted per CTA and released once at its end (0: batched)
};

__device__ __forceinline__ uint32_t chunk_len(const PermArgs& a, int ch) {
  const int64_t rem = a.row_bytes - (int64_t)ch * a.chunk_cap;
  return (uint32_t)(rem < (int64_t)a.chunk_cap ? rem : (int64_t)a.chunk_cap);
}

// ---------------------------------------------------------------------------
// Token-ordered copy pipeline with dynamic work claiming.
//
// Work is handed out as tickets: tickets [0, n_tok) each name tpt
// consecutive tokens, tickets [n_tok, n_tok + n_pad) each name ppt
// consecutive padding rows (in padding-index order).  CTA c starts with the
// fixed batch [c*b, c*b + b) (b = enough tokens to fill its ring), so its
// first loads need no atomic; every later ticket comes from one claim
// counter (work[0]: ticket G*b + the counter's old value), taken whenever the
// ring needs another token.  CTAs on faster SMs simply take more tickets, so
// all of them finish together; the padding tickets come last and fill the
// tail with load-free stores.  (With equal static shares the CTAs' finishing
// times spread over ~30 us of a ~135 us launch.)  A second word (work[1])
// counts CTAs that are done; the last one returns both words to zero, so a
// completed call leaves them ready for the next call.
//
// A token's K destination rows (and, for E4M3, its scale row) are fetched by
// the lanes with cp.async into a token ring in shared memory, and that
// completion is counted on the same mbarrier as the bulk load of the token's
// first chunk, so everything a stage needs has landed when its phase
// completes.  The first loads are issued before the per-expert tables are
// built, which keeps the copy engine busy during the set-up.
// ---------------------------------------------------------------------------
// Releases of the token-ordered pipeline happen in batches: once kRelLag +
// kRelBatch groups are unreleased, one wait, one proxy fence and one gpu-scope
// fence release every group but the newest kRelLag.
constexpr int kRelBatch = MOE_PERM_REL_BATCH;
constexpr int kTokRing = 64;  // tokens whose destination rows are held (until released)
constexpr int kScRing = kMaxStages;  // tokens whose E4M3 scales are held (until processed)
constexpr int64_t kMaxTableTiles = 8192;  // tile table of at most 8 KB per CTA
constexpr int kRecRing = 64;  // committed bulk groups not yet released
static_assert(kRecRing > kRelLag + kRelBatch && kTokRing > kMaxStages + kRelLag + kRelBatch,
              "rings too small for the release lag");

enum : int32_t { kRecNone = 0, kRecToken = 1, kRecPad = 2 };

struct PermShared {
  int32_t off[MOE_MAX_EXPERTS + 1];
  int32_t cnt[MOE_MAX_EXPERTS];
  int32_t padpref[MOE_MAX_EXPERTS + 1];
  int32_t rows[kTokRing][MOE_MAX_TOPK];  // destination rows of token sequence number j % kTokRing
  int32_t rec[kRecRing][3];              // committed groups: {kind, token seq or first pad, end pad}
  int32_t stage_grp[kMaxStages];         // group that last read each stage
  int32_t pre_tok[kMaxStages];           // tokens loaded before the grid wait (early_x)
};

__device__ __forceinline__ void cp_async4(void* sdst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(sdst)), "l"(gsrc)
               : "memory");
}

// The mbarrier's current phase also waits for this thread's earlier cp.async
// copies (the pending count is raised now and lowered when they land).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Lane 0: waits until every bulk group committed before the newest `newer`
// ones has finished reading shared memory.
__device__ __forceinline__ void wait_read_older_than(int newer) {
  if (newer >= 3) bulk_wait_read<3>();
  else if (newer == 2) bulk_wait_read<2>();
  else if (newer == 1) bulk_wait_read<1>();
  else bulk_wait_read<0>();
}

__device__ __forceinline__ void permute_warp(const PermArgs& a, uint8_t* smem, PermShared& sh) {
  const int lane = threadIdx.x & 31;
  const int S = a.stages;
  const int K = a.K, E = a.E, nch = a.n_chunks;
  uint8_t* stage0 = smem;
  uint8_t* zero = smem + (size_t)S * a.stage_bytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(zero + a.stage_bytes);
  float* s_sc = reinterpret_cast<float*>(bar + kMaxStages);  // [kScRing][scale_cols] (E4M3)
  // rows written per 128-row tile by this CTA (tile_table mode; at most 128)
  uint8_t* tbl = reinterpret_cast<uint8_t*>(s_sc + kScRing * a.scale_cols);
  const bool table = a.tile_table > 0;

  const int64_t tpt = a.tokens_per_ticket;
  const int64_t n_tok = (a.T + tpt - 1) / tpt;  // token tickets
  const int first_batch = a.first_tickets;

  // ---- barriers and the fixed first batch: the first loads need neither
  // the tables nor P, nor an atomic ----
  const int64_t dyn0 = (int64_t)gridDim.x * first_batch;  // first counter-issued ticket
  uint32_t pend = 0;
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
    fence_mbarrier_init();
  }
  __syncwarp();
  int64_t k_cur = (int64_t)blockIdx.x * first_batch;  // ticket range in hand
  int64_t k_end = k_cur + first_batch;
  int64_t n_tickets = -1;  // known once the tables are built (padding count)
  int64_t tok_cur = 0, tok_end = 0;  // token range of the ticket in hand
  bool exhausted = false;
  bool ok = true;

  int64_t n_issued = 0, n_tok_issued = 0;
  int64_t issue_t = -1;
  int issue_ch = nch;
  uint32_t n_commit = 0, n_rel = 0;  // lane 0's bulk-group bookkeeping

  const bool fp8 = a.scale_cols > 0;

  // Warp-uniform.  Next token to load, -1 when the work is exhausted, or -2
  // when the next ticket is not a token ticket and padding cannot be handled
  // yet (before the tables exist).
  auto next_ticket = [&](bool allow_pad, int64_t& k) -> bool {
    if (k_cur < k_end) {
      if (!allow_pad && k_cur >= n_tok) return false;
      k = k_cur++;
      return true;
    }
    if (!allow_pad) return false;  // the pending claim may be a padding ticket
    k = dyn0 + (int64_t)__shfl_sync(0xffffffffu, pend, 0);
    if (lane == 0 && k < n_tickets) pend = atomicAdd(a.work, 1u);
    return true;
  };

  // ---- padding rows: tables and helpers ----
  struct PadCursor {
    int e;
    __device__ void seek(const int32_t* padpref, int E, int64_t q) {
      int lo = 0, hi = E - 1;  // last expert with padpref <= q
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (padpref[mid] <= q) lo = mid; else hi = mid - 1;
      }
      e = lo;
    }
  };
  auto pad_row = [&](PadCursor& cur, int64_t q) -> int64_t {
    while (q >= sh.padpref[cur.e + 1]) ++cur.e;
    return (int64_t)sh.off[cur.e] + sh.cnt[cur.e] + (q - sh.padpref[cur.e]);
  };
  // lane 0: +n for padding indices [qa, qb), one add per run inside one expert
  auto release_padding = [&](int64_t qa, int64_t qb) {
    PadCursor cur;
    cur.seek(sh.padpref, E, qa);
    int64_t q = qa;
    while (q < qb) {
      const int64_t r = pad_row(cur, q);
      const int64_t q_end = min(qb, (int64_t)sh.padpref[cur.e + 1]);
      atomic_add_relaxed_gpu(a.tile_ready + r / kTile, (uint32_t)(q_end - q));
      q = q_end;
    }
  };
  // lane 0: release the groups older than the newest kRelLag once they completed
  auto retire = [&]() {
    if (table || a.tile_ready == nullptr || n_commit - n_rel < (uint32_t)(kRelLag + kRelBatch))
      return;
    bulk_wait_all<kRelLag>();
    fence_proxy_async_global();
    fence_acq_rel_gpu();
    while (n_commit - n_rel > (uint32_t)kRelLag) {
      const int32_t* rc = sh.rec[n_rel % kRecRing];
      if (rc[0] == kRecToken) {
        const int32_t* rows = sh.rows[rc[1] % kTokRing];
        for (int j = 0; j < K; ++j)
          if (rows[j] >= 0) atomic_add_relaxed_gpu(a.tile_ready + rows[j] / kTile, 1u);
      } else if (rc[0] == kRecPad) {
        release_padding(rc[1], rc[2]);
      }
      ++n_rel;
    }
  };
  auto push_rec = [&](int32_t kind, int64_t x0, int64_t x1) {  // lane 0, after a commit
    int32_t* rc = sh.rec[n_commit % kRecRing];
    rc[0] = kind;
    rc[1] = (int32_t)x0;
    rc[2] = (int32_t)x1;
    ++n_commit;
  };
  // Warp-uniform: zero rows for padding ticket pb, as one bulk group.
  auto do_padding = [&](int64_t pb) {
    const int64_t qa = pb * a.pad_per_ticket;
    const int64_t qb = min(qa + a.pad_per_ticket, (int64_t)sh.padpref[E]);
    PadCursor cur;
    cur.seek(sh.padpref, E, qa);
    for (int64_t q = qa; q < qb; ++q) {
      const int64_t r = pad_row(cur, q);
      if (fp8)
        for (int cc = lane; cc < a.scale_cols; cc += 32) a.xp_scales[r * a.scale_cols + cc] = 0.0f;
      if (lane == 0)
        for (int ch = 0; ch < nch; ++ch)
          bulk_store_s2g(a.xp + r * a.row_bytes + (int64_t)ch * a.chunk_cap, zero, chunk_len(a, ch));
    }
    __syncwarp();  // the lanes' scale stores precede lane 0's release
    if (lane == 0) {
      bulk_commit();
      push_rec(kRecPad, qa, qb);
      if (table) {
        PadCursor tc;
        tc.seek(sh.padpref, E, qa);
        for (int64_t q = qa; q < qb;) {
          const int64_t r = pad_row(tc, q);
          const int64_t q_end = min(qb, (int64_t)sh.padpref[tc.e + 1]);
          tbl[r / kTile] += (uint8_t)(q_end - q);
          q = q_end;
        }
      }
      retire();
    }
  };

  // Warp-uniform: issue the next unit's load (claiming a token when the
  // current one has no chunk left).  Returns false when nothing was issued.
  auto issue_next = [&](bool allow_pad, bool with_rows) -> bool {
    if (issue_ch == nch) {
      int64_t t = -1;
      while (t < 0) {
        if (tok_cur < tok_end) {
          t = tok_cur++;
          break;
        }
        if (exhausted) return false;
        int64_t k;
        if (!next_ticket(allow_pad, k)) return false;
        if (k < n_tok) {
          tok_cur = k * tpt;
          tok_end = min(a.T, tok_cur + tpt);
        } else if (k < n_tickets) {
          do_padding(k - n_tok);
        } else {
          exhausted = true;
          return false;
        }
      }
      issue_t = t;
      issue_ch = 0;
    }
    const int s = (int)(n_issued % S);
    if (lane == 0 && n_issued >= S)  // the stage's previous group has read it
      wait_read_older_than((int)(n_commit - 1u - (uint32_t)sh.stage_grp[s]));
    if (issue_ch == 0 && !with_rows) {  // rows and scales are read after the grid wait
      if (lane == 0) sh.pre_tok[n_tok_issued] = (int32_t)issue_t;
      ++n_tok_issued;
    } else if (issue_ch == 0) {  // the token's rows (and scales) ride on the same barrier phase
      const int ring = (int)(n_tok_issued % kTokRing);
      bool copied = false;
      if (lane < K) {
        cp_async4(&sh.rows[ring][lane], a.dst_row + issue_t * K + lane);
        copied = true;
      }
      if (fp8)
        for (int cc = lane; cc < a.scale_cols; cc += 32) {
          cp_async4(s_sc + (int)(n_tok_issued % kScRing) * a.scale_cols + cc,
                    a.x_scales + issue_t * a.xs_stride + cc);
          copied = true;
        }
      if (copied) cp_async_arrive(&bar[s]);
      ++n_tok_issued;
      __syncwarp();
    }
    if (lane == 0) {
      const uint32_t len = chunk_len(a, issue_ch);
      mbar_arrive_expect_tx(&bar[s], len);
      bulk_load_g2s(stage0 + (size_t)s * a.stage_bytes,
                    a.x + issue_t * a.x_stride_bytes + (int64_t)issue_ch * a.chunk_cap, len,
                    &bar[s]);
    }
    ++issue_ch;
    ++n_issued;
    return true;
  };

  // ---- first loads, from the first claimed batch (token tickets only) ----
  // With early_x (only inside the combined dispatch call, where x was written
  // before the layout's kernels started) these loads go out before the grid
  // wait, while the layout still runs; the tokens' rows and scales, which
  // the layout produces or which are only needed later, are then read right
  // after the wait.  Otherwise the grid wait came first.
  const bool pre = a.early_x != 0;
  while (n_issued < S && issue_next(false, !pre)) {
  }
  if (pre) {
    pdl_begin();
    __syncwarp();
    for (int64_t j = 0; j < n_tok_issued; ++j) {
      const int64_t t = sh.pre_tok[j];
      if (lane < K) sh.rows[j % kTokRing][lane] = __ldg(a.dst_row + t * K + lane);
      if (fp8)
        for (int cc = lane; cc < a.scale_cols; cc += 32)
          s_sc[(j % kScRing) * a.scale_cols + cc] = __ldg(a.x_scales + t * a.xs_stride + cc);
    }
    __syncwarp();
  }
  if (lane == 0) pend = atomicAdd(a.work, 1u);  // needed only once the batch is used up

  // ---- per-expert tables, the padding prefix sum and the zero chunk ----
  for (int e = lane; e <= E; e += 32) sh.off[e] = __ldg(a.offsets + e);
  for (int e = lane; e < E; e += 32) sh.cnt[e] = __ldg(a.counts + e);
  __syncwarp();
  int bad = 0;
  int run = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    int pad = 0;
    if (e < E) {
      pad = (sh.off[e + 1] - sh.off[e]) - sh.cnt[e];
      if (pad < 0 || pad >= kTile || sh.cnt[e] < 0) {
        bad = 1;
        pad = 0;
      }
    }
    const int incl = warp_inclusive_scan(pad);
    if (e < E) sh.padpref[e] = run + incl - pad;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) sh.padpref[E] = run;
  for (uint32_t i = lane * 16; i < a.stage_bytes; i += 32 * 16)
    *reinterpret_cast<uint4*>(zero + i) = make_uint4(0, 0, 0, 0);
  if (table)
    for (int i = lane * 16; i < a.tile_table; i += 32 * 16)
      *reinterpret_cast<uint4*>(tbl + i) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_shared();
  __syncwarp();
  if (__any_sync(0xffffffffu, bad) || (int64_t)sh.off[E] > a.P_cap || sh.off[0] != 0) {
    if (lane == 0) record_error(a.status, MOE_ERR_BOUNDS);
    ok = false;  // nothing is stored; the loads already issued drain below
  }
  n_tickets = n_tok + ((int64_t)run + a.pad_per_ticket - 1) / a.pad_per_ticket;

  // ---- main loop: process unit u, then top the ring up ----
  int64_t u = 0;
  while (ok) {
    if (u == n_issued && !issue_next(true, true)) break;
    const int s = (int)(u % S);
    int landed = 1;
    if (lane == 0) landed = mbar_wait_bounded(&bar[s], (uint32_t)((u / S) & 1)) ? 1 : 0;
    landed = __shfl_sync(0xffffffffu, landed, 0);
    if (!landed) {
      if (lane == 0) record_error(a.status, MOE_ERR_TIMEOUT);
      ok = false;
      break;
    }
    mbar_try_wait(&bar[s], (uint32_t)((u / S) & 1));  // every lane acquires the landed phase
    const int64_t j = u / nch;
    const int ch = (int)(u % nch);
    int32_t* rows = sh.rows[j % kTokRing];
    if (ch == 0) {  // checked once per token: an out-of-range row is reported and skipped
      if (lane < K) {
        const int32_t r = rows[lane];
        if (r != -1 && (r < 0 || (int64_t)r >= a.P_cap)) {
          record_error(a.status, MOE_ERR_BOUNDS);
          rows[lane] = -1;
        }
      }
      __syncwarp();
      if (fp8) {
        const float* sc = s_sc + (j % kScRing) * a.scale_cols;
        for (int k = 0; k < K; ++k) {
          const int64_t r = rows[k];
          if (r < 0) continue;
          for (int cc = lane; cc < a.scale_cols; cc += 32) a.xp_scales[r * a.scale_cols + cc] = sc[cc];
        }
        __syncwarp();  // the lanes' scale stores precede lane 0's release
      }
    }
    if (lane == 0) {
      const uint32_t len = chunk_len(a, ch);
      const uint8_t* src = stage0 + (size_t)s * a.stage_bytes;
      for (int k = 0; k < K; ++k) {
        const int64_t r = rows[k];
        if (r < 0) continue;
        bulk_store_s2g(a.xp + r * a.row_bytes + (int64_t)ch * a.chunk_cap, src, len);
      }
      bulk_commit();
      sh.stage_grp[s] = (int32_t)n_commit;
      push_rec(ch == nch - 1 ? kRecToken : kRecNone, j, 0);
      if (table && ch == nch - 1)
        for (int k = 0; k < K; ++k)
          if (rows[k] >= 0) tbl[rows[k] / kTile] += 1;
      retire();
    }
    ++u;
    while (n_issued < u + S && issue_next(true, true)) {
    }
  }

  // ---- drain ----
  __syncwarp();
  if (lane == 0) {
    if (!ok) {
      // loads still in flight get a bounded chance to land before the CTA's
      // shared memory is given back
      for (int64_t v = u; v < n_issued; ++v)
        if (!mbar_wait_bounded(&bar[v % S], (uint32_t)((v / S) & 1))) break;
    }
    bulk_wait_all<0>();
    if (ok && table) fence_proxy_async_global();
    if (ok && !table && a.tile_ready != nullptr && n_commit != n_rel) {
      fence_proxy_async_global();
      fence_acq_rel_gpu();
      while (n_rel != n_commit) {
        const int32_t* rc = sh.rec[n_rel % kRecRing];
        if (rc[0] == kRecToken) {
          const int32_t* rws = sh.rows[rc[1] % kTokRing];
          for (int k = 0; k < K; ++k)
            if (rws[k] >= 0) atomic_add_relaxed_gpu(a.tile_ready + rws[k] / kTile, 1u);
        } else if (rc[0] == kRecPad) {
          release_padding(rc[1], rc[2]);
        }
        ++n_rel;
      }
    }
  }
  if (ok && table) {
    // every row this CTA wrote has landed: one release per tile it touched
    __syncwarp();
    fence_acq_rel_gpu();
    for (int i = lane; i < a.tile_table; i += 32)
      if (tbl[i] != 0) atomic_add_relaxed_gpu(a.tile_ready + i, (uint32_t)tbl[i]);
  }
  if (lane == 0) finish_claims(a.work);  // the last CTA out returns both words to zero
}

__global__ void __launch_bounds__(32, 1) permute_kernel(const PermArgs a) {
  if (!a.early_x) pdl_begin();  // with early_x, permute_warp waits after its first loads
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ PermShared sh;
  permute_warp(a, smem, sh);
}

// ---------------------------------------------------------------------------
// Tile-ordered copy pipeline, for overlap with consumers.  The token-ordered
// pipeline above reads each x row once but fills every tile from all CTAs,
// so tiles complete only near the end.  Here the padded rows are cut into
// items of 16 rows (8 per tile) dealt round-robin: CTA c fills items
// c, c + G, ... in that order, row by row (one bulk load of the source
// token's row, one bulk store), adding 16 to the tile's counter as each item
// lands.  Item r belongs to tile r / 8, so tiles complete roughly in index
// order while the copy runs.  x rows are read once per slot (K times per
// token); most of those reads hit L2.  The row -> slot maps (row_src) of the
// next items are fetched two items ahead into registers and published to a
// three-slot shared ring one item ahead of use.
// ---------------------------------------------------------------------------
constexpr int kItemRows = 16;
constexpr int kItemsPerTile = kTile / kItemRows;

struct TileShared {
  int32_t src[3][kItemRows];
};

__device__ __forceinline__ void permute_tiles_warp(const PermArgs& a, const int32_t* row_src,
                                                   const int64_t c, const int64_t G,
                                                   uint8_t* smem, TileShared& sh,
                                                   uint32_t* tile_sums) {
  const int lane = threadIdx.x & 31;
  const int S = a.stages;
  uint8_t* stage0 = smem;
  uint8_t* zero = smem + (size_t)S * a.stage_bytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(zero + a.stage_bytes);

  const int64_t P = __ldg(a.offsets + a.E);
  if (P < 0 || P > a.P_cap || P % kTile != 0) {
    if (lane == 0) record_error(a.status, MOE_ERR_BOUNDS);
    return;
  }
  const int64_t n_items = P / kItemRows;
  const int64_t ni = c < n_items ? (n_items - c + G - 1) / G : 0;  // items of this CTA
  const int nch = a.n_chunks;
  const int64_t per_item = (int64_t)kItemRows * nch;
  const int64_t n_units = ni * per_item;

  for (uint32_t i = lane * 16; i < a.stage_bytes; i += 32 * 16)
    *reinterpret_cast<uint4*>(zero + i) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_shared();
  if (lane == 0) {
    for (int s2 = 0; s2 < S; ++s2) mbar_init(&bar[s2], 1);
    fence_mbarrier_init();
  }
  auto item_row0 = [&](int64_t m) { return (c + m * G) * kItemRows; };  // first padded row
  // row -> slot map of one item: lane l < 16 holds row l, -1 for padding
  int32_t pre = -1;
  auto fetch_src = [&](int64_t m) {
    pre = -1;
    if (lane < kItemRows && m < ni) {
      int32_t v = __ldg(row_src + item_row0(m) + lane);
      if (v < -1 || (int64_t)v >= a.T * a.K) {
        record_error(a.status, MOE_ERR_BOUNDS);
        v = -1;
      }
      pre = v;
    }
  };
  auto publish_src = [&](int64_t m) {
    if (lane < kItemRows) sh.src[m % 3][lane] = pre;
  };
  fetch_src(0);
  publish_src(0);
  fetch_src(1);
  publish_src(1);
  fetch_src(2);  // published when item 1 starts
  __syncwarp();

  auto unit_item = [&](int64_t u) { return u / per_item; };
  auto unit_row = [&](int64_t u) { return (int)((u / nch) % kItemRows); };
  const uint64_t x_policy = make_policy_evict_last();
  auto issue_load = [&](int64_t u) {  // lane 0 only
    const int s2 = (int)(u % S);
    const int64_t m = unit_item(u);
    const int src = sh.src[m % 3][unit_row(u)];
    if (src < 0) {  // padding row: nothing to load; complete the phase
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&bar[s2]))
                   : "memory");
      return;
    }
    const int ch = (int)(u % nch);
    const uint32_t len = chunk_len(a, ch);
    const uint8_t* srcp =
        a.x + (int64_t)(src / a.K) * a.x_stride_bytes + (int64_t)ch * a.chunk_cap;
    mbar_arrive_expect_tx(&bar[s2], len);
    // x is read once per slot: keep it in L2 for the token's other slots
    bulk_load_g2s_hint(stage0 + (size_t)s2 * a.stage_bytes, srcp, len, &bar[s2], x_policy);
  };
  // Lane 0, after the item's groups completed.  The first item of a tile also
  // clears the tile's sum that the consumers accumulate into (nullable): the
  // clear precedes the release, and consumers add only after acquiring the
  // complete tile, so it lands before every add.
  auto release_item = [&](int64_t m) {
    const int64_t row0 = item_row0(m);
    if (tile_sums && (row0 % kTile) == 0) tile_sums[row0 / kTile] = 0u;
    fence_acq_rel_gpu();
    atomic_add_relaxed_gpu(a.tile_ready + row0 / kTile, (uint32_t)kItemRows);
  };

  int64_t issued = 0;
  if (lane == 0)
    for (; issued < n_units && issued < S; ++issued) issue_load(issued);

  int64_t u_fail = -1;
  for (int64_t u = 0; u < n_units; ++u) {
    const int s2 = (int)(u % S);
    const int64_t m = unit_item(u);
    const int i = unit_row(u);
    const int ch = (int)(u % nch);
    if (ch == 0 && i == 0 && m >= 1) {  // item m starts: publish m + 1, fetch m + 2
      publish_src(m + 1);
      fetch_src(m + 2);
      __syncwarp();
    }
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(&bar[s2], (uint32_t)((u / S) & 1)) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      u_fail = u;
      break;
    }
    const int src = sh.src[m % 3][i];
    const int64_t p = item_row0(m) + i;
    if (ch == 0 && a.scale_cols > 0) {  // FP8 scale row (or zeros), all lanes
      float* dst = a.xp_scales + p * a.scale_cols;
      const float* xs = src >= 0 ? a.x_scales + (int64_t)(src / a.K) * a.xs_stride : nullptr;
      for (int cc = lane; cc < a.scale_cols; cc += 32) dst[cc] = xs ? __ldg(xs + cc) : 0.0f;
    }
    if (lane == 0) {
      const uint32_t len = chunk_len(a, ch);
      const uint8_t* from = src >= 0 ? stage0 + (size_t)s2 * a.stage_bytes : zero;
      bulk_store_s2g(a.xp + p * a.row_bytes + (int64_t)ch * a.chunk_cap, from, len);
      bulk_commit();
    }
    if (a.tile_ready) {
      __syncwarp();  // the lanes' scale stores precede lane 0's release
      if (lane == 0) {
        bulk_wait_all<kRelLag>();
        const int64_t ur = u - kRelLag;
        if (ur >= 0 && (ur + 1) % per_item == 0) {
          fence_proxy_async_global();
          release_item(unit_item(ur));
        }
      }
    }
    if (lane == 0) {
      bulk_wait_read<kReadLag>();
      if (u >= kReadLag && issued < n_units) {
        issue_load(issued);
        ++issued;
      }
    }
  }
  if (u_fail >= 0) {
    if (lane == 0) {
      record_error(a.status, MOE_ERR_TIMEOUT);
      bulk_wait_all<0>();
      for (int64_t u = u_fail + 1; u < issued; ++u)
        if (!mbar_wait_bounded(&bar[u % S], (uint32_t)((u / S) & 1))) break;
    }
    return;
  }
  __syncwarp();
  if (lane == 0) {
    bulk_wait_all<0>();
    if (a.tile_ready) {
      fence_proxy_async_global();
      for (int64_t ur = max((int64_t)0, n_units - kRelLag); ur < n_units; ++ur)
        if ((ur + 1) % per_item == 0) release_item(unit_item(ur));
    }
  }
}

// ---------------------------------------------------------------------------
// Producer and consumers in one cooperative launch.  Warp 0 of every CTA is a
// tile-ordered copy pipeline (items of 16 rows, tiles completing roughly in
// index order); warps 1..3 form the CTA's consumer group, which takes the
// same items as its producer: for each, thread 0 of the group polls the
// item's tile counter with ld.acquire.gpu (bounded) until the whole tile is
// published, a named barrier orders that acquire before the group's reads,
// and the group adds the item's share of the tile checksum defined by
// moe_wait_tiles_checksum (weights by word position in the tile, sums mod
// 2^32, so the order of the adds does not matter) -- an expert stand-in that
// must see every byte.  All CTAs are resident at once
// (cooperative launch), so a consumer never waits on a producer that cannot
// run.
// ---------------------------------------------------------------------------
constexpr int kConsumerWarps = 3;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kFusedThreads = 32 + kConsumerThreads;
constexpr int kFusedCtasPerSm = 4;  // copy pipelines per SM (as for short rows)

struct ConsumerArgs {
  const int32_t* row_src;
  uint32_t* checksums;
  int64_t timeout_ns;
};

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// sum over words w_i, i = base + 4v + q, of w_i * (2i + 1) for the 16-byte
// vectors v = first, first + step, ... below n4
__device__ __forceinline__ uint32_t weighted_words(const uint4* p, int64_t n4, int64_t first,
                                                   int64_t step, uint32_t base) {
  uint32_t acc = 0;
#pragma unroll 8
  for (int64_t v = first; v < n4; v += step) {
    const uint4 w = ld_cg_v4(p + v);
    const uint32_t i = base + 4u * (uint32_t)v;
    acc += w.x * (2u * i + 1u) + w.y * (2u * i + 3u) + w.z * (2u * i + 5u) + w.w * (2u * i + 7u);
  }
  return acc;
}

__global__ void __launch_bounds__(kFusedThreads, 1)
permute_consume_kernel(const PermArgs a, const ConsumerArgs cs) {
  pdl_begin();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ TileShared sh;
  __shared__ uint32_t s_red[kConsumerWarps];
  __shared__ int s_ok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    permute_tiles_warp(a, cs.row_src, blockIdx.x, gridDim.x, smem, sh, cs.checksums);
    return;
  }
  // consumers: the same 16-row items this CTA's producer writes, each taken
  // once its whole tile has been published
  const int ct = threadIdx.x - 32;
  const int64_t P = __ldg(a.offsets + a.E);
  if (P < 0 || P > a.P_cap || P % kTile != 0) {  // same value for every consumer thread
    if (ct == 0) record_error(a.status, MOE_ERR_BOUNDS);
    return;
  }
  const int64_t n_items = P / kItemRows;
  const int64_t item4 = (int64_t)kItemRows * a.row_bytes / 16;       // 16-byte words per item
  const int64_t tile_words = (int64_t)kTile * a.row_bytes / 4;       // data words per tile
  const int64_t sitem4 = a.scale_cols > 0 ? (int64_t)kItemRows * a.scale_cols / 4 : 0;
  for (int64_t r = blockIdx.x; r < n_items; r += gridDim.x) {
    const int64_t j = r / kItemsPerTile;
    const int q = (int)(r % kItemsPerTile);
    if (ct == 0) {
      int ok = 0;
      if (read_status(a.status) == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (true) {
          if (ld_acquire_gpu(a.tile_ready + j) == (uint32_t)kTile) {
            ok = 1;
            break;
          }
          if ((int64_t)(globaltimer_ns() - t0) > cs.timeout_ns) break;
          __nanosleep(128);
        }
        if (!ok) record_error(a.status, MOE_ERR_TIMEOUT);
      }
      s_ok = ok;
    }
    consumer_bar();  // orders thread 0's acquire before the group's reads
    const int ok = s_ok;
    uint32_t acc = 0;
    if (ok) {
      const int64_t row0 = r * kItemRows;
      acc = weighted_words(reinterpret_cast<const uint4*>(a.xp + row0 * a.row_bytes), item4, ct,
                           kConsumerThreads, (uint32_t)(q * 4 * item4));
      if (sitem4)
        acc += weighted_words(reinterpret_cast<const uint4*>(a.xp_scales + row0 * a.scale_cols),
                              sitem4, ct, kConsumerThreads,
                              (uint32_t)(tile_words + q * 4 * sitem4));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s_red[warp - 1] = acc;
    consumer_bar();
    if (ct == 0 && ok) {
      uint32_t sum = 0;
      for (int w = 0; w < kConsumerWarps; ++w) sum += s_red[w];
      atomicAdd(cs.checksums + j, sum);  // wraps mod 2^32: order does not matter
    }
    consumer_bar();  // s_ok and s_red are reused by the next item
  }
}

}  // namespace
}  // namespace moe

namespace moe {
namespace {

// Host-side checks shared by the permute entry points; fills everything in
// PermArgs but the ring depth.  Returns MOE_OK or the status to report.
int make_perm_args(const void* x, int dtype, int64_t T, int H, int64_t x_row_stride,
                   const float* x_scales, int64_t x_scales_row_stride, const int32_t* dst_row,
                   int K, const int32_t* expert_counts, const int32_t* expert_offsets, int E,
                   void* xp, float* xp_scales, int64_t P_cap, uint32_t* tile_ready,
                   int32_t* d_status, PermArgs* out) {
  *out = PermArgs{};
  if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (T < 0 || H <= 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 || E > MOE_MAX_EXPERTS)
    return MOE_ERR_INVALID_ARG;
  if (T * (int64_t)K > (int64_t)INT32_MAX || P_cap > (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (P_cap < moe_padded_capacity(T, K, E)) return MOE_ERR_CAPACITY;
  if (x_row_stride < H) return MOE_ERR_INVALID_ARG;
  const int elem = dtype == MOE_DTYPE_BF16 ? 2 : 1;
  const int64_t row_bytes = (int64_t)H * elem;
  if (row_bytes % 16 != 0 || (x_row_stride * elem) % 16 != 0) return MOE_ERR_INVALID_ARG;
  // an empty batch (P_cap = 0) may pass null row buffers
  if ((P_cap > 0 && !xp) || !expert_counts || !expert_offsets || (T > 0 && (!x || !dst_row)))
    return MOE_ERR_INVALID_ARG;
  if (!moe_host::aligned16(xp) || (x && !moe_host::aligned16(x))) return MOE_ERR_INVALID_ARG;
  int scale_cols = 0;
  if (dtype == MOE_DTYPE_E4M3) {
    if (H % 128 != 0 || (P_cap > 0 && !xp_scales) || (T > 0 && !x_scales))
      return MOE_ERR_INVALID_ARG;
    scale_cols = H / 128;
    if (x_scales_row_stride < scale_cols) return MOE_ERR_INVALID_ARG;
  } else if (x_scales || xp_scales) {
    return MOE_ERR_INVALID_ARG;
  }
  PermArgs& a = *out;
  a.x = static_cast<const uint8_t*>(x);
  a.x_stride_bytes = x_row_stride * elem;
  a.row_bytes = row_bytes;
  a.x_scales = x_scales;
  a.xs_stride = x_scales_row_stride;
  a.scale_cols = scale_cols;
  a.dst_row = dst_row;
  a.T = T;
  a.K = K;
  a.counts = expert_counts;
  a.offsets = expert_offsets;
  a.E = E;
  a.xp = static_cast<uint8_t*>(xp);
  a.xp_scales = xp_scales;
  a.P_cap = P_cap;
  a.tile_ready = tile_ready;
  a.status = d_status;
  a.chunk_cap = (uint32_t)(row_bytes < (int64_t)kMaxChunk ? row_bytes : kMaxChunk);
  a.stage_bytes = (a.chunk_cap + 127u) / 128u * 128u;
  a.n_chunks = (int)((row_bytes + a.chunk_cap - 1) / a.chunk_cap);
  a.stages = 0;
  return MOE_OK;
}

// Ring depth for `ctas_per_sm` CTAs sharing an SM's shared memory, with
// `extra` bytes of dynamic shared memory after the stages, the zero chunk and
// the kMaxStages mbarriers; returns the dynamic shared-memory bytes, or 0 if
// even two stages do not fit.
size_t size_ring(PermArgs& a, int ctas_per_sm, size_t static_smem, int optin, size_t extra = 0) {
  const size_t fixed = (size_t)a.stage_bytes + kMaxStages * 8 + extra;
  const size_t per_cta = (size_t)optin / ctas_per_sm - static_smem - 1024;
  int stages = per_cta > fixed ? (int)((per_cta - fixed) / a.stage_bytes) : 0;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) stages = 2;
  a.stages = stages;
  const size_t dyn = (size_t)stages * a.stage_bytes + fixed;
  return dyn + static_smem > (size_t)optin ? 0 : dyn;
}

int optin_smem(int dev) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return -1;
  return optin;
}

// Lets `kernel` request up to all the dynamic shared memory the device
// allows, once per device.  (Setting the exact size of each call instead
// would race between host threads launching different row sizes.)  The
// occupancy still follows the size each launch asks for.
template <typename F>
bool allow_max_dyn_smem(F kernel, int dev, int optin, std::atomic<int>* done) {
  const bool cached = dev >= 0 && dev < moe_host::kMaxCachedDevices;
  if (cached && done[dev].load(std::memory_order_acquire)) return true;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin - (int)fa.sharedSizeBytes) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cached) done[dev].store(1, std::memory_order_release);
  return true;
}

std::atomic<int> g_dyn_perm[moe_host::kMaxCachedDevices];
std::atomic<int> g_dyn_consume[moe_host::kMaxCachedDevices];

}  // namespace
}  // namespace moe

namespace moe {
// The permute's checks and launch (see moe_dispatch_permute).  With dry_run
// the checks run and nothing is launched; early_x lets the kernel issue its
// first x loads before its grid wait, which only a caller that launched the
// layout itself may ask for (x must be complete before the previous kernel
// began).
int permute_launch(const void* x, int dtype, int64_t T, int H, int64_t x_row_stride,
                   const float* x_scales, int64_t x_scales_row_stride, const int32_t* dst_row,
                   int K, const int32_t* expert_counts, const int32_t* expert_offsets, int E,
                   void* xp, float* xp_scales, int64_t P_cap, uint32_t* tile_ready,
                   uint32_t* work, int32_t* d_status, cudaStream_t stream, int early_x,
                   int dry_run) {
  PermArgs a;
  int st = make_perm_args(x, dtype, T, H, x_row_stride, x_scales, x_scales_row_stride, dst_row,
                          K, expert_counts, expert_offsets, E, xp, xp_scales, P_cap, tile_ready,
                          d_status, &a);
  if (st != MOE_OK) return st;
  if (!work || !moe_host::aligned4(work)) return MOE_ERR_INVALID_ARG;
  if (dry_run || T == 0) return MOE_OK;  // T = 0: P = 0, nothing to write

  const int dev = moe_host::current_device();
  const int optin = optin_smem(dev);
  if (optin < 0) return MOE_ERR_CUDA;
  const int ctas_per_sm = perm_ctas_per_sm(a.row_bytes);
  const size_t scale_ring = (size_t)kScRing * a.scale_cols * sizeof(float);
  // Per-CTA tile table (one byte per tile) when the tiles fit
  // kMaxTableTiles; else releases in batches during the copy.
  const int64_t n_tiles = (P_cap + kTile - 1) / kTile;
  a.tile_table = (tile_ready != nullptr && n_tiles <= kMaxTableTiles)
                     ? (int)((n_tiles + 15) / 16 * 16) : 0;
  const size_t dyn = size_ring(a, ctas_per_sm, sizeof(PermShared), optin,
                               scale_ring + (size_t)a.tile_table);
  if (dyn == 0) return MOE_ERR_UNSUPPORTED;
  if (!allow_max_dyn_smem(permute_kernel, dev, optin, g_dyn_perm)) return MOE_ERR_CUDA;

  // Tickets: a token ticket names enough tokens for about 32 KiB of row
  // writes; a padding ticket names as many rows as a token ticket writes.
  const int64_t tok_bytes = (int64_t)K * a.row_bytes;
  a.tokens_per_ticket = std::min<int64_t>(64, std::max<int64_t>(1, (32768 + tok_bytes - 1) / tok_bytes));
  a.pad_per_ticket = (int64_t)K * a.tokens_per_ticket;
  a.first_tickets = (int)std::max<int64_t>(
      1, (a.stages + (int64_t)a.n_chunks * a.tokens_per_ticket - 1) /
             ((int64_t)a.n_chunks * a.tokens_per_ticket));
  a.work = work;
  a.early_x = early_x;

  const int64_t v_bound = T * K + (int64_t)(kTile - 1) * E;
  int64_t grid = (int64_t)moe_host::sm_count(dev) * ctas_per_sm;
  const int64_t by_work = (v_bound + 7) / 8;
  if (grid > by_work) grid = by_work;
  if (grid < 1) grid = 1;
  return moe_host::launch(permute_kernel, dim3((unsigned)grid), dim3(32), dyn, stream, a);
}
}  // namespace moe

extern "C" int moe_dispatch_permute(const void* x, int dtype, int64_t T, int H,
                                    int64_t x_row_stride, const float* x_scales,
                                    int64_t x_scales_row_stride, const int32_t* dst_row, int K,
                                    const int32_t* expert_counts, const int32_t* expert_offsets,
                                    int E, void* xp, float* xp_scales, int64_t P_cap,
                                    uint32_t* tile_ready, uint32_t* work, int32_t* d_status,
                                    void* stream) {
  return moe::permute_launch(x, dtype, T, H, x_row_stride, x_scales, x_scales_row_stride,
                             dst_row, K, expert_counts, expert_offsets, E, xp, xp_scales, P_cap,
                             tile_ready, work, d_status, static_cast<cudaStream_t>(stream), 0, 0);
}

extern "C" int moe_dispatch_permute_consume(
    const void* x, int dtype, int64_t T, int H, int64_t x_row_stride, const float* x_scales,
    int64_t x_scales_row_stride, const int32_t* dst_row, int K, const int32_t* expert_counts,
    const int32_t* expert_offsets, int E, const int32_t* row_src, void* xp, float* xp_scales,
    int64_t P_cap, uint32_t* tile_ready, uint32_t* checksums, int64_t timeout_ns,
    int32_t* d_status, void* stream) {
  using namespace moe;
  if (!tile_ready || !checksums || !row_src || timeout_ns < 0) return MOE_ERR_INVALID_ARG;
  if (xp_scales && !moe_host::aligned16(xp_scales)) return MOE_ERR_INVALID_ARG;
  if (!moe_host::aligned4(checksums)) return MOE_ERR_INVALID_ARG;
  PermArgs a;
  int st = make_perm_args(x, dtype, T, H, x_row_stride, x_scales, x_scales_row_stride, dst_row,
                          K, expert_counts, expert_offsets, E, xp, xp_scales, P_cap, tile_ready,
                          d_status, &a);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;

  const int dev = moe_host::current_device();
  const int optin = optin_smem(dev);
  if (optin < 0) return MOE_ERR_CUDA;
  const size_t static_smem = sizeof(TileShared) + 64;
  const size_t dyn = size_ring(a, kFusedCtasPerSm, static_smem, optin);
  if (dyn == 0) return MOE_ERR_UNSUPPORTED;
  if (!allow_max_dyn_smem(permute_consume_kernel, dev, optin, g_dyn_consume)) return MOE_ERR_CUDA;
  // every CTA must be resident at once (consumers wait on other CTAs' rows):
  // a cooperative launch no larger than the device can hold
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_consume_kernel,
                                                    kFusedThreads, dyn) != cudaSuccess ||
      per_sm < 1)
    return MOE_ERR_UNSUPPORTED;
  if (per_sm > kFusedCtasPerSm) per_sm = kFusedCtasPerSm;
  int64_t grid = (int64_t)moe_host::sm_count(dev) * per_sm;
  const int64_t v_bound = T * K + (int64_t)(kTile - 1) * E;
  const int64_t by_work = (v_bound + 7) / 8;
  if (grid > by_work) grid = by_work;
  if (grid < 1) grid = 1;
  ConsumerArgs c;
  c.row_src = row_src;
  c.checksums = checksums;
  c.timeout_ns = timeout_ns;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, permute_consume_kernel, a, c) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
