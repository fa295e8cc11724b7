// Shared device helpers for the dispatch / combine kernels (sm_100a).
//
// Inline PTX wrappers for the Blackwell features the kernels use: mbarrier
// transaction barriers, non-multicast bulk copies between global and the
// issuing CTA's own shared memory (cp.async.bulk), the async-proxy fences
// they need, gpu-scope acquire loads and release patterns for the
// chunk-completion counters, and %globaltimer for bounded waits.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "moe_dispatch.h"

namespace moe {

constexpr int kTile = MOE_TILE_M;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s for any device-side wait

// ------------------------------------------- programmatic dependent launch --
// Every kernel is launched with programmatic stream serialization and starts
// by waiting until the previous kernel has finished and its writes are
// visible.  No kernel triggers its dependents early: the next kernel's launch
// begins as this grid's CTAs exit, which hides the launch and grid-teardown
// latency without parking the next grid's CTAs on SMs that are still busy.
// (An early trigger at the start of every kernel measured 559 us per decode
// step, no programmatic launch 525 us, this form 514 us; an early trigger in
// the layout's two small grids alone changed nothing.)  Stream order of all
// memory accesses is unchanged.
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}


// Lets the next kernel in the stream launch now (its CTAs park in their own
// pdl_begin until this grid has finished).  Used only by the layout kernels
// inside the combined dispatch call, right after their pdl_begin.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- status --
__device__ __forceinline__ void record_error(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

__device__ __forceinline__ int read_status(const int32_t* status) {
  return status ? *reinterpret_cast<const volatile int32_t*>(status) : 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------ acquire / release atoms --
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Release pattern for the chunk-completion counters: one fence.acq_rel.gpu,
// then relaxed gpu-scope adds.  Under the PTX memory model, observation order
// runs through every later atomic add on the same counter, so a consumer whose
// ld.acquire.gpu reads the final count synchronizes with each writer's fence
// and sees every row those writers published.  One fence per batch of adds
// keeps the release off the copy pipeline's critical path (an acq_rel atom per
// row costs a full fence each).
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ void atomic_add_relaxed_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atomic_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

// ------------------------------------------------------- work claiming --
// The kernels that split their work dynamically share one protocol over two
// caller-provided words: work[0] is a claim counter, work[1] counts CTAs
// that are done.  Both are zero when a launch starts.  CTA c first takes the
// fixed tickets [c*b, c*b + b) (no atomic, so its first loads go out at
// once); every later ticket is dyn0 + the old value of work[0] (dyn0 = G*b),
// claimed one ticket ahead so the atomic's latency is hidden.  Tickets past
// the work are discarded.  The last CTA to finish returns both words to
// zero: its acq_rel add on work[1] comes after every other CTA's, and each
// of those follows all of that CTA's claims.
struct TicketStream {  // one thread's view (the CTA's issuing thread)
  uint32_t* work;
  int64_t k_cur, k_end, dyn0;
  uint32_t pend;

  __device__ void init(uint32_t* w, int64_t first_batch) {
    work = w;
    k_cur = (int64_t)blockIdx.x * first_batch;
    k_end = k_cur + first_batch;
    dyn0 = (int64_t)gridDim.x * first_batch;
    pend = atomicAdd(w, 1u);
  }
  // Next ticket; a new claim is issued only while tickets below `limit`
  // may still exist.
  __device__ int64_t take(int64_t limit) {
    if (k_cur < k_end) return k_cur++;
    const int64_t k = dyn0 + (int64_t)pend;
    if (k < limit) pend = atomicAdd(work, 1u);
    return k;
  }
};

// Called once per CTA by its issuing thread after its last claim.
__device__ __forceinline__ void finish_claims(uint32_t* work) {
  if (atomic_add_acq_rel_gpu(work + 1, 1u) == gridDim.x - 1) {
    work[0] = 0u;
    work[1] = 0u;
  }
}

// ----------------------------------------------------------- shared mem --
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// --------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete; gives up after
// kWaitLimitNs and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ------------------------------------------------------------ bulk copies --
// Global -> this CTA's shared memory, completion counted on `bar` in bytes.
// Source, destination and size must be multiples of 16 bytes.  No multicast.
__device__ __forceinline__ void bulk_load_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Same, with an L2 cache policy (from make_policy_evict_last) on the source.
__device__ __forceinline__ void bulk_load_g2s_hint(void* smem_dst, const void* gsrc,
                                                   uint32_t bytes, uint64_t* bar,
                                                   uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_addr(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// L2 policy that keeps the lines it touches ahead of normal traffic.
__device__ __forceinline__ uint64_t make_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// This CTA's shared memory -> global, tracked by bulk async-groups.
__device__ __forceinline__ void bulk_store_s2g(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(gdst), "r"(smem_addr(smem_src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// All but the N most recent groups have finished READING shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// All but the N most recent groups have COMPLETED (writes performed).
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (bulk copy) reads of that memory.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders completed async-proxy global writes with later generic-proxy
// operations of this thread (the release that publishes them).
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// --------------------------------------------------------- vector access --
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// bf16 pair in a 32-bit word -> two exact floats
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// two floats -> bf16 pair, round to nearest even (cvt.rn.bf16x2.f32)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Warp-wide inclusive scan of an int.
__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += n;
  }
  return v;
}

// Block-wide exclusive scan of in[0..n) into out[0..n] (out[n] = total); any
// n >= 0: each thread sums a contiguous run of ceil(n / blockDim.x) items,
// the runs are scanned across the block, and each thread writes its run's
// prefixes.  blockDim.x must be a multiple of 32 and at most 1024; s_warp
// holds blockDim.x / 32 ints.  Every thread of the block must call it.
__device__ __forceinline__ void block_exclusive_scan(const int* in, int n, int* out,
                                                     int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int local = 0;
  for (int i = b0; i < b1; ++i) local += in[i];
  const int incl = warp_inclusive_scan(local);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < nw ? s_warp[lane] : 0;
    const int wi = warp_inclusive_scan(v);
    if (lane < nw) s_warp[lane] = wi - v;
  }
  __syncthreads();
  int run = s_warp[warp] + incl - local;
  for (int i = b0; i < b1; ++i) {
    const int v = in[i];
    out[i] = run;
    run += v;
  }
  if (b1 == n && b0 < b1) out[n] = run;
  if (n == 0 && tid == 0) out[0] = 0;
  __syncthreads();
}

}  // namespace moe

// ------------------------------------------------------------ host side --
namespace moe_host {

int sm_count(int device);
int current_device();
int launch_status();  // MOE_OK or MOE_ERR_CUDA from cudaGetLastError()

}  // namespace moe_host

// Host launchers shared by the separate calls and the combined dispatch call.
namespace moe {
int layout_launch(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                  int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                  int32_t* rank_offsets, int32_t* dst_row, int32_t* row_src,
                  uint32_t* tile_ready, int64_t P_cap, int32_t* d_status, void* workspace,
                  size_t workspace_bytes, cudaStream_t s, int trigger, int dry_run);
int permute_launch(const void* x, int dtype, int64_t T, int H, int64_t x_row_stride,
                   const float* x_scales, int64_t x_scales_row_stride, const int32_t* dst_row,
                   int K, const int32_t* expert_counts, const int32_t* expert_offsets, int E,
                   void* xp, float* xp_scales, int64_t P_cap, uint32_t* tile_ready,
                   uint32_t* work, int32_t* d_status, cudaStream_t s, int early_x, int dry_run);
}  // namespace moe

namespace moe_host {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launches with programmatic stream serialization allowed (see pdl_begin).
template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Resident blocks per SM of a kernel at a block size, looked up once per
// device and cached (safe to call from several host threads).
constexpr int kMaxCachedDevices = 64;
template <typename F>
int blocks_per_sm(F kernel, int threads, size_t dyn_smem, int device,
                  std::atomic<int>* cache /* [kMaxCachedDevices] */) {
  const bool cached = device >= 0 && device < kMaxCachedDevices;
  if (cached) {
    const int v = cache[device].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, dyn_smem) !=
          cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    n = 1;
  }
  if (cached) cache[device].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace moe_host
