// Host-side helpers shared by the entry points: device queries, status
// strings, sizing functions.
#include <atomic>

#include "common.cuh"

namespace moe_host {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
}  // namespace

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

int sm_count(int device) {
  if (device < 0 || device >= kMaxDevices) return 148;
  int v = g_sm_count[device].load(std::memory_order_relaxed);
  if (v > 0) return v;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
    n = 148;
  g_sm_count[device].store(n, std::memory_order_relaxed);
  return n;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe_host

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_EXPERT_RANGE: return "expert id out of range";
    case MOE_ERR_DUPLICATE_EXPERT: return "expert id repeated within a token";
    case MOE_ERR_CAPACITY: return "padded capacity too small";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_BOUNDS: return "row index outside its buffer";
    default: return "unknown status";
  }
}

int moe_version(void) { return 100; }

int64_t moe_padded_capacity(int64_t T, int K, int E) {
  if (T < 0 || K < 1 || K > MOE_MAX_TOPK || E < 1 || E > MOE_MAX_EXPERTS) return -1;
  const int64_t n = T * (int64_t)K;
  const int64_t ne = n < (int64_t)E ? n : (int64_t)E;
  const int64_t cap = n + (int64_t)(MOE_TILE_M - 1) * ne;
  return (cap + MOE_TILE_M - 1) / MOE_TILE_M * MOE_TILE_M;
}

}  // extern "C"
