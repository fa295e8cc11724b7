// Combined dispatch: the layout followed by the permute in one call (the
// DeepEP pull request's fused unzip takes the top-k ids and the token rows
// and produces the mapping table and the expert buffers in one step; the
// torch_npu npu_moe_distribute_combine API consumes that pair).
//
// The two layout kernels and the permute are launched back to back.  The
// layout kernels let the next kernel launch right after their own grid wait,
// and the permute issues its first batch of x-row loads before its grid wait:
// x is an input of this call, so it was complete before the first layout
// kernel's grid wait returned, which happened before the permute could
// launch.  Its CTAs therefore fill their rings while the layout still runs;
// everything the layout produces (row indices, counts, offsets) and the
// chunk-completion counters it resets are read or written only after the
// permute's grid wait.  Results are identical to moe_dispatch_layout
// followed by moe_dispatch_permute.
#include "common.cuh"

extern "C" int moe_dispatch(const int32_t* topk_idx, int64_t T, int K, int E, int R,
                            const void* x, int dtype, int H, int64_t x_row_stride,
                            const float* x_scales, int64_t x_scales_row_stride,
                            int32_t* expert_counts, int32_t* expert_offsets,
                            int32_t* rank_counts, int32_t* rank_offsets, int32_t* dst_row,
                            int32_t* row_src, uint32_t* tile_ready, int64_t P_cap,
                            void* workspace, size_t workspace_bytes, void* xp,
                            float* xp_scales, uint32_t* work, int32_t* d_status, void* stream) {
  using namespace moe;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // every check first, so an argument error launches nothing
  int st = layout_launch(topk_idx, T, K, E, R, expert_counts, expert_offsets, rank_counts,
                         rank_offsets, dst_row, row_src, tile_ready, P_cap, d_status, workspace,
                         workspace_bytes, s, 1, 1);
  if (st != MOE_OK) return st;
  st = permute_launch(x, dtype, T, H, x_row_stride, x_scales, x_scales_row_stride, dst_row, K,
                      expert_counts, expert_offsets, E, xp, xp_scales, P_cap, tile_ready, work,
                      d_status, s, 1, 1);
  if (st != MOE_OK) return st;
  st = layout_launch(topk_idx, T, K, E, R, expert_counts, expert_offsets, rank_counts,
                     rank_offsets, dst_row, row_src, tile_ready, P_cap, d_status, workspace,
                     workspace_bytes, s, 1, 0);
  if (st != MOE_OK) return st;
  return permute_launch(x, dtype, T, H, x_row_stride, x_scales, x_scales_row_stride, dst_row, K,
                        expert_counts, expert_offsets, E, xp, xp_scales, P_cap, tile_ready, work,
                        d_status, s, 1, 0);
}
