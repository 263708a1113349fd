// internal.h -- host-side interface between the C-ABI layer and the kernel
// launchers of libmoedc.  Not installed; the public interface is moe_dc.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "moe_dc.h"

namespace moe {

// Problem sizes after host validation.
struct Shape {
  int32_t N, H, E, k, S, Ce;
  int64_t C;     // packed recv_capacity (0 in capacity mode)
  int64_t rows;  // rows of the dispatch output
  int64_t P;     // N * k pairs
  uint32_t flags;
  int32_t pad;   // per-expert row multiple (1 = none)
};

// Layout workspace: control words, per-expert totals, scan tile states.
struct LayoutWorkspace {
  uint32_t *ctrl;    // [0] tile ticket, [1] emit blocks done, [2] status bits
  int32_t *totals;   // [E] routed pairs per expert (written by the last tile)
  uint64_t *tiles;   // [T * E] scan tile states (flag << 32 | value)
  int32_t num_tiles; // T
};

// Host checks of moe_dispatch_layout's problem and pointers (everything but
// the workspace); fills *s on success.  Launches nothing.
moe_status check_layout_args(const moe_problem *problem, const int32_t *topk_ids,
                             const int32_t *expert_counts, const int32_t *expert_offsets,
                             const uint32_t *meta, const int32_t *row_src,
                             const int32_t *pair_slot, const uint32_t *status, Shape *s);

int32_t layout_num_tiles(int64_t P);
size_t layout_workspace_bytes(const Shape &s);
LayoutWorkspace layout_workspace_view(const Shape &s, void *workspace);

cudaError_t launch_layout(const Shape &s, const int32_t *ids, int32_t *expert_counts,
                          int32_t *expert_offsets, uint32_t *meta, int32_t *row_src,
                          int32_t *pair_slot, uint8_t *drop_mask, uint32_t *status,
                          const LayoutWorkspace &ws, cudaStream_t stream);

cudaError_t launch_permute_bf16(const Shape &s, const void *hidden, const int32_t *row_src,
                                const int32_t *pair_slot, void *out, cudaStream_t stream);

cudaError_t launch_permute_to_peers(const Shape &s, const void *hidden, const int32_t *row_src,
                                    const int32_t *pair_slot, const uint32_t *meta,
                                    void *const *peer_out, const int64_t *put_offsets,
                                    cudaStream_t stream);

cudaError_t launch_permute_premultiplied(const Shape &s, const void *hidden,
                                         const int32_t *row_src, const int32_t *pair_slot,
                                         const float *gates, void *out, cudaStream_t stream);

cudaError_t launch_permute_fp8_to_peers(const Shape &s, const void *hidden,
                                       const int32_t *row_src, const int32_t *pair_slot,
                                       const uint32_t *meta, void *const *peer_codes,
                                       void *const *peer_scales, const int64_t *put_offsets,
                                       cudaStream_t stream);
cudaError_t launch_permute_nvfp4_to_peers(const Shape &s, const void *hidden,
                                         const int32_t *row_src, const int32_t *pair_slot,
                                         const uint32_t *meta, const float *global_scale,
                                         void *const *peer_codes, void *const *peer_scales,
                                         const int64_t *put_offsets, cudaStream_t stream);
cudaError_t launch_permute_fp8(const Shape &s, const void *hidden, const int32_t *row_src,
                               const int32_t *pair_slot, uint8_t *q, float *scales,
                               cudaStream_t stream);

cudaError_t launch_permute_nvfp4(const Shape &s, const void *hidden, const int32_t *row_src,
                                 const int32_t *pair_slot, const float *global_scale,
                                 uint8_t *q, uint8_t *scales, cudaStream_t stream);

cudaError_t launch_permute_mxfp4(const Shape &s, const void *hidden, const int32_t *row_src,
                                 const int32_t *pair_slot, uint8_t *q, uint8_t *scales,
                                 cudaStream_t stream);

// gates == nullptr: unit weights (the dispatch backward)
cudaError_t launch_combine_from_peers(const Shape &s, const void *const *peer_expert_out,
                                      const int64_t *get_offsets, const uint32_t *meta,
                                      const float *gates, const int32_t *pair_slot, void *out,
                                      cudaStream_t stream);
cudaError_t launch_combine(const Shape &s, const void *expert_out, const float *gates,
                           const int32_t *pair_slot, void *out, cudaStream_t stream);

cudaError_t launch_combine_backward(const Shape &s, const void *grad_y, const void *expert_out,
                                    const float *gates, const int32_t *pair_slot,
                                    const int32_t *row_src, void *grad_expert_out,
                                    float *grad_gates, cudaStream_t stream);

cudaError_t launch_swiglu_quant(const Shape &s, int32_t I, uint32_t format, bool interleaved,
                                const void *gate_up, const int32_t *row_src,
                                const float *global_scale, uint8_t *codes, uint8_t *scales,
                                cudaStream_t stream);

// Each kernel file's debug word (MOE_DEBUG_CHECKS builds; 0 otherwise),
// zeroed when `reset`.
uint32_t debug_violations_layout(bool reset);
uint32_t debug_violations_permute(bool reset);
uint32_t debug_violations_combine(bool reset);
uint32_t debug_violations_swiglu(bool reset);

// Each kernel translation unit's trace attachment (the build with
// -DMOE_TRACE; trace.cuh).
#ifdef MOE_TRACE
cudaError_t trace_attach_layout(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                                cudaStream_t stream);
cudaError_t trace_attach_permute(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                                 cudaStream_t stream);
cudaError_t trace_attach_combine(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                                 cudaStream_t stream);
cudaError_t trace_attach_swiglu(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                                cudaStream_t stream);
#endif

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Resident CTAs per SM of one kernel configuration, queried once per device
// (devices 0..kMaxDevices-1; others are queried on every call).  Each launch
// site keeps its own cache (one per kernel instantiation).
constexpr int kMaxDevices = 64;
struct OccupancyCache {
  std::atomic<int> per_sm[kMaxDevices] = {};
};
inline int resident_ctas(OccupancyCache &cache, const void *kernel, int threads, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (dev >= 0 && dev < kMaxDevices) {
    const int v = cache.per_sm[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
      n < 1)
    n = 1;
  if (dev >= 0 && dev < kMaxDevices) cache.per_sm[dev].store(n, std::memory_order_relaxed);
  return n;
}

// kernel<<<grid, block, smem, stream>>>(args...) with programmatic dependent
// launch allowed (see grid_dependency_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe
