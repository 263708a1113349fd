// noalloc.cu -- moe_dispatch_layout_noalloc: the dispatch layout for callers
// that cannot allocate device memory.  Its scratch (the layout workspace) is a
// fixed-size array in the library's own device memory instead of a buffer the
// caller allocates; everything else is moe_dispatch_layout unchanged.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "moe_dc.h"

namespace {

// The scratch.  Every GPU that loads the library holds these bytes until the
// process exits.  In host code this name is only a stand-in for the symbol,
// not a device address: the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of the scratch, per device

// Device address of the scratch on the current device; looked up once per
// device (the first call on a device, with that device current).
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_dispatch_layout_noalloc(
    const moe_problem *problem, const int32_t *topk_ids, int32_t *expert_counts,
    int32_t *expert_offsets, uint32_t *meta, int32_t *row_src, int32_t *pair_slot,
    uint8_t *drop_mask, uint32_t *status, moe_stream_t stream) {
  // the layout's own host checks first: nothing is enqueued for bad arguments
  moe::Shape s;
  const moe_status st = moe::check_layout_args(problem, topk_ids, expert_counts, expert_offsets,
                                               meta, row_src, pair_slot, status, &s);
  if (st != MOE_OK) return st;
  const size_t need = moe::layout_workspace_bytes(s);
  if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED_SHAPE;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  // All calls share the scratch and it keeps what the last call left there;
  // the layout needs its part zero-filled, so clear it on this call's stream.
  if (cudaMemsetAsync(scratch, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_dispatch_layout(problem, topk_ids, expert_counts, expert_offsets, meta, row_src,
                             pair_slot, drop_mask, status, scratch, stream);
}
