// trace.cuh -- per-CTA trace records (the build with -DMOE_TRACE).
//
// Every kernel opens with MOE_TRACE_CTA(kernel id, variant).  In the trace
// build that declares a TraceCta: thread 0 takes the next slot of the
// attached record buffer and stamps the CTA's start; when the object goes
// out of scope (on every return path of the kernel) the first active lane of
// each warp raises the record's end to its own finishing time, so end_ns is
// the time the CTA's last warp finished.  In other builds the macro is an
// empty statement and the kernels hold no trace code.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_dc.h"

namespace moe {

#ifdef MOE_TRACE
// Where this translation unit's kernels append records (records == nullptr:
// not tracing); set by trace_attach_tu.
struct TraceTarget {
  moe_trace_record *records;
  uint32_t *count;
  uint32_t capacity;
};
static __device__ TraceTarget g_trace;  // one per translation unit

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

class TraceCta {
 public:
  __device__ TraceCta(uint32_t kernel, uint32_t variant) {
    __shared__ moe_trace_record *s_rec;
    if (threadIdx.x == 0) {
      const uint64_t t0 = global_timer_ns();
      const TraceTarget tg = g_trace;
      moe_trace_record *r = nullptr;
      if (tg.records != nullptr) {
        const uint32_t i = atomicAdd(tg.count, 1u);
        if (i < tg.capacity) {
          r = tg.records + i;
          uint64_t grid;
          uint32_t sm;
          asm volatile("mov.u64 %0, %%gridid;" : "=l"(grid));
          asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
          r->start_ns = t0;
          r->grid = grid;
          r->block = blockIdx.x;
          r->smid = (uint16_t)sm;
          r->kernel = (uint8_t)kernel;
          r->variant = (uint8_t)variant;
          // an atomic, so that the warps' atomic maxima are ordered after it
          atomicExch(reinterpret_cast<unsigned long long *>(&r->end_ns),
                     (unsigned long long)t0);
        }
      }
      s_rec = r;
    }
    __syncthreads();
    rec_ = s_rec;
  }
  __device__ ~TraceCta() {
    if (rec_ == nullptr) return;
    const uint32_t active = __activemask();
    if ((int)(threadIdx.x % 32u) == __ffs(active) - 1)
      atomicMax(reinterpret_cast<unsigned long long *>(&rec_->end_ns),
                (unsigned long long)global_timer_ns());
  }
  TraceCta(const TraceCta &) = delete;
  TraceCta &operator=(const TraceCta &) = delete;

 private:
  moe_trace_record *rec_;
};

// Point this translation unit's kernels at a record buffer (host only; a
// copy enqueued on `stream`).
static inline cudaError_t trace_attach_tu(moe_trace_record *records, uint32_t *count,
                                          uint32_t capacity, cudaStream_t stream) {
  const TraceTarget t{records, count, capacity};
  return cudaMemcpyToSymbolAsync(g_trace, &t, sizeof(t), 0, cudaMemcpyHostToDevice, stream);
}

#define MOE_TRACE_CTA(kernel, variant) ::moe::TraceCta moe_trace_cta_((kernel), (variant))
#else
#define MOE_TRACE_CTA(kernel, variant) ((void)0)
#endif

}  // namespace moe
