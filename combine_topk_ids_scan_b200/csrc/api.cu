// api.cu -- the extern "C" entry points of libmoedc.so declared in
// include/moe_dc.h: host-side validation of the problem and the pointers,
// then kernel launches on the caller's stream.  Nothing here allocates or
// synchronises.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "internal.h"
#include "moe_dc.h"

namespace moe {

int device_sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace moe

namespace {

constexpr int64_t kU32Max = 4294967295ll;

static_assert(sizeof(moe_trace_record) == 32, "moe_trace_record is 32 bytes");

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validates the problem and fills the derived sizes.
moe_status make_shape(const moe_problem *p, moe::Shape *s) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens < 0 || p->hidden <= 0 || p->num_experts <= 0 || p->top_k <= 0 ||
      p->num_segments <= 0 || p->expert_capacity < 0 || p->recv_capacity < 0 ||
      p->expert_pad_multiple < 0 || (p->expert_pad_multiple > 1 && p->expert_capacity > 0))
    return MOE_ERR_INVALID_ARG;
  if (p->num_experts > MOE_MAX_EXPERTS || p->top_k > MOE_MAX_TOPK ||
      p->num_experts % p->num_segments != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  s->N = p->num_tokens;
  s->H = p->hidden;
  s->E = p->num_experts;
  s->k = p->top_k;
  s->S = p->num_segments;
  s->Ce = p->expert_capacity;
  s->C = p->expert_capacity > 0 ? 0 : p->recv_capacity;
  s->rows = p->expert_capacity > 0 ? (int64_t)p->num_experts * p->expert_capacity
                                   : p->recv_capacity;
  s->P = (int64_t)p->num_tokens * p->top_k;
  s->flags = p->flags;
  s->pad = p->expert_pad_multiple > 1 ? p->expert_pad_multiple : 1;
  // slots are int32; the [4, S] table counts elements in uint32; padded
  // expert blocks add at most E * (pad - 1) rows
  const int64_t padded = s->P + (int64_t)s->E * (s->pad - 1);
  if (s->rows > 2147483647ll || padded > 2147483647ll) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->rows * s->H > kU32Max || padded * s->H > kU32Max) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace

namespace moe {

moe_status check_layout_args(const moe_problem *problem, const int32_t *topk_ids,
                             const int32_t *expert_counts, const int32_t *expert_offsets,
                             const uint32_t *meta, const int32_t *row_src,
                             const int32_t *pair_slot, const uint32_t *status, Shape *s) {
  moe_status st = make_shape(problem, s);
  if (st != MOE_OK) return st;
  if (!expert_counts || !expert_offsets || !meta || !status) return MOE_ERR_INVALID_ARG;
  if (s->P > 0 && (!topk_ids || !pair_slot)) return MOE_ERR_INVALID_ARG;
  if (s->rows > 0 && !row_src) return MOE_ERR_INVALID_ARG;
  if (!aligned(topk_ids, 4) || !aligned(expert_counts, 4) || !aligned(expert_offsets, 4) ||
      !aligned(meta, 4) || !aligned(row_src, 4) || !aligned(pair_slot, 4) || !aligned(status, 4))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace moe

extern "C" {

int64_t moe_output_rows(const moe_problem *problem) {
  moe::Shape s;
  if (make_shape(problem, &s) != MOE_OK) return -1;
  return s.rows;
}

size_t moe_workspace_bytes(const moe_problem *problem) {
  moe::Shape s;
  if (make_shape(problem, &s) != MOE_OK) return 0;
  return moe::layout_workspace_bytes(s);
}

moe_status moe_dispatch_layout(const moe_problem *problem, const int32_t *topk_ids,
                               int32_t *expert_counts, int32_t *expert_offsets,
                               uint32_t *meta, int32_t *row_src, int32_t *pair_slot,
                               uint8_t *drop_mask, uint32_t *status, void *workspace,
                               moe_stream_t stream) {
  moe::Shape s;
  moe_status st = moe::check_layout_args(problem, topk_ids, expert_counts, expert_offsets, meta,
                                         row_src, pair_slot, status, &s);
  if (st != MOE_OK) return st;
  if (!workspace || !aligned(workspace, 16)) return MOE_ERR_INVALID_ARG;
  moe::LayoutWorkspace ws = moe::layout_workspace_view(s, workspace);
  return from_cuda(moe::launch_layout(s, topk_ids, expert_counts, expert_offsets, meta, row_src,
                                      pair_slot, drop_mask, status, ws,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_problem *problem, const void *hidden_states,
                       const int32_t *row_src, const int32_t *pair_slot, void *out,
                       moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !out || (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden_states, 16) || !aligned(out, 16) || !aligned(row_src, 4) ||
      !aligned(pair_slot, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_bf16(s, hidden_states, row_src, pair_slot, out,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_to_peers(const moe_problem *problem, const void *hidden_states,
                                const int32_t *row_src, const int32_t *pair_slot,
                                const uint32_t *meta, void *const *peer_out,
                                const int64_t *put_offsets, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !peer_out || !put_offsets || (s.Ce == 0 && !meta) ||
      (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden_states, 16) || !aligned(row_src, 4) || !aligned(pair_slot, 4) ||
      !aligned(meta, 4) || !aligned(peer_out, 8) || !aligned(put_offsets, 8))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_to_peers(s, hidden_states, row_src, pair_slot, meta,
                                                peer_out, put_offsets,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_quant_fp8_to_peers(const moe_problem *problem, const void *hidden_states,
                                          const int32_t *row_src, const int32_t *pair_slot,
                                          const uint32_t *meta, void *const *peer_codes,
                                          void *const *peer_scales, const int64_t *put_offsets,
                                          moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !peer_codes || !peer_scales || !put_offsets || (s.Ce == 0 && !meta) ||
      (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden_states, 16) || !aligned(row_src, 4) || !aligned(pair_slot, 4) ||
      !aligned(meta, 4) || !aligned(peer_codes, 8) || !aligned(peer_scales, 8) ||
      !aligned(put_offsets, 8))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_fp8_to_peers(s, hidden_states, row_src, pair_slot, meta,
                                                    peer_codes, peer_scales, put_offsets,
                                                    reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_quant_nvfp4_to_peers(const moe_problem *problem,
                                            const void *hidden_states, const int32_t *row_src,
                                            const int32_t *pair_slot, const uint32_t *meta,
                                            const float *global_scale, void *const *peer_codes,
                                            void *const *peer_scales, const int64_t *put_offsets,
                                            moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 32 != 0 || (s.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !peer_codes || !peer_scales || !put_offsets || !global_scale ||
      (s.Ce == 0 && !meta) || (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden_states, 16) || !aligned(row_src, 4) || !aligned(pair_slot, 4) ||
      !aligned(meta, 4) || !aligned(global_scale, 4) || !aligned(peer_codes, 8) ||
      !aligned(peer_scales, 8) || !aligned(put_offsets, 8))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_nvfp4_to_peers(
      s, hidden_states, row_src, pair_slot, meta, global_scale, peer_codes, peer_scales,
      put_offsets, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_premultiplied(const moe_problem *problem, const void *hidden_states,
                                     const int32_t *row_src, const int32_t *pair_slot,
                                     const float *gates, void *out, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !out || (s.P > 0 && (!hidden_states || !pair_slot || !gates)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden_states, 16) || !aligned(out, 16) || !aligned(row_src, 4) ||
      !aligned(pair_slot, 4) || !aligned(gates, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_premultiplied(s, hidden_states, row_src, pair_slot, gates,
                                                     out, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_quant_fp8(const moe_problem *problem, const void *hidden_states,
                                 const int32_t *row_src, const int32_t *pair_slot,
                                 uint8_t *out_e4m3, float *scales, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !out_e4m3 || !scales || (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden_states, 16) || !aligned(out_e4m3, 16) || !aligned(scales, 4) ||
      !aligned(row_src, 4) || !aligned(pair_slot, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_fp8(s, hidden_states, row_src, pair_slot, out_e4m3,
                                           scales, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_quant_nvfp4(const moe_problem *problem, const void *hidden_states,
                                   const int32_t *row_src, const int32_t *pair_slot,
                                   const float *global_scale, uint8_t *out_e2m1,
                                   uint8_t *scales_e4m3, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !out_e2m1 || !scales_e4m3 || !global_scale ||
      (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  const uintptr_t scale_align = (s.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES) ? 4 : 2;
  if (!aligned(hidden_states, 16) || !aligned(out_e2m1, 16) ||
      !aligned(scales_e4m3, scale_align) || !aligned(global_scale, 4) || !aligned(row_src, 4) ||
      !aligned(pair_slot, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_nvfp4(s, hidden_states, row_src, pair_slot, global_scale,
                                             out_e2m1, scales_e4m3,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_quant_mxfp4(const moe_problem *problem, const void *hidden_states,
                                   const int32_t *row_src, const int32_t *pair_slot,
                                   uint8_t *out_e2m1, uint8_t *scales_e8m0, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  if (!row_src || !out_e2m1 || !scales_e8m0 || (s.P > 0 && (!hidden_states || !pair_slot)))
    return MOE_ERR_INVALID_ARG;
  const uintptr_t scale_align = (s.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES) ? 4 : 1;
  if (!aligned(hidden_states, 16) || !aligned(out_e2m1, 16) ||
      !aligned(scales_e8m0, scale_align) || !aligned(row_src, 4) || !aligned(pair_slot, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_permute_mxfp4(s, hidden_states, row_src, pair_slot, out_e2m1,
                                             scales_e8m0,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_problem *problem, const void *expert_out, const float *gates,
                       const int32_t *pair_slot, void *out, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.N == 0) return MOE_OK;
  if (!out || !gates || !pair_slot || (s.rows > 0 && !expert_out)) return MOE_ERR_INVALID_ARG;
  if (!aligned(expert_out, 16) || !aligned(out, 16) || !aligned(gates, 4) ||
      !aligned(pair_slot, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine(s, expert_out, gates, pair_slot, out,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine_from_peers(const moe_problem *problem, const void *const *peer_expert_out,
                                  const int64_t *get_offsets, const uint32_t *meta,
                                  const float *gates, const int32_t *pair_slot, void *out,
                                  moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.N == 0) return MOE_OK;
  if (!out || !gates || !pair_slot || !peer_expert_out || !get_offsets || (s.Ce == 0 && !meta))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(peer_expert_out, 8) || !aligned(get_offsets, 8) || !aligned(meta, 4) ||
      !aligned(gates, 4) || !aligned(pair_slot, 4) || !aligned(out, 16))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine_from_peers(s, peer_expert_out, get_offsets, meta, gates,
                                                  pair_slot, out,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_backward(const moe_problem *problem, const void *grad_out,
                                const int32_t *pair_slot, void *grad_hidden,
                                moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.N == 0) return MOE_OK;
  if (!grad_hidden || !pair_slot || (s.rows > 0 && !grad_out)) return MOE_ERR_INVALID_ARG;
  if (!aligned(grad_out, 16) || !aligned(grad_hidden, 16) || !aligned(pair_slot, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine(s, grad_out, nullptr, pair_slot, grad_hidden,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine_backward(const moe_problem *problem, const void *grad_y,
                                const void *expert_out, const float *gates,
                                const int32_t *pair_slot, const int32_t *row_src,
                                void *grad_expert_out, float *grad_gates, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (s.H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.N == 0 && s.rows == 0) return MOE_OK;
  if ((s.N > 0 && (!grad_y || !gates || !pair_slot || !grad_gates)) ||
      (s.rows > 0 && (!expert_out || !row_src || !grad_expert_out)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(grad_y, 16) || !aligned(expert_out, 16) || !aligned(grad_expert_out, 16) ||
      !aligned(gates, 4) || !aligned(grad_gates, 4) || !aligned(pair_slot, 4) ||
      !aligned(row_src, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine_backward(s, grad_y, expert_out, gates, pair_slot, row_src,
                                                grad_expert_out, grad_gates,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_swiglu_quant(const moe_problem *problem, int32_t intermediate, uint32_t format,
                            uint32_t gate_up_layout, const void *gate_up,
                            const int32_t *row_src, const float *global_scale,
                            uint8_t *codes, uint8_t *scales, moe_stream_t stream) {
  moe::Shape s;
  moe_status st = make_shape(problem, &s);
  if (st != MOE_OK) return st;
  if (intermediate <= 0 || format > MOE_QUANT_MXFP6_E3M2 ||
      gate_up_layout > MOE_GATE_UP_INTERLEAVED)
    return MOE_ERR_INVALID_ARG;
  if (intermediate % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int64_t I = intermediate;
  if (s.rows * 2 * I > 2147483647ll * 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s.rows == 0) return MOE_OK;
  const bool has_scales = format != MOE_QUANT_BF16;
  if (!gate_up || !row_src || !codes || (has_scales && !scales) ||
      (format == MOE_QUANT_NVFP4 && !global_scale))
    return MOE_ERR_INVALID_ARG;
  const bool fp6 = format == MOE_QUANT_MXFP6_E2M3 || format == MOE_QUANT_MXFP6_E3M2;
  if (!aligned(gate_up, 16) || !aligned(codes, fp6 ? 8 : 16) ||
      (has_scales && !aligned(scales, format == MOE_QUANT_NVFP4 ? 2 : 1)) ||
      (global_scale && !aligned(global_scale, 4)) || !aligned(row_src, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_swiglu_quant(s, intermediate, format,
                                            gate_up_layout == MOE_GATE_UP_INTERLEAVED, gate_up,
                                            row_src, global_scale, codes, scales,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

const char *moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK:
      return "ok";
    case MOE_ERR_INVALID_ARG:
      return "invalid argument (null or misaligned pointer, negative size, bad field)";
    case MOE_ERR_UNSUPPORTED_SHAPE:
      return "unsupported shape (size outside the library's limits)";
    case MOE_ERR_CUDA:
      return "CUDA error while launching";
    case MOE_ERR_NOT_BUILT:
      return "not in this build (see the build options in moe_dc.h)";
    default:
      return "unknown status";
  }
}

const char *moe_version(void) {
#if defined(MOE_DEBUG_CHECKS) && defined(MOE_TRACE)
  return "moedc 0.2.0 (sm_100a, device index checks, trace records)";
#elif defined(MOE_DEBUG_CHECKS)
  return "moedc 0.2.0 (sm_100a, device index checks)";
#elif defined(MOE_TRACE)
  return "moedc 0.2.0 (sm_100a, trace records)";
#else
  return "moedc 0.2.0 (sm_100a)";
#endif
}

moe_status moe_trace_attach(moe_trace_record *records, uint32_t capacity, uint32_t *count,
                            moe_stream_t stream) {
#ifdef MOE_TRACE
  if (records != nullptr && (count == nullptr || capacity == 0)) return MOE_ERR_INVALID_ARG;
  if (!aligned(records, 8) || !aligned(count, 4)) return MOE_ERR_INVALID_ARG;
  if (records == nullptr) {
    count = nullptr;
    capacity = 0;
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err = moe::trace_attach_layout(records, count, capacity, st);
  if (err == cudaSuccess) err = moe::trace_attach_permute(records, count, capacity, st);
  if (err == cudaSuccess) err = moe::trace_attach_combine(records, count, capacity, st);
  if (err == cudaSuccess) err = moe::trace_attach_swiglu(records, count, capacity, st);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
#else
  (void)records;
  (void)capacity;
  (void)count;
  (void)stream;
  return MOE_ERR_NOT_BUILT;
#endif
}

int64_t moe_debug_violations(int reset) {
#ifdef MOE_DEBUG_CHECKS
  return (int64_t)(moe::debug_violations_layout(reset != 0) |
                   moe::debug_violations_permute(reset != 0) |
                   moe::debug_violations_combine(reset != 0) |
                   moe::debug_violations_swiglu(reset != 0));
#else
  (void)reset;
  return -1;
#endif
}

}  // extern "C"
