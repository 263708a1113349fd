// combine.cu -- gather each token's k expert-output rows back and sum them
// weighted by the token's gates: fp32 fused multiply-adds in fixed j order,
// one round-to-nearest-even to bf16 at the end.
//
// Definitions: DeepSpeed combine docstring (gather each token's expert results
// back and weight them by the gate values); NeMo AutoModel TokenDispatcher
// config moe_router_dtype = 'fp32' (routing weights and the weighted average
// in fp32); Mojo MAX ep_comm router_weights_wrapper_type (an fp32 weight per
// (token, k)).
//
// One warp per token (persistent grid).  Lane j < k fetches the pair's row
// and gate, shuffles broadcast them; per step each lane loads one 16-byte
// vector (8 bf16) from every live row -- U steps at once, so up to k*U
// independent 16-byte loads per lane are in flight -- and writes one 16-byte
// vector of the result.  With few tokens (fewer than the resident warps) a
// token's row is split into `splits` column spans of `span` vectors, one
// warp each, so that small batches still fill the GPU; every output element
// is the same fma chain whatever the split.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "trace.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kFull = 0xFFFFFFFFu;

template <int KMAX, int U>
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const uint4 *__restrict__ x, const float *__restrict__ gates,
                   const int32_t *__restrict__ pair_slot, uint4 *__restrict__ out, int32_t N,
                   int32_t k, int64_t rows, int32_t vecs, int32_t splits, int32_t span) {
  MOE_TRACE_CTA(gates ? MOE_TRACE_COMBINE : MOE_TRACE_PERMUTE_BACKWARD, KMAX);
  allow_dependents();
  grid_dependency_wait();
  const int lane = threadIdx.x % kWarp;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) / kWarp;

  for (int64_t item = gw; item < (int64_t)N * splits; item += nw) {
    const int64_t t = item / splits;
    const int32_t vb = (int32_t)(item % splits) * span;
    const int32_t ve = min(vecs, vb + span);
    int32_t my_slot = -1;
    float my_w = 0.0f;
    if (lane < k) {
      const int32_t s = __ldg(pair_slot + t * k + lane);
      if (s >= 0 && s < rows) {
        my_slot = s;
        // no gates: unit weights (the dispatch backward); fmaf(1, x, acc)
        // is exactly acc + x
        my_w = gates ? __ldg(gates + t * k + lane) : 1.0f;
      }
    }
    int64_t row[KMAX];
    float w[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int32_t s = __shfl_sync(kFull, my_slot, j);
      row[j] = s >= 0 && MOE_IN_RANGE(s, rows, kDbgCombineRow) ? s : -1;
      w[j] = __shfl_sync(kFull, my_w, j);
    }
    uint4 *dst = out + t * vecs;
    for (int v0 = vb; v0 < ve; v0 += kWarp * U) {
      uint4 in[KMAX][U];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * kWarp + lane;
          in[j][u] = (row[j] >= 0 && v < ve) ? ld_stream_v4(x + row[j] * vecs + v)
                                              : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * kWarp + lane;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (row[j] < 0) continue;
          const uint32_t e[4] = {in[j][u].x, in[j][u].y, in[j][u].z, in[j][u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(w[j], bf16lo(e[i]), acc[2 * i]);
            acc[2 * i + 1] = fmaf(w[j], bf16hi(e[i]), acc[2 * i + 1]);
          }
        }
        if (v < ve)
          st_v4(dst + v, make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7])));
      }
    }
  }
}

// Combine fused with the expert-parallel return (the reverse of the fused
// send): the expert output of local row r of segment s is read straight from
// rank s's expert-output buffer peer_x[s] at row get[s] + (r - start_s) --
// where that rank received the row -- instead of being shipped back first.
// combine_kernel's units, loads and fp32 fma order, so the result is the
// one moe_combine gives on the returned rows.  Each CTA stages the S segment
// starts and sizes, get offsets and buffer addresses in shared memory (24
// bytes per rank); a lane holding pair j resolves its row's source address
// and the warp broadcasts the k addresses.
template <int KMAX, int U>
__global__ void __launch_bounds__(kThreads)
    combine_from_peers_kernel(const uint4 *const *__restrict__ peer_x,
                              const int64_t *__restrict__ get, const uint32_t *__restrict__ meta,
                              const float *__restrict__ gates,
                              const int32_t *__restrict__ pair_slot, uint4 *__restrict__ out,
                              int32_t N, int32_t k, int64_t rows, int32_t vecs, int32_t splits,
                              int32_t span, int32_t S, int32_t H, int32_t static_seg_rows) {
  MOE_TRACE_CTA(MOE_TRACE_COMBINE_FROM_PEERS, KMAX);
  allow_dependents();
  extern __shared__ uint64_t peer_smem[];
  const uint4 **s_ptr = reinterpret_cast<const uint4 **>(peer_smem);
  int64_t *s_get = reinterpret_cast<int64_t *>(peer_smem + S);
  int32_t *s_start = reinterpret_cast<int32_t *>(peer_smem + 2 * S);
  int32_t *s_rows = s_start + S;
  grid_dependency_wait();
  for (int i = threadIdx.x; i < S; i += kThreads) {
    s_ptr[i] = peer_x[i];
    s_get[i] = __ldg(get + i);
    if (static_seg_rows > 0) {
      s_start[i] = i * static_seg_rows;
      s_rows[i] = static_seg_rows;
    } else {
      s_start[i] = (int32_t)(__ldg(meta + S + i) / (uint32_t)H);
      s_rows[i] = (int32_t)(__ldg(meta + i) / (uint32_t)H);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x % kWarp;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) / kWarp;

  for (int64_t item = gw; item < (int64_t)N * splits; item += nw) {
    const int64_t t = item / splits;
    const int32_t vb = (int32_t)(item % splits) * span;
    const int32_t ve = min(vecs, vb + span);
    const uint4 *my_src = nullptr;
    float my_w = 0.0f;
    if (lane < k) {
      const int32_t r = __ldg(pair_slot + t * k + lane);
      if (r >= 0 && r < rows && MOE_IN_RANGE(r, rows, kDbgCombineRow)) {
        int lo = 0, hi = S - 1;  // last segment starting at or before r
        while (lo < hi) {
          const int mid = (lo + hi + 1) / 2;
          if (s_start[mid] <= r) lo = mid;
          else hi = mid - 1;
        }
        if (r >= s_start[lo] && r - s_start[lo] < s_rows[lo]) {
          my_src = s_ptr[lo] + (s_get[lo] + (r - s_start[lo])) * (int64_t)vecs;
          my_w = __ldg(gates + t * k + lane);
        }
      }
    }
    const uint4 *src[KMAX];
    float w[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      src[j] = reinterpret_cast<const uint4 *>(
          __shfl_sync(kFull, reinterpret_cast<unsigned long long>(my_src), j));
      w[j] = __shfl_sync(kFull, my_w, j);
    }
    uint4 *dst = out + t * vecs;
    for (int v0 = vb; v0 < ve; v0 += kWarp * U) {
      uint4 in[KMAX][U];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * kWarp + lane;
          in[j][u] = (src[j] != nullptr && v < ve) ? ld_stream_v4(src[j] + v)
                                                   : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * kWarp + lane;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (src[j] == nullptr) continue;
          const uint32_t e[4] = {in[j][u].x, in[j][u].y, in[j][u].z, in[j][u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(w[j], bf16lo(e[i]), acc[2 * i]);
            acc[2 * i + 1] = fmaf(w[j], bf16hi(e[i]), acc[2 * i + 1]);
          }
        }
        if (v < ve)
          st_v4(dst + v, make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7])));
      }
    }
  }
}

// Combine backward.  y[t] = sum_j w[t,j] x[slot(t,j)], so the expert rows get
// grad_x[slot(t,j)] = bf16(w[t,j] * grad_y[t]) and the gates get
// grad_w[t,j] = <grad_y[t], x[slot(t,j)]>.  One warp per token: per step a
// lane loads two 16-byte vectors (32 columns apart) of grad_y and of each
// live row -- all of them before any store of the step, so 2(k+1) loads are
// in flight per lane -- writes the scaled gradient vectors to each row and
// accumulates the dot products in fp32 (elements in order, then the vectors
// in order, the same order as one vector per step); the lanes' partial dots
// are summed by an xor-shuffle tree.  Rows no pair owns (row_src -1) are
// zero-filled by a second phase, 32 rows per warp.  One CTA per SM (up to
// 255 registers): measured on B200 at the metric shape, 349 us with one
// vector per step at 2 CTAs per SM, 341 us with two at 2 CTAs (a spill),
// 323 us with two at 1 CTA.
template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    combine_backward_kernel(const uint4 *__restrict__ grad_y, const uint4 *__restrict__ x,
                            const float *__restrict__ gates,
                            const int32_t *__restrict__ pair_slot,
                            const int32_t *__restrict__ row_src, uint4 *__restrict__ grad_x,
                            float *__restrict__ grad_gates, int32_t N, int32_t k, int64_t rows,
                            int32_t vecs) {
  MOE_TRACE_CTA(MOE_TRACE_COMBINE_BACKWARD, KMAX);
  allow_dependents();
  grid_dependency_wait();
  const int lane = threadIdx.x % kWarp;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) / kWarp;

  for (int64_t t = gw; t < N; t += nw) {
    int32_t my_slot = -1;
    float my_w = 0.0f;
    if (lane < k) {
      const int32_t s = __ldg(pair_slot + t * k + lane);
      if (s >= 0 && s < rows) {
        my_slot = s;
        my_w = __ldg(gates + t * k + lane);
      }
    }
    int64_t row[KMAX];
    float w[KMAX], dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int32_t s = __shfl_sync(kFull, my_slot, j);
      row[j] = s >= 0 && MOE_IN_RANGE(s, rows, kDbgCombineRow) ? s : -1;
      w[j] = __shfl_sync(kFull, my_w, j);
      dot[j] = 0.0f;
    }
    const uint4 *gy = grad_y + t * vecs;
    for (int v0 = lane; v0 < vecs; v0 += 2 * kWarp) {
      uint4 g4u[2], inu[2][KMAX];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int v = v0 + u * kWarp;
        g4u[u] = v < vecs ? ld_stream_v4(gy + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          inu[u][j] = (row[j] >= 0 && v < vecs) ? ld_stream_v4(x + row[j] * vecs + v)
                                                : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int v = v0 + u * kWarp;
        if (v >= vecs) break;
        const uint4 g4 = g4u[u];
        const uint4 *in = inu[u];
        const uint32_t ge[4] = {g4.x, g4.y, g4.z, g4.w};
        float g[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          g[2 * i] = bf16lo(ge[i]);
          g[2 * i + 1] = bf16hi(ge[i]);
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (row[j] < 0) continue;
          const uint32_t xe[4] = {in[j].x, in[j].y, in[j].z, in[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dot[j] = fmaf(g[2 * i], bf16lo(xe[i]), dot[j]);
            dot[j] = fmaf(g[2 * i + 1], bf16hi(xe[i]), dot[j]);
          }
          st_v4(grad_x + row[j] * vecs + v,
                make_uint4(pack_bf16x2(w[j] * g[0], w[j] * g[1]),
                           pack_bf16x2(w[j] * g[2], w[j] * g[3]),
                           pack_bf16x2(w[j] * g[4], w[j] * g[5]),
                           pack_bf16x2(w[j] * g[6], w[j] * g[7])));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      float d = dot[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(kFull, d, o);
      if (lane == j && j < k) grad_gates[t * k + j] = row[j] >= 0 ? d : 0.0f;
    }
  }

  // rows no pair owns carry no gradient
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t c = gw; c * kWarp < rows; c += nw) {
    const int64_t r = c * kWarp + lane;
    uint32_t m = __ballot_sync(kFull, r < rows && __ldg(row_src + r) < 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      uint4 *dst = grad_x + (c * kWarp + j) * vecs;
      for (int v = lane; v < vecs; v += kWarp) st_v4(dst + v, zero);
    }
  }
}

// Grid of a persistent kernel: resident CTAs per SM x SMs, or fewer when
// there is less work.
template <typename Kernel>
int grid_for(Kernel kernel, int64_t N, OccupancyCache &cache, size_t smem = 0) {
  const int per_sm = resident_ctas(cache, reinterpret_cast<const void *>(kernel), kThreads, smem);
  const int64_t need = std::max<int64_t>(1, (N + kThreads / kWarp - 1) / (kThreads / kWarp));
  return (int)std::min<int64_t>(need, (int64_t)per_sm * device_sm_count());
}

template <int KMAX>
cudaError_t launch_backward(const Shape &s, const uint4 *gy, const uint4 *x, const float *gates,
                            const int32_t *pair_slot, const int32_t *row_src, uint4 *gx,
                            float *grad_gates, int64_t work, cudaStream_t stream) {
  static OccupancyCache cache;
  auto kernel = combine_backward_kernel<KMAX>;
  return launch_pdl(kernel, dim3(grid_for(kernel, work, cache)), dim3(kThreads), 0, stream, gy, x,
                    gates, pair_slot, row_src, gx, grad_gates, s.N, s.k, s.rows, s.H / 8);
}

template <int KMAX, int U>
cudaError_t launch_from_peers(const Shape &s, const uint4 *const *peer_x, const int64_t *get,
                              const uint32_t *meta, const float *gates,
                              const int32_t *pair_slot, uint4 *o, cudaStream_t stream) {
  static OccupancyCache cache;
  auto kernel = combine_from_peers_kernel<KMAX, U>;
  const size_t smem = (size_t)24 * s.S;
  if (smem > 48 * 1024) {
    const cudaError_t err =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  // column spans per token as in launch_forward
  const int32_t vecs = s.H / 8;
  const int32_t step = kWarp * U;
  const int32_t steps = (vecs + step - 1) / step;
  const int64_t resident = (int64_t)resident_ctas(cache, reinterpret_cast<const void *>(kernel),
                                                  kThreads, smem) *
                           device_sm_count() * (kThreads / kWarp);
  int32_t splits = 1;
  if ((int64_t)s.N * 2 < resident)
    splits = (int32_t)std::min<int64_t>(steps, (resident + s.N - 1) / s.N);
  const int32_t span = (steps + splits - 1) / splits * step;
  splits = (vecs + span - 1) / span;
  const int32_t static_seg = s.Ce > 0 ? (s.E / s.S) * s.Ce : 0;
  return launch_pdl(kernel, dim3(grid_for(kernel, (int64_t)s.N * splits, cache, smem)),
                    dim3(kThreads), smem, stream, peer_x, get, meta, gates, pair_slot, o, s.N,
                    s.k, s.rows, vecs, splits, span, s.S, s.H, static_seg);
}

template <int KMAX, int U>
cudaError_t launch_forward(const Shape &s, const uint4 *x, const float *gates,
                           const int32_t *pair_slot, uint4 *o, cudaStream_t stream) {
  static OccupancyCache cache;
  auto kernel = combine_kernel<KMAX, U>;
  // column spans per token: 1 when the tokens alone fill the resident warps
  // (half of them at least), else enough spans of whole U-steps to do so
  const int32_t vecs = s.H / 8;
  const int32_t step = kWarp * U;
  const int32_t steps = (vecs + step - 1) / step;
  const int64_t resident = (int64_t)resident_ctas(cache, reinterpret_cast<const void *>(kernel),
                                                  kThreads, 0) *
                           device_sm_count() * (kThreads / kWarp);
  int32_t splits = 1;
  if ((int64_t)s.N * 2 < resident)
    splits = (int32_t)std::min<int64_t>(steps, (resident + s.N - 1) / s.N);
  const int32_t span = (steps + splits - 1) / splits * step;
  splits = (vecs + span - 1) / span;
  return launch_pdl(kernel, dim3(grid_for(kernel, (int64_t)s.N * splits, cache)), dim3(kThreads),
                    0, stream, x, gates, pair_slot, o, s.N, s.k, s.rows, vecs, splits, span);
}

}  // namespace

uint32_t debug_violations_combine(bool reset) { return read_debug_violations(reset); }

#ifdef MOE_TRACE
cudaError_t trace_attach_combine(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                              cudaStream_t stream) {
  return trace_attach_tu(records, count, capacity, stream);
}
#endif

cudaError_t launch_combine_backward(const Shape &s, const void *grad_y, const void *expert_out,
                                    const float *gates, const int32_t *pair_slot,
                                    const int32_t *row_src, void *grad_expert_out,
                                    float *grad_gates, cudaStream_t stream) {
  const uint4 *gy = static_cast<const uint4 *>(grad_y);
  const uint4 *x = static_cast<const uint4 *>(expert_out);
  uint4 *gx = static_cast<uint4 *>(grad_expert_out);
  const int64_t work = std::max<int64_t>((int64_t)s.N, (s.rows + kWarp - 1) / kWarp);
  if (work == 0) return cudaSuccess;
  if (s.k <= 4)
    return launch_backward<4>(s, gy, x, gates, pair_slot, row_src, gx, grad_gates, work, stream);
  if (s.k <= 8)
    return launch_backward<8>(s, gy, x, gates, pair_slot, row_src, gx, grad_gates, work, stream);
  return launch_backward<16>(s, gy, x, gates, pair_slot, row_src, gx, grad_gates, work, stream);
}

cudaError_t launch_combine_from_peers(const Shape &s, const void *const *peer_expert_out,
                                      const int64_t *get_offsets, const uint32_t *meta,
                                      const float *gates, const int32_t *pair_slot, void *out,
                                      cudaStream_t stream) {
  if (s.N == 0) return cudaSuccess;
  const uint4 *const *px = reinterpret_cast<const uint4 *const *>(peer_expert_out);
  uint4 *o = static_cast<uint4 *>(out);
  if (s.k <= 2) return launch_from_peers<2, 4>(s, px, get_offsets, meta, gates, pair_slot, o, stream);
  if (s.k <= 4) return launch_from_peers<4, 2>(s, px, get_offsets, meta, gates, pair_slot, o, stream);
  if (s.k <= 8) return launch_from_peers<8, 2>(s, px, get_offsets, meta, gates, pair_slot, o, stream);
  return launch_from_peers<16, 1>(s, px, get_offsets, meta, gates, pair_slot, o, stream);
}

cudaError_t launch_combine(const Shape &s, const void *expert_out, const float *gates,
                           const int32_t *pair_slot, void *out, cudaStream_t stream) {
  if (s.N == 0) return cudaSuccess;
  const uint4 *x = static_cast<const uint4 *>(expert_out);
  uint4 *o = static_cast<uint4 *>(out);
  if (s.k <= 2) return launch_forward<2, 4>(s, x, gates, pair_slot, o, stream);
  if (s.k <= 4) return launch_forward<4, 2>(s, x, gates, pair_slot, o, stream);
  if (s.k <= 8) return launch_forward<8, 2>(s, x, gates, pair_slot, o, stream);
  return launch_forward<16, 1>(s, x, gates, pair_slot, o, stream);
}

}  // namespace moe
