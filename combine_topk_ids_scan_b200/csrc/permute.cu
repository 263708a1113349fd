// permute.cu -- dispatch permute: write each token's hidden row to the k rows
// its pairs were given by the layout, optionally quantising on the way, and
// zero every padding row.
//
// Movement is token-major ("push"): one warp per token reads the token's row
// from HBM once with 16-byte streaming loads and stores it (or its quantised
// form) to each of its k destination rows with 16-byte stores, so the
// quantisation is computed once per token, not once per copy.  A second phase
// of the same persistent grid scans row_src 32 rows per warp and zero-fills
// the rows whose source is -1.
//
// Formats: NKI "Permute A2AV Kernel API Reference" ([C, H] packed rows then
// deterministic zero padding); Mojo MAX ep_comm BF16TokenFormat,
// BlockwiseFP8TokenFormat (1x128 blocks, fp32 scale = amax/448),
// NVBlockScaledTokenFormat and Struct_ep_dispatch_async_block_scaled_nv (E2M1
// codes, one E4M3 scale per 16 elements, caller-supplied global scale).  The
// ep_comm page's EP_COPY_SRC_WIDTH (8 source elements per thread per copy
// item) is the same 16-byte bf16 vector used here.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kFull = 0xFFFFFFFFu;

// Lane j < k holds pair (t, j)'s row, or -1 when the pair has no row in
// [0, rows).  Returns the ballot of lanes holding a row.
__device__ __forceinline__ uint32_t load_token_slots(const int32_t *__restrict__ pair_slot,
                                                     int64_t t, int k, int64_t rows, int lane,
                                                     int32_t &my_slot) {
  my_slot = -1;
  if (lane < k) {
    const int32_t s = __ldg(pair_slot + t * k + lane);
    if (s >= 0 && s < rows) my_slot = s;
  }
  return __ballot_sync(kFull, my_slot >= 0);
}

// ------------------------------------------------------------------- bf16
template <int U>
__global__ void __launch_bounds__(kThreads)
    permute_bf16_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                        const int32_t *__restrict__ pair_slot, uint4 *__restrict__ out,
                        int32_t N, int32_t k, int64_t rows, int32_t vecs) {
  const int lane = threadIdx.x % kWarp;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) / kWarp;

  for (int64_t t = gw; t < N; t += nw) {
    int32_t my_slot;
    const uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
    if (live == 0) continue;
    const uint4 *src = hidden + t * vecs;
    for (int v0 = 0; v0 < vecs; v0 += kWarp * U) {
      uint4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * kWarp + lane;
        if (v < vecs) x[u] = ld_stream_v4(src + v);
      }
      uint32_t m = live;
      while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        uint4 *dst = out + (int64_t)__shfl_sync(kFull, my_slot, j) * vecs;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * kWarp + lane;
          if (v < vecs) st_v4(dst + v, x[u]);
        }
      }
    }
  }

  // padding rows
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t c = gw; c * kWarp < rows; c += nw) {
    const int64_t r = c * kWarp + lane;
    uint32_t m = __ballot_sync(kFull, r < rows && __ldg(row_src + r) < 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      uint4 *dst = out + (c * kWarp + j) * vecs;
      for (int v = lane; v < vecs; v += kWarp) st_v4(dst + v, zero);
    }
  }
}

// ------------------------------------------------------------------- FP8
// Lane handles 16 consecutive elements per step (two 16-byte loads, one
// 16-byte store of codes); 8 lanes form one 1x128 block; a warp step covers
// 512 elements.
template <int U>
__global__ void __launch_bounds__(kThreads)
    permute_fp8_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                       const int32_t *__restrict__ pair_slot, uint8_t *__restrict__ q,
                       float *__restrict__ scales, int32_t N, int32_t k, int64_t rows,
                       int32_t H) {
  const int lane = threadIdx.x % kWarp;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) / kWarp;
  const int32_t vecs = H / 8;
  const int32_t nb = H / 128;

  for (int64_t t = gw; t < N; t += nw) {
    int32_t my_slot;
    const uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
    if (live == 0) continue;
    const uint4 *src = hidden + t * vecs;
    for (int c0 = 0; c0 < H; c0 += 512 * U) {
      uint4 a[U], b[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int col = c0 + u * 512 + lane * 16;
        if (col < H) {
          a[u] = ld_stream_v4(src + col / 8);
          b[u] = ld_stream_v4(src + col / 8 + 1);
        } else {
          a[u] = b[u] = make_uint4(0, 0, 0, 0);
        }
      }
      uint4 codes[U];
      float scale[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[8] = {a[u].x, a[u].y, a[u].z, a[u].w, b[u].x, b[u].y, b[u].z, b[u].w};
        float f[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f[2 * i] = bf16lo(w[i]);
          f[2 * i + 1] = bf16hi(w[i]);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
        uint32_t c[4] = {0, 0, 0, 0};
        float sc = 0.0f;
        if (amax > 0.0f) {
          sc = amax / 448.0f;  // IEEE round-to-nearest division
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = cvt_e4m3x2(f[4 * i] / sc, f[4 * i + 1] / sc);
            const uint32_t hi = cvt_e4m3x2(f[4 * i + 2] / sc, f[4 * i + 3] / sc);
            c[i] = lo | (hi << 16);
          }
        }
        codes[u] = make_uint4(c[0], c[1], c[2], c[3]);
        scale[u] = sc;
      }
      uint32_t m = live;
      while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const int64_t s = __shfl_sync(kFull, my_slot, j);
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int col = c0 + u * 512 + lane * 16;
          if (col < H) {
            st_v4(reinterpret_cast<uint4 *>(q + s * H + col), codes[u]);
            if ((lane & 7) == 0) scales[s * nb + col / 128] = scale[u];
          }
        }
      }
    }
  }

  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t c = gw; c * kWarp < rows; c += nw) {
    const int64_t r = c * kWarp + lane;
    uint32_t m = __ballot_sync(kFull, r < rows && __ldg(row_src + r) < 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      const int64_t row = c * kWarp + j;
      uint4 *dst = reinterpret_cast<uint4 *>(q + row * H);
      for (int v = lane; v < H / 16; v += kWarp) st_v4(dst + v, zero);
      for (int b = lane; b < nb; b += kWarp) scales[row * nb + b] = 0.0f;
    }
  }
}

// ------------------------------------------------------------------- NVFP4
// Lane handles 32 consecutive elements per step (two 16-element blocks, four
// 16-byte loads, one 16-byte store of codes, one 2-byte store of scales); a
// warp step covers 1024 elements.
__device__ __forceinline__ uint32_t nvfp4_block(const float *f, float gs, uint32_t &codes_lo,
                                                uint32_t &codes_hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
  const float sf = (amax / 6.0f) / gs;
  const uint32_t sq = cvt_e4m3x2(sf, 0.0f) & 0xFFu;
  const float d = e4m3_to_float(sq) * gs;
  uint32_t c[2] = {0, 0};
  if (d > 0.0f) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t word = 0;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = 8 * h + 2 * m;
        word |= cvt_e2m1x2(f[i] / d, f[i + 1] / d) << (8 * m);
      }
      c[h] = word;
    }
  }
  codes_lo = c[0];
  codes_hi = c[1];
  return sq;
}

__global__ void __launch_bounds__(kThreads)
    permute_nvfp4_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                         const int32_t *__restrict__ pair_slot,
                         const float *__restrict__ global_scale, uint8_t *__restrict__ q,
                         uint8_t *__restrict__ scales, int32_t N, int32_t k, int64_t rows,
                         int32_t H) {
  const int lane = threadIdx.x % kWarp;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) / kWarp;
  const int32_t vecs = H / 8;
  const int32_t qrow = H / 2, srow = H / 16;
  const float gs = __ldg(global_scale);

  for (int64_t t = gw; t < N; t += nw) {
    int32_t my_slot;
    const uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
    if (live == 0) continue;
    const uint4 *src = hidden + t * vecs;
    for (int c0 = 0; c0 < H; c0 += 1024) {
      const int col = c0 + lane * 32;
      const bool active = col < H;
      uint4 x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        x[i] = active ? ld_stream_v4(src + col / 8 + i) : make_uint4(0, 0, 0, 0);
      float f[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f[8 * i + 2 * e] = bf16lo(w[e]);
          f[8 * i + 2 * e + 1] = bf16hi(w[e]);
        }
      }
      uint4 codes;
      const uint32_t sq0 = nvfp4_block(f, gs, codes.x, codes.y);
      const uint32_t sq1 = nvfp4_block(f + 16, gs, codes.z, codes.w);
      const uint16_t sq = (uint16_t)(sq0 | (sq1 << 8));
      uint32_t m = live;
      while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const int64_t s = __shfl_sync(kFull, my_slot, j);
        if (active) {
          st_v4(reinterpret_cast<uint4 *>(q + s * qrow + col / 2), codes);
          *reinterpret_cast<uint16_t *>(scales + s * srow + col / 16) = sq;
        }
      }
    }
  }

  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t c = gw; c * kWarp < rows; c += nw) {
    const int64_t r = c * kWarp + lane;
    uint32_t m = __ballot_sync(kFull, r < rows && __ldg(row_src + r) < 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      const int64_t row = c * kWarp + j;
      uint4 *dst = reinterpret_cast<uint4 *>(q + row * qrow);
      for (int v = lane; v < qrow / 16; v += kWarp) st_v4(dst + v, zero);
      uint16_t *sdst = reinterpret_cast<uint16_t *>(scales + row * srow);
      for (int v = lane; v < srow / 2; v += kWarp) sdst[v] = 0;
    }
  }
}

template <typename Kernel>
int persistent_blocks(Kernel kernel) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  return per_sm * device_sm_count();
}

template <typename Kernel>
int grid_for(Kernel kernel, const Shape &s) {
  // enough warps for every token and every 32-row padding chunk, capped at
  // one full wave of resident blocks
  const int64_t warps = std::max<int64_t>((int64_t)s.N, (s.rows + kWarp - 1) / kWarp);
  const int64_t need = std::max<int64_t>(1, (warps + kThreads / kWarp - 1) / (kThreads / kWarp));
  return (int)std::min<int64_t>(need, persistent_blocks(kernel));
}

}  // namespace

cudaError_t launch_permute_bf16(const Shape &s, const void *hidden, const int32_t *row_src,
                                const int32_t *pair_slot, void *out, cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  auto kernel = permute_bf16_kernel<4>;
  kernel<<<grid_for(kernel, s), kThreads, 0, stream>>>(
      static_cast<const uint4 *>(hidden), row_src, pair_slot, static_cast<uint4 *>(out), s.N,
      s.k, s.rows, s.H / 8);
  return cudaGetLastError();
}

cudaError_t launch_permute_fp8(const Shape &s, const void *hidden, const int32_t *row_src,
                               const int32_t *pair_slot, uint8_t *q, float *scales,
                               cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  auto kernel = permute_fp8_kernel<2>;
  kernel<<<grid_for(kernel, s), kThreads, 0, stream>>>(static_cast<const uint4 *>(hidden),
                                                        row_src, pair_slot, q, scales, s.N,
                                                        s.k, s.rows, s.H);
  return cudaGetLastError();
}

cudaError_t launch_permute_nvfp4(const Shape &s, const void *hidden, const int32_t *row_src,
                                 const int32_t *pair_slot, const float *global_scale,
                                 uint8_t *q, uint8_t *scales, cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  auto kernel = permute_nvfp4_kernel;
  kernel<<<grid_for(kernel, s), kThreads, 0, stream>>>(static_cast<const uint4 *>(hidden),
                                                        row_src, pair_slot, global_scale, q,
                                                        scales, s.N, s.k, s.rows, s.H);
  return cudaGetLastError();
}

}  // namespace moe
