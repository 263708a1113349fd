// permute.cu -- dispatch permute: write each token's hidden row to the k rows
// its pairs were given by the layout, optionally quantising on the way, and
// zero every padding row.
//
// Movement is token-major ("push"): each token's row is read from HBM once
// with 16-byte streaming loads and stored (or its quantised form) to each of
// its k destination rows with 16-byte stores, so the quantisation is computed
// once per token, not once per copy.  A warp issues its row loads before the
// load of the token's pair_slot entries, so the two latencies overlap.  The unit of work is one chunk of one
// token (512 elements for bf16, 1024 for the quantisers): one warp takes one
// unit and exits.  Short warps over a grid of many blocks keep the write
// stream denser than long-lived persistent warps do (measured on B200 for the
// bf16 permute at N=8192, H=7168, k=8: 195 us persistent, 170 us with
// 1024-element units, 166 us with 512).
//
// Padding rows (row_src -1) are zero-filled by padding warps placed first in
// the grid: warp g checks the 32 rows [32g, 32g+32) and zero-fills those
// without a source.  Scheduled first, they cost little when there is no
// padding, and a long run of padding rows is written while the token units
// run instead of as a tail (measured on B200, bf16 with 32K padding rows of
// 98K: 240 us vs 336 us with the padding warps last).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "trace.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr int kChunk = 1024;     // elements of one token per unit (quantisers)
constexpr int kBf16Chunk = 512;  // elements of one token per unit (bf16)

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

// Ballot of the rows of [32g, 32g+32) without a source: row_src -1, or at or
// past `rows` but below `check_rows`.
__device__ __forceinline__ uint32_t padding_mask(int64_t g, int lane,
                                                 const int32_t *__restrict__ row_src,
                                                 int64_t rows, int64_t check_rows) {
  const int64_t r = g * kWarp + lane;
  return __ballot_sync(kFull, r < check_rows && (r >= rows || __ldg(row_src + r) < 0));
}

// Share c of `parts` near-equal shares of [0, n): [b, e).
__device__ __forceinline__ void share_of(int c, int parts, int32_t n, int32_t &b, int32_t &e) {
  const int32_t per = (n + parts - 1) / parts;
  b = min(n, c * per);
  e = min(n, b + per);
}

// Zero 16-byte vectors [v0, v1) of each row in `m` (rows 32g + bit) and,
// when scales is not null, 2-byte words [s0, s1) of its scale row.
__device__ __forceinline__ void zero_rows(uint32_t m, int64_t g, int lane, uint4 *out,
                                          int32_t row_vecs, int32_t v0, int32_t v1,
                                          uint16_t *scales, int32_t scale_words, int32_t s0,
                                          int32_t s1) {
  const uint4 zero = make_uint4(0, 0, 0, 0);
  while (m) {
    const int j = __ffs(m) - 1;
    m &= m - 1;
    const int64_t row = g * kWarp + j;
    uint4 *dst = out + row * row_vecs;
    for (int v = v0 + lane; v < v1; v += kWarp) st_v4(dst + v, zero);
    if (scales) {
      uint16_t *sd = scales + row * scale_words;
      for (int v = s0 + lane; v < s1; v += kWarp) sd[v] = 0;
    }
  }
}

// ------------------------------------------------------------------- bf16
// Unit = (token, 512 elements): each lane loads 2 vectors of 8 bf16.
__global__ void __launch_bounds__(kThreads)
    permute_bf16_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                        const int32_t *__restrict__ pair_slot, uint4 *__restrict__ out,
                        int32_t N, int32_t k, int64_t rows, int32_t vecs, int32_t chunks,
                        int32_t psplit) {
  MOE_TRACE_CTA(MOE_TRACE_PERMUTE_BF16, 0);
  allow_dependents();
  grid_dependency_wait();
  constexpr int U = kBf16Chunk / 8 / kWarp;  // 2
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  const int64_t pad_units = (rows + kWarp - 1) / kWarp * psplit;
  if (w0 < pad_units) {
    const int64_t g = w0 / psplit;
    if (const uint32_t m = padding_mask(g, lane, row_src, rows, rows)) {
      int32_t v0, v1;
      share_of((int)(w0 % psplit), psplit, vecs, v0, v1);
      zero_rows(m, g, lane, out, vecs, v0, v1, nullptr, 0, 0, 0);
    }
    return;
  }
  const int64_t w = w0 - pad_units;
  if (w < units) {
    const int64_t t = w / chunks;
    const int v0 = (int)(w % chunks) * (kBf16Chunk / 8);
    const uint4 *src = hidden + t * vecs;
    uint4 x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp + lane;
      if (v < vecs) x[u] = ld_stream_v4(src + v);
    }
    int32_t my_slot;
    uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
    while (live) {
      const int j = __ffs(live) - 1;
      live &= live - 1;
      const int64_t s = __shfl_sync(kFull, my_slot, j);
      if (!MOE_IN_RANGE(s, rows, kDbgPermuteRow)) continue;
      uint4 *dst = out + s * vecs;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * kWarp + lane;
        if (v < vecs) st_v4(dst + v, x[u]);
      }
    }
  }

}

// ------------------------------------------------------- dispatch to peers
// Expert-parallel dispatch with the send step fused into the permute: the
// rows of segment s (experts [sL, (s+1)L): local rows [start_s, start_s +
// rows_s)) are stored straight into rank s's receive buffer peer_out[s] at
// rows put[s] + (r - start_s), instead of into a local send buffer that an
// all-to-all then ships.  peer_out[s] is any device pointer this GPU can
// store to (a peer mapping over NVLink / NVSwitch, or this rank's own buffer
// for its own segment).  The bf16 permute's units; a lane holding pair j
// finds its row's segment by binary search over the segment starts (staged
// in shared memory) and the warp broadcasts the destination row.  Padding
// rows inside a segment are zeroed at the destination; rows past the last
// segment are not sent.
__device__ __forceinline__ int segment_of(int64_t r, const int32_t *s_start,
                                          const int32_t *s_rows, int32_t S) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {  // last s with start[s] <= r
    const int mid = (lo + hi + 1) / 2;
    if (s_start[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  return (r >= s_start[lo] && r - s_start[lo] < s_rows[lo]) ? lo : -1;
}

// Segment starts and rows into shared memory: packed mode from meta rows 0-1
// (elements), capacity mode the static blocks of L * Ce rows.  Called by
// every thread; the caller synchronises the block afterwards.
__device__ __forceinline__ void stage_segments(const uint32_t *__restrict__ meta, int32_t S,
                                               int32_t H, int32_t static_seg_rows,
                                               int32_t *s_start, int32_t *s_rows) {
  for (int i = threadIdx.x; i < S; i += kThreads) {
    if (static_seg_rows > 0) {
      s_start[i] = i * static_seg_rows;
      s_rows[i] = static_seg_rows;
    } else {
      s_start[i] = (int32_t)(__ldg(meta + S + i) / (uint32_t)H);
      s_rows[i] = (int32_t)(__ldg(meta + i) / (uint32_t)H);
    }
  }
}

// Per-rank table of the quantised peer kernels in shared memory: code and
// scale buffer addresses and put offsets (8 bytes each), then the segment
// starts and rows; 32 * S bytes.
struct PeerTable {
  uint8_t **codes;
  uint8_t **scales;
  int64_t *put;
  int32_t *start;
  int32_t *rows;
};
__device__ __forceinline__ PeerTable stage_peer_table(uint64_t *smem, const uint32_t *meta,
                                                      int32_t S, int32_t H,
                                                      int32_t static_seg_rows,
                                                      uint8_t *const *peer_codes,
                                                      uint8_t *const *peer_scales,
                                                      const int64_t *__restrict__ put) {
  PeerTable t;
  t.codes = reinterpret_cast<uint8_t **>(smem);
  t.scales = reinterpret_cast<uint8_t **>(smem + S);
  t.put = reinterpret_cast<int64_t *>(smem + 2 * S);
  t.start = reinterpret_cast<int32_t *>(smem + 3 * S);
  t.rows = t.start + S;
  stage_segments(meta, S, H, static_seg_rows, t.start, t.rows);
  for (int i = threadIdx.x; i < S; i += kThreads) {
    t.codes[i] = peer_codes[i];
    t.scales[i] = peer_scales[i];
    t.put[i] = __ldg(put + i);
  }
  return t;
}

// Code and scale row addresses of local row r in its rank's receive buffers
// (false when r belongs to no segment).
__device__ __forceinline__ bool peer_rows(int64_t r, const PeerTable &t, int32_t S,
                                          int64_t code_bytes, int64_t scale_bytes,
                                          uint8_t *&q, uint8_t *&sc) {
  const int sg = segment_of(r, t.start, t.rows, S);
  if (sg < 0) return false;
  const int64_t pr = t.put[sg] + (r - t.start[sg]);
  q = t.codes[sg] + pr * code_bytes;
  sc = t.scales[sg] + pr * scale_bytes;
  return true;
}

// Destination of local row r (nullptr when r belongs to no segment).
__device__ __forceinline__ uint4 *peer_row(int64_t r, const int32_t *s_start,
                                           const int32_t *s_rows, int32_t S,
                                           uint4 *const *__restrict__ peer_out,
                                           const int64_t *__restrict__ put, int32_t vecs) {
  const int sg = segment_of(r, s_start, s_rows, S);
  if (sg < 0) return nullptr;
  return peer_out[sg] + (put[sg] + (r - s_start[sg])) * (int64_t)vecs;
}

__global__ void __launch_bounds__(kThreads)
    permute_to_peers_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                            const int32_t *__restrict__ pair_slot,
                            const uint32_t *__restrict__ meta, uint4 *const *__restrict__ peer_out,
                            const int64_t *__restrict__ put, int32_t N, int32_t k, int64_t rows,
                            int32_t vecs, int32_t chunks, int32_t psplit, int32_t S, int32_t H,
                            int32_t static_seg_rows) {
  MOE_TRACE_CTA(MOE_TRACE_PERMUTE_TO_PEERS, 0);
  allow_dependents();
  extern __shared__ int32_t seg_smem[];  // [S] starts, [S] rows
  int32_t *s_start = seg_smem, *s_rows = seg_smem + S;
  grid_dependency_wait();
  stage_segments(meta, S, H, static_seg_rows, s_start, s_rows);
  __syncthreads();
  constexpr int U = kBf16Chunk / 8 / kWarp;  // 2
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  const int64_t pad_units = (rows + kWarp - 1) / kWarp * psplit;
  if (w0 < pad_units) {
    const int64_t g = w0 / psplit;
    uint32_t m = padding_mask(g, lane, row_src, rows, rows);
    int32_t v0, v1;
    share_of((int)(w0 % psplit), psplit, vecs, v0, v1);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      uint4 *dst = peer_row(g * kWarp + j, s_start, s_rows, S, peer_out, put, vecs);
      if (dst)
        for (int v = v0 + lane; v < v1; v += kWarp) st_v4(dst + v, zero);
    }
    return;
  }
  const int64_t w = w0 - pad_units;
  if (w >= units) return;
  const int64_t t = w / chunks;
  const int v0 = (int)(w % chunks) * (kBf16Chunk / 8);
  const uint4 *src = hidden + t * vecs;
  uint4 x[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int v = v0 + u * kWarp + lane;
    if (v < vecs) x[u] = ld_stream_v4(src + v);
  }
  int32_t my_slot;
  const uint32_t live_rows = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
  uint4 *my_dst = my_slot >= 0 ? peer_row(my_slot, s_start, s_rows, S, peer_out, put, vecs)
                               : nullptr;
  uint32_t live = live_rows & __ballot_sync(kFull, my_dst != nullptr);
  while (live) {
    const int j = __ffs(live) - 1;
    live &= live - 1;
    uint4 *dst = reinterpret_cast<uint4 *>(
        __shfl_sync(kFull, reinterpret_cast<unsigned long long>(my_dst), j));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp + lane;
      if (v < vecs) st_v4(dst + v, x[u]);
    }
  }
}

// --------------------------------------------------- pre-multiplied gates
// DeepSpeed's pre-multiplication of the token representations by their
// router scores before expert compute: the bf16 permute's units, but pair
// (t, j)'s row is bf16(w[t,j] * x[t]) -- one fp32 product and one rounding
// (nearest even) per element.
__device__ __forceinline__ uint4 scale_bf16x8(const uint4 &v, float g) {
  return make_uint4(pack_bf16x2(g * bf16lo(v.x), g * bf16hi(v.x)),
                    pack_bf16x2(g * bf16lo(v.y), g * bf16hi(v.y)),
                    pack_bf16x2(g * bf16lo(v.z), g * bf16hi(v.z)),
                    pack_bf16x2(g * bf16lo(v.w), g * bf16hi(v.w)));
}

__global__ void __launch_bounds__(kThreads)
    permute_premultiplied_kernel(const uint4 *__restrict__ hidden,
                                 const int32_t *__restrict__ row_src,
                                 const int32_t *__restrict__ pair_slot,
                                 const float *__restrict__ gates, uint4 *__restrict__ out,
                                 int32_t N, int32_t k, int64_t rows, int32_t vecs,
                                 int32_t chunks, int32_t psplit) {
  MOE_TRACE_CTA(MOE_TRACE_PERMUTE_PREMULTIPLIED, 0);
  allow_dependents();
  grid_dependency_wait();
  constexpr int U = kBf16Chunk / 8 / kWarp;  // 2
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  const int64_t pad_units = (rows + kWarp - 1) / kWarp * psplit;
  if (w0 < pad_units) {
    const int64_t g = w0 / psplit;
    if (const uint32_t m = padding_mask(g, lane, row_src, rows, rows)) {
      int32_t v0, v1;
      share_of((int)(w0 % psplit), psplit, vecs, v0, v1);
      zero_rows(m, g, lane, out, vecs, v0, v1, nullptr, 0, 0, 0);
    }
    return;
  }
  const int64_t w = w0 - pad_units;
  if (w >= units) return;
  const int64_t t = w / chunks;
  const int v0 = (int)(w % chunks) * (kBf16Chunk / 8);
  const uint4 *src = hidden + t * vecs;
  uint4 x[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int v = v0 + u * kWarp + lane;
    if (v < vecs) x[u] = ld_stream_v4(src + v);
  }
  int32_t my_slot;
  uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
  const float my_w = lane < k ? __ldg(gates + t * k + lane) : 0.0f;
  while (live) {
    const int j = __ffs(live) - 1;
    live &= live - 1;
    const float g = __shfl_sync(kFull, my_w, j);
    const int64_t s = __shfl_sync(kFull, my_slot, j);
    if (!MOE_IN_RANGE(s, rows, kDbgPermuteRow)) continue;
    uint4 *dst = out + s * vecs;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp + lane;
      if (v < vecs) st_v4(dst + v, scale_bf16x8(x[u], g));
    }
  }
}

// ------------------------------------------------------------------- FP8
// One lane's 16 consecutive elements (a: the first 8, b: the next 8) of a
// 1x128 block that 8 consecutive lanes share -> 16 E4M3 codes; returns the
// block's scale amax / 448 (0 and zero codes for an all-zero block).  The
// block amax is three xor-shuffles, so all 32 lanes call it together.
__device__ __forceinline__ float fp8_quant16(const uint4 &a, const uint4 &b, uint4 &codes) {
  const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float f[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = bf16lo(wd[i]);
    f[2 * i + 1] = bf16hi(wd[i]);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = max_abs3(amax, f[2 * i], f[2 * i + 1]);
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
  uint32_t cw[4] = {0, 0, 0, 0};
  float sc = 0.0f;
  if (amax > 0.0f) {
    sc = amax / 448.0f;  // IEEE round-to-nearest division
    float2 qt[8];        // x / sc, |x / sc| <= 448
    if (sc >= kQuotientMinDivisor && sc <= kQuotientMaxDivisor) {
      const float rs = __frcp_rn(sc);
#pragma unroll
      for (int i = 0; i < 8; ++i) qt[i] = rn_quotient2(make_float2(f[2 * i], f[2 * i + 1]), sc, rs);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) qt[i] = make_float2(f[2 * i] / sc, f[2 * i + 1] / sc);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) cw[i] = cvt_e4m3x4(qt[2 * i], qt[2 * i + 1]);
  }
  codes = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  return sc;
}

// Unit = (token, 1024 elements).  A lane takes 16 consecutive elements per
// half (two 16-byte loads -> one 16-byte store of codes); 8 lanes form one
// 1x128 block; a half-unit covers 512 elements.
__global__ void __launch_bounds__(kThreads)
    permute_fp8_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                       const int32_t *__restrict__ pair_slot, uint8_t *__restrict__ q,
                       float *__restrict__ scales, int32_t N, int32_t k, int64_t rows,
                       int32_t H, int32_t chunks, int32_t psplit) {
  MOE_TRACE_CTA(MOE_TRACE_PERMUTE_FP8, 0);
  allow_dependents();
  grid_dependency_wait();
  constexpr int U = kChunk / 512;  // 2
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  const int64_t pad_units = (rows + kWarp - 1) / kWarp * psplit;
  const int32_t vecs = H / 8;
  const int32_t nb = H / 128;
  if (w0 < pad_units) {
    const int64_t g = w0 / psplit;
    if (const uint32_t m = padding_mask(g, lane, row_src, rows, rows)) {
      const int c = (int)(w0 % psplit);
      int32_t v0, v1, s0, s1;
      share_of(c, psplit, H / 16, v0, v1);
      share_of(c, psplit, 2 * nb, s0, s1);
      zero_rows(m, g, lane, reinterpret_cast<uint4 *>(q), H / 16, v0, v1,
                reinterpret_cast<uint16_t *>(scales), 2 * nb, s0, s1);
    }
    return;
  }
  const int64_t w = w0 - pad_units;

  if (w < units) {
    const int64_t t = w / chunks;
    const int c0 = (int)(w % chunks) * kChunk;
    int32_t my_slot;
    uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
    const uint4 *src = hidden + t * vecs;
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
    for (int u = 0; u < U; ++u) scale[u] = fp8_quant16(a[u], b[u], codes[u]);
    while (live) {
      const int j = __ffs(live) - 1;
      live &= live - 1;
      const int64_t s = __shfl_sync(kFull, my_slot, j);
      if (!MOE_IN_RANGE(s, rows, kDbgPermuteRow)) continue;
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

  // codes: H bytes per row, 64 vectors per chunk; scales: nb floats per row
  // = 2*nb 2-byte words, 16 words (8 scales) per chunk
}

// ------------------------------------------------------------------- NVFP4
// Unit = (token, 1024 elements).  A lane takes 32 consecutive elements (two
// 16-element blocks, four 16-byte loads) and stores 16 bytes of codes and
// 2 bytes of scales.
__device__ __forceinline__ uint32_t nvfp4_block(const float *f, float gs, uint32_t &codes_lo,
                                                uint32_t &codes_hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = max_abs3(amax, f[2 * i], f[2 * i + 1]);
  const float sf = (amax / 6.0f) / gs;
  const uint32_t sq = cvt_e4m3x2(sf, 0.0f) & 0xFFu;
  const float d = e4m3_to_float(sq) * gs;
  uint32_t c[2] = {0, 0};
  if (d > 0.0f) {
    float2 qt[8];  // x / d
    // |x / d| <= 12.01 unless the block scale saturated at 448 (0x7E): an
    // unsaturated E4M3 scale is at least half of amax / 6
    if (sq < 0x7Eu && d >= kQuotientMinDivisor && d <= kQuotientMaxDivisor) {
      const float rd = __frcp_rn(d);
#pragma unroll
      for (int i = 0; i < 8; ++i) qt[i] = rn_quotient2(make_float2(f[2 * i], f[2 * i + 1]), d, rd);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) qt[i] = make_float2(f[2 * i] / d, f[2 * i + 1] / d);
    }
    c[0] = cvt_e2m1x8(qt[0], qt[1], qt[2], qt[3]);
    c[1] = cvt_e2m1x8(qt[4], qt[5], qt[6], qt[7]);
  }
  codes_lo = c[0];
  codes_hi = c[1];
  return sq;
}

// MX token format (OCP MXFP4): one block of 32 -> 16 bytes of E2M1 codes and
// the E8M0 scale code; an all-zero block is scale 0, codes 0.
__device__ __forceinline__ uint32_t mxfp4_block(const float *f, uint4 &codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = max_abs3(amax, f[2 * i], f[2 * i + 1]);
  uint32_t c[4] = {0, 0, 0, 0};
  uint32_t sc = 0;
  if (amax > 0.0f) {
    sc = mx_scale_code(amax, 2);
    const float m = pow2i(127 - (int)sc);  // 2^-X, a normal float
    float2 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul2_rn(make_float2(f[2 * i], f[2 * i + 1]), make_float2(m, m));
#pragma unroll
    for (int h = 0; h < 4; ++h) c[h] = cvt_e2m1x8(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
  }
  codes = make_uint4(c[0], c[1], c[2], c[3]);
  return sc;
}

// Block-scale atom layout (Mojo MAX ep_comm SF_ATOM_M = (32, 4),
// SF_ROW_STRIDE_LOCAL = 16, SF_ATOM_ELEMS_LOCAL = 512): byte of scale (m, c)
// when a 128-row tile spans `col_tiles` atoms.
__device__ __forceinline__ int64_t sf_atom_offset(int64_t m, int32_t c, int32_t col_tiles) {
  return ((m >> 7) * col_tiles + (c >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (c & 3);
}

// MX == false: NVFP4 (two 16-element blocks per lane, E4M3 scales);
// MX == true: MXFP4 (one 32-element block per lane, E8M0 scales).
// SWIZZLED: scales in the block-scale atom layout.  The token row's loads
// are issued first, before the pair_slot load and its ballot.  The MXFP4
// linear-scale kernel is held to 5 resident CTAs per SM (at most 48
// registers; measured on B200 at the metric shape: 61.4 -> 60.0 us), the
// NVFP4 and the atom-layout kernels to 4 (NVFP4 with its loads first: 65.5 us
// at 5 CTAs with a 4-byte spill, 63.5 us at 4 without one).
template <bool MX, bool SWIZZLED>
__global__ void __launch_bounds__(kThreads, (SWIZZLED || !MX) ? 4 : 5)
    permute_fp4_kernel(const uint4 *__restrict__ hidden, const int32_t *__restrict__ row_src,
                       const int32_t *__restrict__ pair_slot,
                       const float *__restrict__ global_scale, uint8_t *__restrict__ q,
                       uint8_t *__restrict__ scales, int32_t N, int32_t k, int64_t rows,
                       int32_t H, int32_t chunks, int32_t psplit) {
  MOE_TRACE_CTA(MX ? MOE_TRACE_PERMUTE_MXFP4 : MOE_TRACE_PERMUTE_NVFP4, SWIZZLED ? 1 : 0);
  constexpr bool swizzled = SWIZZLED;
  allow_dependents();
  grid_dependency_wait();
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  // swizzled scales: the rows that only complete the last 128-row tile are
  // padding for the scales too
  const int64_t check_rows = swizzled ? (rows + 127) / 128 * 128 : rows;
  const int64_t pad_units = (check_rows + kWarp - 1) / kWarp * psplit;
  const int32_t vecs = H / 8;
  const int32_t qrow = H / 2, srow = MX ? H / 32 : H / 16;
  const int32_t groups = (srow + 3) / 4;  // 4-scale groups per row (atom layout)
  if (w0 < pad_units) {
    // codes: H/2 bytes per row; scales: linear srow bytes per row, or the
    // row's `groups` 4-byte groups in the atom layout; this warp zeroes its
    // share c of each of them
    const int64_t g = w0 / psplit;
    const int c = (int)(w0 % psplit);
    const uint32_t m = padding_mask(g, lane, row_src, rows, check_rows);
    int32_t v0, v1;
    share_of(c, psplit, qrow / 16, v0, v1);
    if (m && !swizzled && MX) {
      int32_t s0, s1;
      share_of(c, psplit, srow, s0, s1);
      uint32_t mm = m;
      const uint4 zero = make_uint4(0, 0, 0, 0);
      while (mm) {
        const int j = __ffs(mm) - 1;
        mm &= mm - 1;
        const int64_t row = g * kWarp + j;
        uint4 *dst = reinterpret_cast<uint4 *>(q) + row * (qrow / 16);
        for (int v = v0 + lane; v < v1; v += kWarp) st_v4(dst + v, zero);
        for (int v = s0 + lane; v < s1; v += kWarp) scales[row * srow + v] = 0;
      }
    } else if (m && !swizzled) {
      int32_t s0, s1;
      share_of(c, psplit, srow / 2, s0, s1);
      zero_rows(m, g, lane, reinterpret_cast<uint4 *>(q), qrow / 16, v0, v1,
                reinterpret_cast<uint16_t *>(scales), srow / 2, s0, s1);
    } else if (m) {
      int32_t g0, g1;
      share_of(c, psplit, groups, g0, g1);
      uint32_t mm = m;
      const uint4 zero = make_uint4(0, 0, 0, 0);
      while (mm) {
        const int j = __ffs(mm) - 1;
        mm &= mm - 1;
        const int64_t row = g * kWarp + j;
        if (row < rows) {
          uint4 *dst = reinterpret_cast<uint4 *>(q) + row * (qrow / 16);
          for (int v = v0 + lane; v < v1; v += kWarp) st_v4(dst + v, zero);
        }
        for (int gg = g0 + lane; gg < g1; gg += kWarp) {
          const int64_t off = sf_atom_offset(row, 4 * gg, groups);
          if (MOE_IN_RANGE(off, check_rows * groups * 4, kDbgScaleOffset))
            st_u32_evict_last(scales + off, 0u);
        }
      }
    }
    return;
  }
  const int64_t w = w0 - pad_units;

  if (w < units) {
    const int64_t t = w / chunks;
    const int col = (int)(w % chunks) * kChunk + lane * 32;
    const bool active = col < H;
    const uint4 *src = hidden + t * vecs;
    uint4 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      x[i] = active ? ld_stream_v4(src + col / 8 + i) : make_uint4(0, 0, 0, 0);
    int32_t my_slot;
    uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
    const float gs = MX ? 0.0f : __ldg(global_scale);
    // x[i] holds the lane's elements 8i..8i+7.  MXFP4 unpacks its one
    // 32-element block; NVFP4 unpacks one 16-element block at a time, so
    // that only 16 floats are live (under the 5-CTA bound the 32-float form
    // spilled 40 bytes per thread: 7 local stores and 10 local loads per
    // unit, now 1 and 4, and none at 4 CTAs per SM; measured on B200 at the
    // metric shape: 71.5 -> 69.0 us)
    float f[MX ? 32 : 16];
    const auto unpack = [&](int i0, int n) {
#pragma unroll
      for (int i = 0; i < n; ++i) {
        const uint32_t wd[4] = {x[i0 + i].x, x[i0 + i].y, x[i0 + i].z, x[i0 + i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f[8 * i + 2 * e] = bf16lo(wd[e]);
          f[8 * i + 2 * e + 1] = bf16hi(wd[e]);
        }
      }
    };
    uint4 codes;
    uint32_t sq, quad;
    if constexpr (MX) {
      unpack(0, 4);
      sq = mxfp4_block(f, codes);
      // atom layout: lanes 4g..4g+3 hold scale columns 4g..4g+3 -- one
      // 4-byte store per four lanes (inactive lanes contribute zeros: the
      // column padding of a partial last group)
      const uint32_t a = active ? sq : 0u;
      quad = a | (__shfl_down_sync(kFull, a, 1) << 8) | (__shfl_down_sync(kFull, a, 2) << 16) |
             (__shfl_down_sync(kFull, a, 3) << 24);
    } else {
      unpack(0, 2);
      const uint32_t sq0 = nvfp4_block(f, gs, codes.x, codes.y);
      unpack(2, 2);
      const uint32_t sq1 = nvfp4_block(f, gs, codes.z, codes.w);
      sq = sq0 | (sq1 << 8);
      // atom layout: an even lane holds scale columns 4g, 4g+1 and its odd
      // neighbour 4g+2, 4g+3 -- one 4-byte store per pair of lanes (an
      // inactive neighbour contributes zeros: the column padding of a
      // partial last group)
      quad = sq | (__shfl_down_sync(kFull, active ? sq : 0u, 1) << 16);
    }
    const int sc_col = MX ? col / 32 : col / 16;
    while (live) {
      const int j = __ffs(live) - 1;
      live &= live - 1;
      const int64_t s = __shfl_sync(kFull, my_slot, j);
      if (active && MOE_IN_RANGE(s, rows, kDbgPermuteRow)) {
        st_v4(reinterpret_cast<uint4 *>(q + s * qrow + col / 2), codes);
        if (!swizzled) {
          if (MX) scales[s * srow + sc_col] = (uint8_t)sq;
          else *reinterpret_cast<uint16_t *>(scales + s * srow + sc_col) = (uint16_t)sq;
        } else if ((lane & (MX ? 3 : 1)) == 0) {
          const int64_t off = sf_atom_offset(s, sc_col, groups);
          if (MOE_IN_RANGE(off, check_rows * groups * 4, kDbgScaleOffset))
            st_u32_evict_last(scales + off, quad);
        }
      }
    }
  }
}

// ------------------------------------------- quantised dispatch to peers
// The FP8 and NVFP4 dispatches with the send fused in, as
// permute_to_peers_kernel does for bf16 rows: the codes and the linear
// scales of local row r of segment s are stored into rank s's receive
// buffers peer_codes[s] / peer_scales[s] at row put[s] + (r - start_s), in
// the layouts of moe_permute_quant_fp8 / moe_permute_quant_nvfp4 (row-major
// scales).  The units and arithmetic of permute_fp8_kernel and of
// permute_fp4_kernel's NVFP4 path; a lane holding pair j finds its row's
// segment and receive row, and the warp broadcasts both.  Padding rows
// inside a segment are zeroed at the destination; rows past the last
// segment are not sent.
__global__ void __launch_bounds__(kThreads)
    permute_fp8_to_peers_kernel(const uint4 *__restrict__ hidden,
                                const int32_t *__restrict__ row_src,
                                const int32_t *__restrict__ pair_slot,
                                const uint32_t *__restrict__ meta,
                                uint8_t *const *__restrict__ peer_codes,
                                float *const *__restrict__ peer_scales,
                                const int64_t *__restrict__ put, int32_t N, int32_t k,
                                int64_t rows, int32_t H, int32_t chunks, int32_t psplit, int32_t S,
                                int32_t static_seg_rows) {
  MOE_TRACE_CTA(MOE_TRACE_PERMUTE_FP8_TO_PEERS, 0);
  allow_dependents();
  extern __shared__ uint64_t table_smem[];
  grid_dependency_wait();
  const PeerTable tab =
      stage_peer_table(table_smem, meta, S, H, static_seg_rows,
                       peer_codes, reinterpret_cast<uint8_t *const *>(peer_scales), put);
  __syncthreads();
  constexpr int U = kChunk / 512;  // 2
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  const int64_t pad_units = (rows + kWarp - 1) / kWarp * psplit;
  const int32_t vecs = H / 8;
  const int32_t nb = H / 128;
  if (w0 < pad_units) {
    const int64_t g = w0 / psplit;
    uint32_t m = padding_mask(g, lane, row_src, rows, rows);
    const int c = (int)(w0 % psplit);
    int32_t v0, v1, s0, s1;
    share_of(c, psplit, H / 16, v0, v1);
    share_of(c, psplit, nb, s0, s1);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      uint8_t *q, *sc;
      if (!peer_rows(g * kWarp + j, tab, S, H, 4 * nb, q, sc)) continue;
      uint4 *qd = reinterpret_cast<uint4 *>(q);
      float *sd = reinterpret_cast<float *>(sc);
      for (int v = v0 + lane; v < v1; v += kWarp) st_v4(qd + v, zero);
      for (int v = s0 + lane; v < s1; v += kWarp) sd[v] = 0.0f;
    }
    return;
  }
  const int64_t w = w0 - pad_units;
  if (w >= units) return;
  const int64_t t = w / chunks;
  const int c0 = (int)(w % chunks) * kChunk;
  const uint4 *src = hidden + t * vecs;
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
  int32_t my_slot;
  uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
  // this lane's pair: its receive rows (resolved before the quantisation, so
  // the pointer loads overlap it)
  uint8_t *my_q = nullptr, *my_s = nullptr;
  const bool mine = my_slot >= 0 && peer_rows(my_slot, tab, S, H, 4 * nb, my_q, my_s);
  live &= __ballot_sync(kFull, mine);
  uint4 codes[U];
  float scale[U];
#pragma unroll
  for (int u = 0; u < U; ++u) scale[u] = fp8_quant16(a[u], b[u], codes[u]);
  while (live) {
    const int j = __ffs(live) - 1;
    live &= live - 1;
    uint8_t *qd = reinterpret_cast<uint8_t *>(
        __shfl_sync(kFull, reinterpret_cast<unsigned long long>(my_q), j));
    float *sd = reinterpret_cast<float *>(
        __shfl_sync(kFull, reinterpret_cast<unsigned long long>(my_s), j));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int col = c0 + u * 512 + lane * 16;
      if (col < H) {
        st_v4(reinterpret_cast<uint4 *>(qd + col), codes[u]);
        if ((lane & 7) == 0) sd[col / 128] = scale[u];
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 4)
    permute_nvfp4_to_peers_kernel(const uint4 *__restrict__ hidden,
                                  const int32_t *__restrict__ row_src,
                                  const int32_t *__restrict__ pair_slot,
                                  const uint32_t *__restrict__ meta,
                                  const float *__restrict__ global_scale,
                                  uint8_t *const *__restrict__ peer_codes,
                                  uint8_t *const *__restrict__ peer_scales,
                                  const int64_t *__restrict__ put, int32_t N, int32_t k,
                                  int64_t rows, int32_t H, int32_t chunks, int32_t psplit,
                                  int32_t S, int32_t static_seg_rows) {
  MOE_TRACE_CTA(MOE_TRACE_PERMUTE_NVFP4_TO_PEERS, 0);
  allow_dependents();
  extern __shared__ uint64_t table_smem[];
  grid_dependency_wait();
  const PeerTable tab =
      stage_peer_table(table_smem, meta, S, H, static_seg_rows, peer_codes, peer_scales, put);
  __syncthreads();
  const int lane = threadIdx.x % kWarp;
  const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  const int64_t units = (int64_t)N * chunks;
  const int64_t pad_units = (rows + kWarp - 1) / kWarp * psplit;
  const int32_t vecs = H / 8;
  const int32_t qrow = H / 2, srow = H / 16;
  if (w0 < pad_units) {
    const int64_t g = w0 / psplit;
    uint32_t m = padding_mask(g, lane, row_src, rows, rows);
    const int c = (int)(w0 % psplit);
    int32_t v0, v1, s0, s1;
    share_of(c, psplit, qrow / 16, v0, v1);  // 16-byte code vectors
    share_of(c, psplit, srow / 2, s0, s1);   // 2-byte scale pairs
    const uint4 zero = make_uint4(0, 0, 0, 0);
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1;
      uint8_t *q, *sc;
      if (!peer_rows(g * kWarp + j, tab, S, qrow, srow, q, sc)) continue;
      uint4 *qd = reinterpret_cast<uint4 *>(q);
      uint16_t *sd = reinterpret_cast<uint16_t *>(sc);
      for (int v = v0 + lane; v < v1; v += kWarp) st_v4(qd + v, zero);
      for (int v = s0 + lane; v < s1; v += kWarp) sd[v] = 0;
    }
    return;
  }
  const int64_t w = w0 - pad_units;
  if (w >= units) return;
  const int64_t t = w / chunks;
  const int col = (int)(w % chunks) * kChunk + lane * 32;
  const bool active = col < H;
  const uint4 *src = hidden + t * vecs;
  uint4 x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    x[i] = active ? ld_stream_v4(src + col / 8 + i) : make_uint4(0, 0, 0, 0);
  int32_t my_slot;
  uint32_t live = load_token_slots(pair_slot, t, k, rows, lane, my_slot);
  // this lane's pair: its receive rows (resolved before the quantisation, so
  // the pointer loads overlap it)
  uint8_t *my_q = nullptr, *my_s = nullptr;
  const bool mine = my_slot >= 0 && peer_rows(my_slot, tab, S, qrow, srow, my_q, my_s);
  live &= __ballot_sync(kFull, mine);
  const float gs = __ldg(global_scale);
  // two 16-element blocks, one at a time (16 floats live)
  float f[16];
  uint4 codes;
  uint32_t sq = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 v = x[2 * h + i];
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[8 * i + 2 * e] = bf16lo(wd[e]);
        f[8 * i + 2 * e + 1] = bf16hi(wd[e]);
      }
    }
    uint32_t lo, hi;
    sq |= nvfp4_block(f, gs, lo, hi) << (8 * h);
    if (h == 0) {
      codes.x = lo;
      codes.y = hi;
    } else {
      codes.z = lo;
      codes.w = hi;
    }
  }
  while (live) {
    const int j = __ffs(live) - 1;
    live &= live - 1;
    uint8_t *qd = reinterpret_cast<uint8_t *>(
        __shfl_sync(kFull, reinterpret_cast<unsigned long long>(my_q), j));
    uint8_t *sd = reinterpret_cast<uint8_t *>(
        __shfl_sync(kFull, reinterpret_cast<unsigned long long>(my_s), j));
    if (active) {
      st_v4(reinterpret_cast<uint4 *>(qd + col / 2), codes);
      *reinterpret_cast<uint16_t *>(sd + col / 16) = (uint16_t)sq;
    }
  }
}

// Block-scale atom layout from linear scales, in place, one CTA per 128-row
// tile.  When the scale columns per row (nsf) are a multiple of 4, a tile's
// linear scales ([128, nsf] row-major, rows past `rows` unwritten) and its
// atoms (nsf/4 atoms of 512 bytes) occupy the same bytes of the buffer, so
// the permute writes linear scales there first (whole 64- or 32-byte runs
// per warp instead of 4-byte pieces of 8 different rows per 32-byte sector)
// and this kernel reads the whole tile into shared memory, then writes it
// back in atom order; rows at or past `rows` become zeros.  (Leaving the
// padding rows' scales to this kernel -- the permute skips them, this kernel
// reads row_src first and loads only rows that hold a token -- measured the
// same on B200 at the metric shape with 128-padded experts: the permute
// 4 us faster, this kernel 3.5 us slower.)  Shared layout:
// word (m, g) of 4-scale group g at g * 129 + (m % 32) * 4 + m / 32 -- the
// atom order, so the write-back reads consecutive words, padded by one word
// per group so that the scattered writes of a warp (consecutive g) fall in
// distinct banks.
constexpr int kAtomThreads = 256;
constexpr int kAtomGroupWords = 129;

inline size_t atom_tile_smem(int32_t nsf) {  // the larger of the two layouts
  return (size_t)(nsf / 4) * kAtomGroupWords * sizeof(uint32_t);
}

// VEC: the buffer is 16-byte aligned and the groups per row a multiple of
// 4, and the tile moves as 16-byte vectors, kAtomBatch loads in flight per
// thread before their shared-memory stores; else as 4-byte words through the
// padded layout above.  VEC shared layout: group g's 128 words in atom order
// as 32 chunks of 4 (chunk c = m % 32 holds m / 32 = 0..3), with the chunk
// index XORed by (g / 4) % 8 and the words of a chunk rotated by
// (g / 32) % 4.  A warp's scatter of one word per thread (32 consecutive
// values of g / 4, one m) then falls in 32 distinct banks, and the
// write-back reads each chunk as one 16-byte shared load (a warp reads one
// group's 512 bytes, no conflict) and undoes the rotation in registers.
constexpr int kAtomBatch = 8;

__device__ __forceinline__ uint32_t atom_vec_slot(int32_t m, int32_t g) {
  const int32_t q = g >> 2;
  return (uint32_t)g * 128u + (uint32_t)(((m & 31) ^ (q & 7)) * 4 + (((m >> 5) + (q >> 3)) & 3));
}

template <bool VEC>
__global__ void __launch_bounds__(kAtomThreads)
    scales_to_atoms_kernel(uint32_t *__restrict__ scales, int64_t rows, int32_t groups) {
  MOE_TRACE_CTA(MOE_TRACE_SCALES_TO_ATOMS, VEC ? 1 : 0);
  allow_dependents();
  extern __shared__ uint32_t tile_words[];
  grid_dependency_wait();
  const int64_t tile = blockIdx.x;
  const int64_t left = rows - tile * 128;
  const int32_t nrows = left < 128 ? (int32_t)left : 128;
  uint32_t *base = scales + tile * 128 * groups;  // the tile's words (either layout)
  const int32_t words = 128 * groups;
  const auto put = [&](int32_t w, uint32_t v) {  // linear word w -> shared, atom order
    const int32_t m = w / groups, g = w - m * groups;
    tile_words[g * kAtomGroupWords + (m & 31) * 4 + (m >> 5)] = m < nrows ? v : 0u;
  };
  if constexpr (VEC) {
    // groups % 4 == 0 (the scale columns are a multiple of 16), so a vector
    // never straddles two rows
    const uint4 *vb = reinterpret_cast<const uint4 *>(base);
    const int32_t vecs = words / 4;
    const int32_t valid = nrows * groups / 4;  // vectors of rows < nrows
    for (int32_t v0 = threadIdx.x; v0 < vecs; v0 += kAtomThreads * kAtomBatch) {
      uint4 x[kAtomBatch];
#pragma unroll
      for (int b = 0; b < kAtomBatch; ++b) {
        const int32_t v = v0 + b * kAtomThreads;
        x[b] = v < valid ? vb[v] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int b = 0; b < kAtomBatch; ++b) {
        const int32_t v = v0 + b * kAtomThreads;
        if (v < vecs) {  // words (m, g0 .. g0 + 3); rows past nrows were loaded as 0
          const int32_t m = 4 * v / groups, g0 = 4 * v - m * groups;
          uint32_t *t = tile_words + atom_vec_slot(m, g0);  // g0 .. g0+3 share g / 4
          t[0] = x[b].x;
          t[128] = x[b].y;
          t[256] = x[b].z;
          t[384] = x[b].w;
        }
      }
    }
    __syncthreads();
    uint4 *ob = reinterpret_cast<uint4 *>(base);
    for (int32_t v = threadIdx.x; v < vecs; v += kAtomThreads) {
      // output vector v: group g = v / 32, atom chunk c = v % 32
      const int32_t g = v >> 5, c = v & 31, q = g >> 2;
      const uint4 p = *reinterpret_cast<const uint4 *>(tile_words + g * 128 + (c ^ (q & 7)) * 4);
      uint4 o;
      switch ((q >> 3) & 3) {  // word o of the chunk sits at (o + r) % 4
        case 0: o = p; break;
        case 1: o = make_uint4(p.y, p.z, p.w, p.x); break;
        case 2: o = make_uint4(p.z, p.w, p.x, p.y); break;
        default: o = make_uint4(p.w, p.x, p.y, p.z); break;
      }
      ob[v] = o;
    }
  } else {
    for (int32_t w = threadIdx.x; w < words; w += kAtomThreads) put(w, w < nrows * groups ? base[w] : 0u);
    __syncthreads();
    for (int32_t w = threadIdx.x; w < words; w += kAtomThreads) {
      const int32_t g = w >> 7, wi = w & 127;
      base[w] = tile_words[g * kAtomGroupWords + wi];
    }
  }
}

// Padding warps per 32-row group: when the problem has more rows than pairs
// (capacity layouts, padded experts, a recv_capacity above N*k) some rows
// are certainly padding, and a group of 32 padding rows is shared by as many
// warps as a token row has units (each zeroes the same column share of the
// group's padding rows); otherwise one warp per group, which exits at once
// when its rows all have a source.  Measured on B200 at N=128, H=7168,
// E=256, k=8 with [256, 5] rows (340 padding rows): bf16 25.3 us with one
// warp per group.
inline int32_t padding_split(const Shape &s, int32_t chunks) {
  return s.rows > s.P ? chunks : 1;
}

// One warp per unit: ceil(check_rows / 32) * psplit padding warps, then
// N * chunks token units.
inline int64_t unit_blocks(const Shape &s, int32_t chunks, int64_t check_rows, int32_t psplit) {
  const int64_t warps = (check_rows + kWarp - 1) / kWarp * psplit + (int64_t)s.N * chunks;
  return std::max<int64_t>(1, (warps + kThreads / kWarp - 1) / (kThreads / kWarp));
}

inline int32_t chunks_of(int32_t H, int32_t chunk) { return (H + chunk - 1) / chunk; }

}  // namespace

uint32_t debug_violations_permute(bool reset) { return read_debug_violations(reset); }

#ifdef MOE_TRACE
cudaError_t trace_attach_permute(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                                 cudaStream_t stream) {
  return trace_attach_tu(records, count, capacity, stream);
}
#endif

cudaError_t launch_permute_bf16(const Shape &s, const void *hidden, const int32_t *row_src,
                                const int32_t *pair_slot, void *out, cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kBf16Chunk);
  const int32_t ps = padding_split(s, chunks);
  return launch_pdl(permute_bf16_kernel, dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)),
                    dim3(kThreads), 0, stream, static_cast<const uint4 *>(hidden), row_src,
                    pair_slot, static_cast<uint4 *>(out), s.N, s.k, s.rows, s.H / 8, chunks, ps);
}

cudaError_t launch_permute_premultiplied(const Shape &s, const void *hidden,
                                         const int32_t *row_src, const int32_t *pair_slot,
                                         const float *gates, void *out, cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kBf16Chunk);
  const int32_t ps = padding_split(s, chunks);
  return launch_pdl(permute_premultiplied_kernel,
                    dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)), dim3(kThreads), 0, stream,
                    static_cast<const uint4 *>(hidden), row_src, pair_slot, gates,
                    static_cast<uint4 *>(out), s.N, s.k, s.rows, s.H / 8, chunks, ps);
}

cudaError_t launch_permute_to_peers(const Shape &s, const void *hidden, const int32_t *row_src,
                                    const int32_t *pair_slot, const uint32_t *meta,
                                    void *const *peer_out, const int64_t *put_offsets,
                                    cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kBf16Chunk);
  const int32_t ps = padding_split(s, chunks);
  const int32_t static_seg = s.Ce > 0 ? (s.E / s.S) * s.Ce : 0;
  return launch_pdl(permute_to_peers_kernel, dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)),
                    dim3(kThreads), (size_t)2 * s.S * sizeof(int32_t), stream,
                    static_cast<const uint4 *>(hidden), row_src, pair_slot, meta,
                    reinterpret_cast<uint4 *const *>(peer_out), put_offsets, s.N, s.k, s.rows,
                    s.H / 8, chunks, ps, s.S, s.H, static_seg);
}

// Shared memory of the quantised peer kernels' table (PeerTable), and the
// opt-in a kernel needs above the default 48 KB (S up to 2048: 64 KB).
inline size_t peer_table_smem(int32_t S) { return (size_t)32 * S; }
template <typename K>
cudaError_t allow_smem(K kernel, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t launch_permute_fp8_to_peers(const Shape &s, const void *hidden,
                                       const int32_t *row_src, const int32_t *pair_slot,
                                       const uint32_t *meta, void *const *peer_codes,
                                       void *const *peer_scales, const int64_t *put_offsets,
                                       cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kChunk);
  const int32_t ps = padding_split(s, chunks);
  const int32_t static_seg = s.Ce > 0 ? (s.E / s.S) * s.Ce : 0;
  const size_t smem = peer_table_smem(s.S);
  const cudaError_t err = allow_smem(permute_fp8_to_peers_kernel, smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(permute_fp8_to_peers_kernel,
                    dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)), dim3(kThreads), smem,
                    stream, static_cast<const uint4 *>(hidden),
                    row_src, pair_slot, meta, reinterpret_cast<uint8_t *const *>(peer_codes),
                    reinterpret_cast<float *const *>(peer_scales), put_offsets, s.N, s.k, s.rows,
                    s.H, chunks, ps, s.S, static_seg);
}

cudaError_t launch_permute_nvfp4_to_peers(const Shape &s, const void *hidden,
                                         const int32_t *row_src, const int32_t *pair_slot,
                                         const uint32_t *meta, const float *global_scale,
                                         void *const *peer_codes, void *const *peer_scales,
                                         const int64_t *put_offsets, cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kChunk);
  const int32_t ps = padding_split(s, chunks);
  const int32_t static_seg = s.Ce > 0 ? (s.E / s.S) * s.Ce : 0;
  const size_t smem = peer_table_smem(s.S);
  const cudaError_t err = allow_smem(permute_nvfp4_to_peers_kernel, smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(permute_nvfp4_to_peers_kernel,
                    dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)), dim3(kThreads), smem,
                    stream, static_cast<const uint4 *>(hidden),
                    row_src, pair_slot, meta, global_scale,
                    reinterpret_cast<uint8_t *const *>(peer_codes),
                    reinterpret_cast<uint8_t *const *>(peer_scales), put_offsets, s.N, s.k,
                    s.rows, s.H, chunks, ps, s.S, static_seg);
}

cudaError_t launch_permute_fp8(const Shape &s, const void *hidden, const int32_t *row_src,
                               const int32_t *pair_slot, uint8_t *q, float *scales,
                               cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kChunk);
  const int32_t ps = padding_split(s, chunks);
  return launch_pdl(permute_fp8_kernel, dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)),
                    dim3(kThreads), 0, stream, static_cast<const uint4 *>(hidden), row_src,
                    pair_slot, q, scales, s.N, s.k, s.rows, s.H, chunks, ps);
}

// Atom-layout scales through linear scales and the in-place tile kernel:
// possible when the scale columns per row are a multiple of 4 and a tile's
// scales fit in shared memory.
inline bool atoms_in_place(int32_t nsf) {
  return nsf % 4 == 0 && atom_tile_smem(nsf) <= 200 * 1024;
}

cudaError_t launch_scales_to_atoms(const Shape &s, int32_t nsf, uint8_t *scales,
                                   cudaStream_t stream) {
  const bool vec = reinterpret_cast<uintptr_t>(scales) % 16 == 0 && (nsf / 4) % 4 == 0;
  // both layouts get the padded size: 3 tiles per SM at H = 7168 (the
  // vector layout's exact 56 KB would fit 4; measured slower on B200, 19.1
  // vs 17.9 us for the f1 dispatch's 766 tiles)
  const size_t smem = atom_tile_smem(nsf);
  auto kernel = vec ? scales_to_atoms_kernel<true> : scales_to_atoms_kernel<false>;
  if (smem > 48 * 1024) {
    const cudaError_t err =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(kernel, dim3((unsigned)((s.rows + 127) / 128)), dim3(kAtomThreads), smem,
                    stream, reinterpret_cast<uint32_t *>(scales), s.rows, nsf / 4);
}

cudaError_t launch_permute_nvfp4(const Shape &s, const void *hidden, const int32_t *row_src,
                                 const int32_t *pair_slot, const float *global_scale,
                                 uint8_t *q, uint8_t *scales, cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kChunk);
  const bool swizzled = (s.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES) != 0;
  const int32_t ps = padding_split(s, chunks);
  if (swizzled && atoms_in_place(s.H / 16)) {
    const cudaError_t err = launch_pdl(
        permute_fp4_kernel<false, false>, dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)),
        dim3(kThreads), 0, stream, static_cast<const uint4 *>(hidden), row_src, pair_slot,
        global_scale, q, scales, s.N, s.k, s.rows, s.H, chunks, ps);
    if (err != cudaSuccess) return err;
    return launch_scales_to_atoms(s, s.H / 16, scales, stream);
  }
  const int64_t check_rows = swizzled ? (s.rows + 127) / 128 * 128 : s.rows;
  return launch_pdl(swizzled ? permute_fp4_kernel<false, true> : permute_fp4_kernel<false, false>,
                    dim3((unsigned)unit_blocks(s, chunks, check_rows, ps)), dim3(kThreads), 0,
                    stream, static_cast<const uint4 *>(hidden), row_src, pair_slot, global_scale,
                    q, scales, s.N, s.k, s.rows, s.H, chunks, ps);
}

cudaError_t launch_permute_mxfp4(const Shape &s, const void *hidden, const int32_t *row_src,
                                 const int32_t *pair_slot, uint8_t *q, uint8_t *scales,
                                 cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const int32_t chunks = chunks_of(s.H, kChunk);
  const bool swizzled = (s.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES) != 0;
  const int32_t ps = padding_split(s, chunks);
  if (swizzled && atoms_in_place(s.H / 32)) {
    const cudaError_t err = launch_pdl(
        permute_fp4_kernel<true, false>, dim3((unsigned)unit_blocks(s, chunks, s.rows, ps)),
        dim3(kThreads), 0, stream, static_cast<const uint4 *>(hidden), row_src, pair_slot,
        static_cast<const float *>(nullptr), q, scales, s.N, s.k, s.rows, s.H, chunks, ps);
    if (err != cudaSuccess) return err;
    return launch_scales_to_atoms(s, s.H / 32, scales, stream);
  }
  const int64_t check_rows = swizzled ? (s.rows + 127) / 128 * 128 : s.rows;
  return launch_pdl(swizzled ? permute_fp4_kernel<true, true> : permute_fp4_kernel<true, false>,
                    dim3((unsigned)unit_blocks(s, chunks, check_rows, ps)), dim3(kThreads), 0,
                    stream, static_cast<const uint4 *>(hidden), row_src, pair_slot,
                    static_cast<const float *>(nullptr), q, scales, s.N, s.k, s.rows, s.H,
                    chunks, ps);
}

}  // namespace moe
