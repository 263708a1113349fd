// swiglu.cu -- fused SwiGLU + requantisation of the experts' gate/up rows
// (Mojo MAX ep_comm: fused_silu_kernel, fused_silu_mx_kernel,
// fused_silu_nvfp4_kernel, fused_silu_mxfp8_interleaved_kernel; MXTokenFormat).
//
// For every dispatch row r with a routed token (row_src[r] >= 0 -- the
// layout's answer to how many rows were received, read on the device),
// y = silu(gate) * up in fp32 and y is quantised to NVFP4 (E2M1 + E4M3 per 16
// + global scale, as the dispatch does), MXFP8 (E4M3 + E8M0 per 32) or MXFP4
// (E2M1 + E8M0 per 32).  Rows without a token are zero bytes and their input
// is not read.
//
// e^x is one fixed fp32 operation sequence (Cody-Waite range reduction, the
// degree-7 Taylor polynomial in Horner form with fmaf, scaling by 2^n;
// Cody & Waite, Software Manual for the Elementary Functions, 1980), not the
// library expf, so that the quantised codes are a reproducible function of
// the inputs.  Products and sums outside it use __fmul_rn / __fadd_rn so the
// compiler cannot contract them.
//
// One warp per unit (row, 1024 columns of the intermediate size I); a lane
// owns 32 consecutive columns: eight 16-byte loads of gate/up, one MX block
// or two NVFP4 blocks.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr int kUnitCols = 1024;

__device__ __forceinline__ float pow2i(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }

__device__ __forceinline__ float fixed_exp(float x) {
  if (x != x) return x;
  if (x > 88.75f) return __uint_as_float(0x7F800000u);
  if (x < -104.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, 1.44269504f));
  float r = fmaf(-n, 0.693145751953125f, x);
  r = fmaf(-n, 1.42860682e-06f, r);
  float p = 1.98412698e-04f;
  p = fmaf(p, r, 1.38888889e-03f);
  p = fmaf(p, r, 8.33333333e-03f);
  p = fmaf(p, r, 4.16666667e-02f);
  p = fmaf(p, r, 1.66666667e-01f);
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  const int ni = (int)n;
  if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2i(127)), pow2i(ni - 127));
  if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2i(ni + 64)), pow2i(-64));
  return __fmul_rn(p, pow2i(ni));
}

__device__ __forceinline__ float swiglu(float g, float u) {
  const float silu = __fdiv_rn(g, __fadd_rn(1.0f, fixed_exp(-g)));
  return __fmul_rn(silu, u);
}

// floor(log2(a)) of a finite a > 0, subnormals included.
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = (int)((b >> 23) & 0xFFu);
  if (e != 0) return e - 127;
  return (31 - __clz((int)(b & 0x7FFFFFu))) - 149;
}

// y * 2^-X for X in [-127, 127], as two exact scalings when 2^-X alone is not
// a normal float.
__device__ __forceinline__ float scale_down(float y, int X) {
  return -X >= -126 ? __fmul_rn(y, pow2i(-X)) : __fmul_rn(__fmul_rn(y, pow2i(-X - 64)), pow2i(64));
}

template <int FORMAT, bool INTERLEAVED>
__global__ void __launch_bounds__(kThreads)
    swiglu_quant_kernel(const uint4 *__restrict__ gate_up, const int32_t *__restrict__ row_src,
                        const float *__restrict__ global_scale, uint8_t *__restrict__ codes,
                        uint8_t *__restrict__ scales, int64_t rows, int32_t I, int32_t chunks) {
  const int lane = threadIdx.x % kWarp;
  const int64_t w = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kWarp;
  if (w >= rows * chunks) return;
  const int64_t r = w / chunks;
  const int c = (int)(w % chunks) * kUnitCols + lane * 32;
  const bool active = c < I;
  const int64_t code_row = FORMAT == 1 ? I : I / 2;
  const int64_t scale_row = FORMAT == 0 ? I / 16 : I / 32;
  uint8_t *cd = codes + r * code_row + (FORMAT == 1 ? c : c / 2);
  uint8_t *sd = scales + r * scale_row + (FORMAT == 0 ? c / 16 : c / 32);
  if (!active) return;

  if (__ldg(row_src + r) < 0) {  // no routed token: zero bytes, input not read
    const uint4 zero = make_uint4(0, 0, 0, 0);
    st_v4(reinterpret_cast<uint4 *>(cd), zero);
    if (FORMAT == 1) st_v4(reinterpret_cast<uint4 *>(cd) + 1, zero);
    if (FORMAT == 0) *reinterpret_cast<uint16_t *>(sd) = 0;
    else *sd = 0;
    return;
  }

  // ---- 32 gate and 32 up values
  const int64_t row_vecs = (int64_t)I / 4;  // 2I bf16 = I/4 vectors of 8
  const uint4 *in = gate_up + r * row_vecs;
  uint4 gv[4], uv[4];
  if (INTERLEAVED) {
    uint4 iv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) iv[i] = ld_stream_v4(in + c / 4 + i);
    // element pairs (g, u) in each 32-bit word
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 a = iv[2 * i], b = iv[2 * i + 1];
      gv[i] = make_uint4(__byte_perm(a.x, a.y, 0x5410), __byte_perm(a.z, a.w, 0x5410),
                         __byte_perm(b.x, b.y, 0x5410), __byte_perm(b.z, b.w, 0x5410));
      uv[i] = make_uint4(__byte_perm(a.x, a.y, 0x7632), __byte_perm(a.z, a.w, 0x7632),
                         __byte_perm(b.x, b.y, 0x7632), __byte_perm(b.z, b.w, 0x7632));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      gv[i] = ld_stream_v4(in + c / 8 + i);
      uv[i] = ld_stream_v4(in + I / 8 + c / 8 + i);
    }
  }
  float y[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t g4[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
    const uint32_t u4[4] = {uv[i].x, uv[i].y, uv[i].z, uv[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      y[8 * i + 2 * e] = swiglu(bf16lo(g4[e]), bf16lo(u4[e]));
      y[8 * i + 2 * e + 1] = swiglu(bf16hi(g4[e]), bf16hi(u4[e]));
    }
  }

  if (FORMAT == 0) {
    // ---- NVFP4: the dispatch's rule on the fp32 values, two blocks of 16
    const float gs = __ldg(global_scale);
    uint32_t cw[4] = {0, 0, 0, 0};
    uint32_t sq2 = 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[16 * b + i]));
      const uint32_t sq = cvt_e4m3x2(__fdiv_rn(__fdiv_rn(amax, 6.0f), gs), 0.0f) & 0xFFu;
      const float d = __fmul_rn(e4m3_to_float(sq), gs);
      sq2 |= sq << (8 * b);
      if (d > 0.0f) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t word = 0;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int i = 16 * b + 8 * h + 2 * m;
            word |= cvt_e2m1x2(__fdiv_rn(y[i], d), __fdiv_rn(y[i + 1], d)) << (8 * m);
          }
          cw[2 * b + h] = word;
        }
      }
    }
    st_v4(reinterpret_cast<uint4 *>(cd), make_uint4(cw[0], cw[1], cw[2], cw[3]));
    *reinterpret_cast<uint16_t *>(sd) = (uint16_t)sq2;
  } else {
    // ---- MX: one block of 32, E8M0 scale 2^X, X = floor(log2 amax) - emax
    constexpr int kEmax = FORMAT == 1 ? 8 : 2;
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(y[i]));
    uint32_t sc = 0;
    uint32_t cw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (amax > 0.0f) {
      sc = (uint32_t)min(254, max(0, floor_log2(amax) - kEmax + 127));
      const int X = (int)sc - 127;
      if (FORMAT == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t lo = cvt_e4m3x2(scale_down(y[4 * i], X), scale_down(y[4 * i + 1], X));
          const uint32_t hi =
              cvt_e4m3x2(scale_down(y[4 * i + 2], X), scale_down(y[4 * i + 3], X));
          cw[i] = lo | (hi << 16);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t word = 0;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int e = 8 * i + 2 * m;
            word |= cvt_e2m1x2(scale_down(y[e], X), scale_down(y[e + 1], X)) << (8 * m);
          }
          cw[i] = word;
        }
      }
    }
    st_v4(reinterpret_cast<uint4 *>(cd), make_uint4(cw[0], cw[1], cw[2], cw[3]));
    if (FORMAT == 1)
      st_v4(reinterpret_cast<uint4 *>(cd) + 1, make_uint4(cw[4], cw[5], cw[6], cw[7]));
    *sd = (uint8_t)sc;
  }
}

template <int FORMAT, bool INTERLEAVED>
cudaError_t launch(const uint4 *in, const int32_t *row_src, const float *gs, uint8_t *codes,
                   uint8_t *scales, int64_t rows, int32_t I, cudaStream_t stream) {
  const int32_t chunks = (I + kUnitCols - 1) / kUnitCols;
  const int64_t warps = rows * chunks;
  const int64_t blocks = std::max<int64_t>(1, (warps + kThreads / kWarp - 1) / (kThreads / kWarp));
  swiglu_quant_kernel<FORMAT, INTERLEAVED><<<(unsigned)blocks, kThreads, 0, stream>>>(
      in, row_src, gs, codes, scales, rows, I, chunks);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_swiglu_quant(const Shape &s, int32_t I, uint32_t format, bool interleaved,
                                const void *gate_up, const int32_t *row_src,
                                const float *global_scale, uint8_t *codes, uint8_t *scales,
                                cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const uint4 *in = static_cast<const uint4 *>(gate_up);
  switch (format * 2 + (interleaved ? 1 : 0)) {
    case 0: return launch<0, false>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
    case 1: return launch<0, true>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
    case 2: return launch<1, false>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
    case 3: return launch<1, true>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
    case 4: return launch<2, false>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
    default: return launch<2, true>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
  }
}

}  // namespace moe
