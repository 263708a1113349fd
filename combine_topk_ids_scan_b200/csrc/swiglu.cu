// swiglu.cu -- fused SwiGLU + requantisation of the experts' gate/up rows
// (Mojo MAX ep_comm: fused_silu_kernel, fused_silu_mx_kernel,
// fused_silu_nvfp4_kernel, fused_silu_nvfp4_interleaved_kernel,
// fused_silu_mxfp8_interleaved_kernel, fused_silu_mxfp6_kernel).
//
// For every dispatch row r with a routed token (row_src[r] >= 0 -- the
// layout's answer to how many rows were received, read on the device),
// y = silu(gate) * up in fp32 and y is written as bf16 or quantised to NVFP4
// (E2M1 + E4M3 per 16 + global scale, as the dispatch does), MXFP8 (E4M3 +
// E8M0 per 32), MXFP4 (E2M1 + E8M0 per 32) or MXFP6 (E2M3 or E3M2 + E8M0 per
// 32, 6-bit codes packed four to three bytes).  Rows without a token are
// zero bytes and their input is not read.
//
// e^x is one fixed fp32 operation sequence (Cody-Waite range reduction, the
// degree-7 Taylor polynomial in Horner form with fused multiply-adds, scaling
// by 2^n; Cody & Waite, Software Manual for the Elementary Functions, 1980),
// not the library expf, so that the quantised codes are a reproducible
// function of the inputs.  The kernel evaluates it two columns at a time with
// the packed fp32x2 operations of sm_100 (__fmul2_rn, __fadd2_rn, __ffma2_rn):
// each half of a packed operation rounds exactly as the scalar operation, so
// the result is that of the scalar sequence bit for bit.
//
// silu(g) depends on the 16-bit gate value alone, so each CTA first
// evaluates it once for every bf16 g with 2^-25 <= |g| < 128 (32 binades of
// 128 significands per sign, 8192 fp32 values = 32 KB of shared memory) and
// afterwards reads it from that table.  A lane whose 32 gate values include
// one outside the table (zero, tiny, huge, inf, NaN) evaluates the same
// sequence directly, so the table changes no result, only the work.
//
// Two persistent kernels.  swiglu_quant_kernel (the NVFP4 and MXFP6
// outputs) deals the row-major list of (row, 16-column group) pairs out lane
// by lane, so no lane idles when I is not a multiple of 1024: an NVFP4 lane
// owns one whole block, so its scale work stays in one lane; an MXFP6 lane
// owns half of a 32-column block and shares the block maximum with its
// neighbour by one shuffle.  (32-column groups per lane, the first form,
// put lanes 64 bytes apart, and the L1 data path saturated.)
// swiglu_split_kernel (MXFP8, MXFP4, bf16; split or interleaved gate/up)
// gives each warp 512 columns of a row with short column runs per lane, so
// that its loads and stores are contiguous per warp instruction.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "trace.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kGroupCols = 32;  // columns of one lane

// silu table: slot (b mod 4096) + 4096 * sign for the bf16 patterns b whose
// magnitude bits lie in [0x3300, 0x4300), i.e. 2^-25 <= |g| < 2^7.  Those are
// 4096 consecutive values, so b mod 4096 is one-to-one on them.
constexpr uint32_t kTabFirst = 0x3300u;
constexpr int kTabHalf = 4096;
constexpr int kTabSize = 2 * kTabHalf;

// max / min that return NaN when either operand is NaN
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float min_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ float2 splat(float v) { return make_float2(v, v); }

// e^x of both halves.
//  * Range: the sequence gives +inf at x = 88.75 (2^128 overflows) and +0 at
//    x = -104 (below half the smallest subnormal), so clamping x to
//    [-104, 88.75] is exactly "x > 88.75 -> inf, x < -104 -> 0"; NaN passes
//    through the clamp and the arithmetic.
//  * n = rint(x log2 e) by the 1.5 * 2^23 shifter: for |t| < 2^22, t + 1.5 * 2^23
//    rounds t to the nearest integer, ties to even (the sum's unit is 1), the
//    subtraction is exact, and the integer n sits in the sum's low bits.
//  * 2^n as two normal factors 2^floor(n/2) * 2^ceil(n/2): for n in
//    [-150, 128] p * 2^floor(n/2) is exact, so the product rounds once, to
//    RN(p * 2^n), whichever way the scalar sequence splits the scaling.
__device__ __forceinline__ float2 fixed_exp2(float2 x) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  x.x = min_nan(max_nan(x.x, -104.0f), 88.75f);
  x.y = min_nan(max_nan(x.y, -104.0f), 88.75f);
  const float2 sh = __fadd2_rn(__fmul2_rn(x, splat(1.44269504f)), splat(kShift));
  const float2 n = __fadd2_rn(sh, splat(-kShift));
  float2 r = __ffma2_rn(n, splat(-0.693145751953125f), x);  // ln 2, high 16 bits
  r = __ffma2_rn(n, splat(-1.42860682e-06f), r);             // ln 2, the rest
  float2 p = splat(1.98412698e-04f);                         // 1/7!
  p = __ffma2_rn(p, r, splat(1.38888889e-03f));
  p = __ffma2_rn(p, r, splat(8.33333333e-03f));
  p = __ffma2_rn(p, r, splat(4.16666667e-02f));
  p = __ffma2_rn(p, r, splat(1.66666667e-01f));
  p = __ffma2_rn(p, r, splat(0.5f));
  p = __ffma2_rn(p, r, splat(1.0f));
  p = __ffma2_rn(p, r, splat(1.0f));
  const int n0 = __float_as_int(sh.x) - 0x4B400000, n1 = __float_as_int(sh.y) - 0x4B400000;
  p = __fmul2_rn(p, make_float2(pow2i(n0 >> 1), pow2i(n1 >> 1)));               // 2^floor(n/2)
  return __fmul2_rn(p, make_float2(pow2i((n0 + 1) >> 1), pow2i((n1 + 1) >> 1)));  // 2^ceil(n/2)
}

// silu(g) = g / (1 + e^-g) of both halves; IEEE division.
__device__ __forceinline__ float2 silu2(float2 g) {
  const float2 d = __fadd2_rn(splat(1.0f), fixed_exp2(make_float2(-g.x, -g.y)));
  return make_float2(__fdiv_rn(g.x, d.x), __fdiv_rn(g.y, d.y));
}

// The gate value of table slot i.
__device__ __forceinline__ float tab_gate(int i) {
  const uint32_t mag = kTabFirst + (((uint32_t)i - kTabFirst) & 0xFFFu);
  return __uint_as_float((((uint32_t)(i >> 12) << 15) | mag) << 16);
}

// Byte offsets into the table of the low and high bf16 of a 32-bit word:
// 4 * ((b & 0xFFF) | (sign << 12)) for each half b.
__device__ __forceinline__ void table_offsets(uint32_t w, uint32_t &lo, uint32_t &hi) {
  const uint32_t m = ((w << 2) & 0x3FFC3FFCu) | ((w >> 1) & 0x40004000u);
  lo = m & 0x7FFCu;
  hi = m >> 16;
}
__device__ __forceinline__ float table_at(const float *tab, uint32_t off) {
  return *reinterpret_cast<const float *>(reinterpret_cast<const char *>(tab) + off);
}

// Eight floats -> eight OCP MX FP6 codes (E2M3 or E3M2, nearest even,
// saturating), packed at bits [6i, 6i + 6) of a 48-bit little-endian value
// returned as (low 32 bits, high 16 bits).  The conversion leaves each 6-bit
// code in the low bits of its byte.
template <bool E2M3>
__device__ __forceinline__ void cvt_fp6x8(const float2 *v, uint32_t &lo32, uint32_t &hi16) {
  uint32_t p[4];  // p[i] = code(2i) | code(2i + 1) << 8
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (E2M3)
      asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e2m3x2.f32 t, %2, %1;\n\t"
          "cvt.u32.u16 %0, t;\n\t}"
          : "=r"(p[i])
          : "f"(v[i].x), "f"(v[i].y));
    else
      asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e3m2x2.f32 t, %2, %1;\n\t"
          "cvt.u32.u16 %0, t;\n\t}"
          : "=r"(p[i])
          : "f"(v[i].x), "f"(v[i].y));
  }
  // two codes a | b << 8 -> a | b << 6 (12 bits)
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = p[i] - 192u * (p[i] >> 8);
  const uint32_t g0 = q[0] | (q[1] << 12), g1 = q[2] | (q[3] << 12);  // 24 bits each
  lo32 = g0 | (g1 << 24);
  hi16 = g1 >> 8;
}

// Bits 12..15 and 28..31 of the result are zero iff both bf16 of w are in
// the table: for a magnitude in [0x3300, 0x4300), magnitude + 0x4D00 lies in
// [0x8000, 0x9000) (and never carries into the other half, being at most
// 0xCCFF), so flipping bit 15 leaves it below 0x1000.
__device__ __forceinline__ uint32_t table_check(uint32_t w) {
  return ((w & 0x7FFF7FFFu) + 0x4D004D00u) ^ 0x80008000u;
}
constexpr uint32_t kTableCheckBits = 0xF000F000u;



// One lane's 32 columns [c, c + 32) of row r.
template <int FORMAT, bool INTERLEAVED>
__device__ __forceinline__ void swiglu_group(const float *tab, const uint4 *__restrict__ gate_up,
                                             const int32_t *__restrict__ row_src, float gs,
                                             uint8_t *__restrict__ codes,
                                             uint8_t *__restrict__ scales, int64_t r, int32_t c,
                                             int32_t I) {
  // bytes of codes per column group of 32 and per row
  constexpr int kCodeBytes = FORMAT == 1 ? 32 : FORMAT == 3 ? 64 : FORMAT >= 4 ? 24 : 16;
  const int64_t code_row = (int64_t)I / 32 * kCodeBytes;
  const int64_t scale_row = FORMAT == 0 ? I / 16 : I / 32;
  uint8_t *cd = codes + r * code_row + (int64_t)(c / 32) * kCodeBytes;
  uint8_t *sd = scales + r * scale_row + (FORMAT == 0 ? c / 16 : c / 32);

  if (__ldg(row_src + r) < 0) {  // no routed token: zero bytes, input not read
    if (kCodeBytes == 24) {
      uint2 *d2 = reinterpret_cast<uint2 *>(cd);
#pragma unroll
      for (int i = 0; i < 3; ++i) d2[i] = make_uint2(0, 0);
    } else {
#pragma unroll
      for (int i = 0; i < kCodeBytes / 16; ++i) st_v4(reinterpret_cast<uint4 *>(cd) + i, make_uint4(0, 0, 0, 0));
    }
    if (FORMAT == 0) *reinterpret_cast<uint16_t *>(sd) = 0;
    else if (FORMAT != 3) *sd = 0;
    return;
  }

  // ---- 32 gate and 32 up values
  const uint4 *in = gate_up + r * ((int64_t)I / 4);  // 2I bf16 = I/4 vectors of 8
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

  // ---- y = silu(g) * u, two columns at a time: y[j] = columns 2j, 2j+1
  uint32_t check = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    check |= table_check(gv[i].x) | table_check(gv[i].y) | table_check(gv[i].z) |
             table_check(gv[i].w);
  float2 y[16];
  if ((check & kTableCheckBits) == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t g4[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t lo, hi;
        table_offsets(g4[e], lo, hi);
        y[4 * i + e] = make_float2(table_at(tab, lo), table_at(tab, hi));
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t g4[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) y[4 * i + e] = silu2(make_float2(bf16lo(g4[e]), bf16hi(g4[e])));
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u4[4] = {uv[i].x, uv[i].y, uv[i].z, uv[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      y[4 * i + e] = __fmul2_rn(y[4 * i + e], make_float2(bf16lo(u4[e]), bf16hi(u4[e])));
  }

  if (FORMAT == 3) {
    // ---- bf16, rounded to nearest even
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(y[j].x, y[j].y);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      st_v4(reinterpret_cast<uint4 *>(cd) + i,
            make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
  } else if (FORMAT >= 4) {
    // ---- MXFP6 (E2M3 emax 2, E3M2 emax 4): one block of 32, 24 bytes
    constexpr int kEmax = FORMAT == 4 ? 2 : 4;
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = max_abs3(amax, y[j].x, y[j].y);
    uint32_t sc = 0;
    uint32_t cw[6] = {0, 0, 0, 0, 0, 0};
    if (amax > 0.0f) {
      sc = mx_scale_code(amax, kEmax);
      const float2 s2 = splat(pow2i(127 - (int)sc));
      float2 v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __fmul2_rn(y[j], s2);
      // 48 bits per 8 codes: words (lo, hi16) of four groups -> six words
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) cvt_fp6x8<FORMAT == 4>(v + 4 * g, lo[g], hi[g]);
      // group g occupies bits [48g, 48g + 48) of the 192-bit run
      cw[0] = lo[0];
      cw[1] = hi[0] | (lo[1] << 16);
      cw[2] = (lo[1] >> 16) | (hi[1] << 16);
      cw[3] = lo[2];
      cw[4] = hi[2] | (lo[3] << 16);
      cw[5] = (lo[3] >> 16) | (hi[3] << 16);
    }
    uint2 *d2 = reinterpret_cast<uint2 *>(cd);
    d2[0] = make_uint2(cw[0], cw[1]);
    d2[1] = make_uint2(cw[2], cw[3]);
    d2[2] = make_uint2(cw[4], cw[5]);
    *sd = (uint8_t)sc;
  } else if (FORMAT == 0) {
    // ---- NVFP4: the dispatch's rule on the fp32 values, two blocks of 16
    uint32_t cw[4] = {0, 0, 0, 0};
    uint32_t sq2 = 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = max_abs3(amax, y[8 * b + j].x, y[8 * b + j].y);
      const uint32_t sq = cvt_e4m3x2(__fdiv_rn(__fdiv_rn(amax, 6.0f), gs), 0.0f) & 0xFFu;
      const float d = __fmul_rn(e4m3_to_float(sq), gs);
      sq2 |= sq << (8 * b);
      if (d > 0.0f) {
        float2 q[8];
        // |y / d| <= 12.01 unless the block scale saturated at 448 (0x7E): an
        // unsaturated E4M3 scale is at least half of amax / 6
        if (sq < 0x7Eu && d >= kQuotientMinDivisor && d <= kQuotientMaxDivisor) {
          const float rd = __frcp_rn(d);
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = rn_quotient2(y[8 * b + j], d, rd);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            q[j] = make_float2(__fdiv_rn(y[8 * b + j].x, d), __fdiv_rn(y[8 * b + j].y, d));
        }
        cw[2 * b] = cvt_e2m1x8(q[0], q[1], q[2], q[3]);
        cw[2 * b + 1] = cvt_e2m1x8(q[4], q[5], q[6], q[7]);
      }
    }
    st_v4(reinterpret_cast<uint4 *>(cd), make_uint4(cw[0], cw[1], cw[2], cw[3]));
    *reinterpret_cast<uint16_t *>(sd) = (uint16_t)sq2;
  } else {
    // ---- MX: one block of 32, E8M0 scale 2^X, X = floor(log2 amax) - emax
    constexpr int kEmax = FORMAT == 1 ? 8 : 2;
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = max_abs3(amax, y[j].x, y[j].y);
    uint32_t sc = 0;
    uint32_t cw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (amax > 0.0f) {
      sc = mx_scale_code(amax, kEmax);
      // X = sc - 127 lies in [-127, 127 - kEmax], so 2^-X is a normal float
      // and y * 2^-X is one rounding
      const float2 s2 = splat(pow2i(127 - (int)sc));
      if (FORMAT == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          cw[i] = cvt_e4m3x4(__fmul2_rn(y[2 * i], s2), __fmul2_rn(y[2 * i + 1], s2));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          cw[i] = cvt_e2m1x8(__fmul2_rn(y[4 * i], s2), __fmul2_rn(y[4 * i + 1], s2),
                             __fmul2_rn(y[4 * i + 2], s2), __fmul2_rn(y[4 * i + 3], s2));
      }
    }
    st_v4(reinterpret_cast<uint4 *>(cd), make_uint4(cw[0], cw[1], cw[2], cw[3]));
    if (FORMAT == 1)
      st_v4(reinterpret_cast<uint4 *>(cd) + 1, make_uint4(cw[4], cw[5], cw[6], cw[7]));
    *sd = (uint8_t)sc;
  }
}

// One lane's NVFP4 block: the 16 columns [c, c + 16) of row r, the rule of
// the 32-column group above on one block.  Lanes 32 bytes apart (split
// gate/up) or 64 bytes apart (interleaved) instead of 64 / 128, so each
// warp-wide 16-byte load touches a quarter / half as many cache lines, while
// each block's scale work stays in one lane.
template <bool INTERLEAVED>
__device__ __forceinline__ void swiglu_nvfp4_block(const float *tab,
                                                   const uint4 *__restrict__ gate_up,
                                                   const int32_t *__restrict__ row_src, float gs,
                                                   uint8_t *__restrict__ codes,
                                                   uint8_t *__restrict__ scales, int64_t r,
                                                   int32_t c, int32_t I) {
  uint8_t *cd = codes + r * ((int64_t)I / 2) + c / 2;  // 8 bytes of codes
  uint8_t *sd = scales + r * ((int64_t)I / 16) + c / 16;
  if (__ldg(row_src + r) < 0) {  // no routed token: zero bytes, input not read
    *reinterpret_cast<uint2 *>(cd) = make_uint2(0, 0);
    *sd = 0;
    return;
  }
  const uint4 *in = gate_up + r * ((int64_t)I / 4);  // 2I bf16 = I/4 vectors of 8
  uint4 gv[2], uv[2];
  if (INTERLEAVED) {
    uint4 iv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) iv[i] = ld_stream_v4(in + c / 4 + i);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 a = iv[2 * i], b = iv[2 * i + 1];
      gv[i] = make_uint4(__byte_perm(a.x, a.y, 0x5410), __byte_perm(a.z, a.w, 0x5410),
                         __byte_perm(b.x, b.y, 0x5410), __byte_perm(b.z, b.w, 0x5410));
      uv[i] = make_uint4(__byte_perm(a.x, a.y, 0x7632), __byte_perm(a.z, a.w, 0x7632),
                         __byte_perm(b.x, b.y, 0x7632), __byte_perm(b.z, b.w, 0x7632));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      gv[i] = ld_stream_v4(in + c / 8 + i);
      uv[i] = ld_stream_v4(in + I / 8 + c / 8 + i);
    }
  }
  uint32_t check = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    check |= table_check(gv[i].x) | table_check(gv[i].y) | table_check(gv[i].z) |
             table_check(gv[i].w);
  float2 y[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t g4[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((check & kTableCheckBits) == 0) {
        uint32_t lo, hi;
        table_offsets(g4[e], lo, hi);
        y[4 * i + e] = make_float2(table_at(tab, lo), table_at(tab, hi));
      } else {
        y[4 * i + e] = silu2(make_float2(bf16lo(g4[e]), bf16hi(g4[e])));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t u4[4] = {uv[i].x, uv[i].y, uv[i].z, uv[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      y[4 * i + e] = __fmul2_rn(y[4 * i + e], make_float2(bf16lo(u4[e]), bf16hi(u4[e])));
  }
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) amax = max_abs3(amax, y[j].x, y[j].y);
  const uint32_t sq = cvt_e4m3x2(__fdiv_rn(__fdiv_rn(amax, 6.0f), gs), 0.0f) & 0xFFu;
  const float d = __fmul_rn(e4m3_to_float(sq), gs);
  uint32_t cw[2] = {0, 0};
  if (d > 0.0f) {
    float2 q[8];
    // |y / d| <= 12.01 unless the block scale saturated at 448 (0x7E)
    if (sq < 0x7Eu && d >= kQuotientMinDivisor && d <= kQuotientMaxDivisor) {
      const float rd = __frcp_rn(d);
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = rn_quotient2(y[j], d, rd);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = make_float2(__fdiv_rn(y[j].x, d), __fdiv_rn(y[j].y, d));
    }
    cw[0] = cvt_e2m1x8(q[0], q[1], q[2], q[3]);
    cw[1] = cvt_e2m1x8(q[4], q[5], q[6], q[7]);
  }
  *reinterpret_cast<uint2 *>(cd) = make_uint2(cw[0], cw[1]);
  *sd = (uint8_t)sq;
}

// One lane's half of an MXFP6 block: the 16 columns [c, c + 16) of row r;
// the block's other half is the partner lane (lane ^ 1, columns c ^ 16),
// which the dealing of column groups keeps in the same warp and row (G is
// even).  The block maximum is one xor-shuffle over the two lanes, both
// derive the same E8M0 scale; each packs its 16 six-bit codes into 12 bytes
// (bits [96 h, 96 h + 96) of the block's 24), the even lane stores the scale.
template <int FORMAT, bool INTERLEAVED>
__device__ __forceinline__ void swiglu_mxfp6_half(const float *tab,
                                                  const uint4 *__restrict__ gate_up,
                                                  const int32_t *__restrict__ row_src,
                                                  uint8_t *__restrict__ codes,
                                                  uint8_t *__restrict__ scales, int64_t r,
                                                  int32_t c, int32_t I, int lane) {
  constexpr int kEmax = FORMAT == 4 ? 2 : 4;
  const bool upper = (c & 16) != 0;
  uint32_t *cd = reinterpret_cast<uint32_t *>(codes + r * ((int64_t)I / 32 * 24) +
                                              (int64_t)(c / 32) * 24 + (upper ? 12 : 0));
  uint8_t *sd = scales + r * ((int64_t)I / 32) + c / 32;
  if (__ldg(row_src + r) < 0) {  // no routed token (the partner lane is in the same row)
    cd[0] = cd[1] = cd[2] = 0;
    if (!upper) *sd = 0;
    return;
  }
  const uint4 *in = gate_up + r * ((int64_t)I / 4);
  uint4 gv[2], uv[2];
  if (INTERLEAVED) {
    uint4 iv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) iv[i] = ld_stream_v4(in + c / 4 + i);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 a = iv[2 * i], b = iv[2 * i + 1];
      gv[i] = make_uint4(__byte_perm(a.x, a.y, 0x5410), __byte_perm(a.z, a.w, 0x5410),
                         __byte_perm(b.x, b.y, 0x5410), __byte_perm(b.z, b.w, 0x5410));
      uv[i] = make_uint4(__byte_perm(a.x, a.y, 0x7632), __byte_perm(a.z, a.w, 0x7632),
                         __byte_perm(b.x, b.y, 0x7632), __byte_perm(b.z, b.w, 0x7632));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      gv[i] = ld_stream_v4(in + c / 8 + i);
      uv[i] = ld_stream_v4(in + I / 8 + c / 8 + i);
    }
  }
  uint32_t check = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    check |= table_check(gv[i].x) | table_check(gv[i].y) | table_check(gv[i].z) |
             table_check(gv[i].w);
  float2 y[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t g4[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
    const uint32_t u4[4] = {uv[i].x, uv[i].y, uv[i].z, uv[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 sg;
      if ((check & kTableCheckBits) == 0) {
        uint32_t lo, hi;
        table_offsets(g4[e], lo, hi);
        sg = make_float2(table_at(tab, lo), table_at(tab, hi));
      } else {
        sg = silu2(make_float2(bf16lo(g4[e]), bf16hi(g4[e])));
      }
      y[4 * i + e] = __fmul2_rn(sg, make_float2(bf16lo(u4[e]), bf16hi(u4[e])));
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) amax = max_abs3(amax, y[j].x, y[j].y);
  // the two lanes of the block (same branch, same row): exactly those two
  amax = fmaxf(amax, __shfl_xor_sync(3u << (lane & 30), amax, 1));
  uint32_t sc = 0, w[3] = {0, 0, 0};
  if (amax > 0.0f) {
    sc = mx_scale_code(amax, kEmax);
    const float2 s2 = splat(pow2i(127 - (int)sc));
    float2 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __fmul2_rn(y[j], s2);
    uint32_t lo[2], hi[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) cvt_fp6x8<FORMAT == 4>(v + 4 * g, lo[g], hi[g]);
    w[0] = lo[0];
    w[1] = hi[0] | (lo[1] << 16);
    w[2] = (lo[1] >> 16) | (hi[1] << 16);
  }
  cd[0] = w[0];
  cd[1] = w[1];
  cd[2] = w[2];
  if (!upper) *sd = (uint8_t)sc;
}

// ---- split layout: coalesced warp units
// A warp takes a unit of 512 columns of one row; lane l holds the 8 columns
// [c0 + 256 s + 8 l, +8) for s = 0, 1, so every 16-byte load and every code
// store of the warp covers one contiguous run (measured on B200: the
// lane-contiguous groups above, 64 bytes apart per lane, kept the L1TEX data
// path at 91% of its peak).  A 32-column MX block spans 4 lanes: its
// maximum is a two-step xor-shuffle reduction.  Used for MXFP8, MXFP4 and
// bf16 (measured on B200, rows = 65,536, I = 3584, N(0,1) inputs: 238 -> 231,
// 217 -> 209, 298 -> 209 us); for NVFP4 and MXFP6 the per-block scale work,
// repeated by every lane of a block, made it slower than the lane-contiguous
// kernel, which they keep.
constexpr int kUnitCols = 512;

template <int FORMAT>
__device__ __forceinline__ void swiglu_unit_split(const float *tab, const uint4 *__restrict__ gate_up,
                                                  bool live, uint8_t *__restrict__ codes,
                                                  uint8_t *__restrict__ scales, int64_t r,
                                                  int32_t c0, int32_t I, int lane) {
  static_assert(FORMAT == 1 || FORMAT == 2 || FORMAT == 3, "MXFP8, MXFP4 or bf16");
  constexpr uint32_t kFull = 0xFFFFFFFFu;
  // code bytes per 8 columns
  constexpr int kCode8 = FORMAT == 1 ? 8 : FORMAT == 3 ? 16 : 4;
  const int64_t code_row = (int64_t)I / 8 * kCode8;
  const int64_t scale_row = I / 32;
  const uint4 *in = gate_up + r * ((int64_t)I / 4);  // 2I bf16 = I/4 vectors of 8

  int c[2];
  bool act[2];
  uint4 gv[2], uv[2];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    c[s] = c0 + s * (kUnitCols / 2) + 8 * lane;
    act[s] = c[s] < I;
    gv[s] = uv[s] = make_uint4(0, 0, 0, 0);
    if (live && act[s]) {
      gv[s] = ld_stream_v4(in + c[s] / 8);
      uv[s] = ld_stream_v4(in + I / 8 + c[s] / 8);
    }
  }

  // ---- y = silu(g) * u: y[4 s + e] = columns c[s] + 2e, +1
  float2 y[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) y[j] = make_float2(0.0f, 0.0f);
  if (live) {
    uint32_t check = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s)
      if (act[s])
        check |= table_check(gv[s].x) | table_check(gv[s].y) | table_check(gv[s].z) |
                 table_check(gv[s].w);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const uint32_t g4[4] = {gv[s].x, gv[s].y, gv[s].z, gv[s].w};
      const uint32_t u4[4] = {uv[s].x, uv[s].y, uv[s].z, uv[s].w};
      if ((check & kTableCheckBits) == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t lo, hi;
          table_offsets(g4[e], lo, hi);
          y[4 * s + e] = make_float2(table_at(tab, lo), table_at(tab, hi));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) y[4 * s + e] = silu2(make_float2(bf16lo(g4[e]), bf16hi(g4[e])));
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        y[4 * s + e] = __fmul2_rn(y[4 * s + e], make_float2(bf16lo(u4[e]), bf16hi(u4[e])));
    }
  }

#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const float2 *v = y + 4 * s;
    uint8_t *cd = codes + r * code_row + (int64_t)(c[s] / 8) * kCode8;
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = max_abs3(amax, v[e].x, v[e].y);
    if (FORMAT == 3) {
      // ---- bf16, rounded to nearest even
      if (act[s])
        st_v4(reinterpret_cast<uint4 *>(cd),
              make_uint4(pack_bf16x2(v[0].x, v[0].y), pack_bf16x2(v[1].x, v[1].y),
                         pack_bf16x2(v[2].x, v[2].y), pack_bf16x2(v[3].x, v[3].y)));
    } else {
      // ---- MX: 32-column blocks over lane quads, E8M0 scale 2^X
      constexpr int kEmax = FORMAT == 1 ? 8 : 2;
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
      // an all-zero block is scale 0 and codes 0 (also for -0 elements)
      const bool nz = amax > 0.0f;
      const uint32_t sc = nz ? mx_scale_code(amax, kEmax) : 0u;
      const float2 s2 = splat(pow2i(127 - (int)sc));
      float2 w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = __fmul2_rn(v[e], s2);
      if (FORMAT == 1) {
        if (act[s])
          *reinterpret_cast<uint2 *>(cd) = nz ? make_uint2(cvt_e4m3x4(w[0], w[1]),
                                                           cvt_e4m3x4(w[2], w[3]))
                                              : make_uint2(0u, 0u);
      } else {
        if (act[s])
          *reinterpret_cast<uint32_t *>(cd) = nz ? cvt_e2m1x8(w[0], w[1], w[2], w[3]) : 0u;
      }
      if (act[s] && (lane & 3) == 0) scales[r * scale_row + c[s] / 32] = (uint8_t)sc;
    }
  }
}

// Interleaved gate/up, same warp units: the unit's 512 columns are 1024
// interleaved bf16; lane l holds the 4 columns [c0 + 4 l + 128 j, +4) of
// the 16-byte vectors l + 32 j (j = 0..3), so loads and stores are again
// contiguous per warp instruction.  A 32-column MX block spans 8 lanes.
template <int FORMAT>
__device__ __forceinline__ void swiglu_unit_interleaved(const float *tab,
                                                        const uint4 *__restrict__ gate_up,
                                                        bool live, uint8_t *__restrict__ codes,
                                                        uint8_t *__restrict__ scales, int64_t r,
                                                        int32_t c0, int32_t I, int lane) {
  static_assert(FORMAT == 1 || FORMAT == 2 || FORMAT == 3, "MXFP8, MXFP4 or bf16");
  constexpr uint32_t kFull = 0xFFFFFFFFu;
  const uint4 *in = gate_up + r * ((int64_t)I / 4) + c0 / 4;  // 2I bf16 = I/4 vectors
  int c[4];
  bool act[4];
  uint4 iv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    c[j] = c0 + 4 * lane + (kUnitCols / 4) * j;
    act[j] = c[j] < I;
    iv[j] = live && act[j] ? ld_stream_v4(in + lane + 32 * j) : make_uint4(0, 0, 0, 0);
  }
  // each 32-bit word is one (gate, up) pair: gate in the low half
  float2 y[8];  // y[2j + h] = columns c[j] + 2h, +1
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = make_float2(0.0f, 0.0f);
  if (live) {
    uint32_t check = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (act[j])
        check |= table_check(iv[j].x) | table_check(iv[j].y) | table_check(iv[j].z) |
                 table_check(iv[j].w);
    const bool in_table = (check & kTableCheckBits & 0xFFFFu) == 0;  // gate halves only
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t wd[4] = {iv[j].x, iv[j].y, iv[j].z, iv[j].w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t a = wd[2 * h], b = wd[2 * h + 1];
        float2 sl;
        if (in_table) {
          uint32_t lo_a, hi_a, lo_b, hi_b;
          table_offsets(a, lo_a, hi_a);
          table_offsets(b, lo_b, hi_b);
          sl = make_float2(table_at(tab, lo_a), table_at(tab, lo_b));
        } else {
          sl = silu2(make_float2(bf16lo(a), bf16lo(b)));
        }
        y[2 * j + h] = __fmul2_rn(sl, make_float2(bf16hi(a), bf16hi(b)));
      }
    }
  }

#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 p0 = y[2 * j], p1 = y[2 * j + 1];
    if (FORMAT == 3) {
      // ---- bf16, rounded to nearest even
      if (act[j])
        *reinterpret_cast<uint2 *>(codes + r * (2 * (int64_t)I) + 2 * (int64_t)c[j]) =
            make_uint2(pack_bf16x2(p0.x, p0.y), pack_bf16x2(p1.x, p1.y));
    } else {
      // ---- MX: 32-column blocks over 8 lanes, E8M0 scale 2^X
      constexpr int kEmax = FORMAT == 1 ? 8 : 2;
      float amax = max_abs3(max_abs3(0.0f, p0.x, p0.y), p1.x, p1.y);
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
      // an all-zero block is scale 0 and codes 0 (also for -0 elements)
      const bool nz = amax > 0.0f;
      const uint32_t sc = nz ? mx_scale_code(amax, kEmax) : 0u;
      const float2 s2 = splat(pow2i(127 - (int)sc));
      const float2 w0 = __fmul2_rn(p0, s2), w1 = __fmul2_rn(p1, s2);
      if (FORMAT == 1) {
        if (act[j])
          *reinterpret_cast<uint32_t *>(codes + r * (int64_t)I + c[j]) =
              nz ? cvt_e4m3x4(w0, w1) : 0u;
      } else if (act[j]) {
        const float2 z = make_float2(0.0f, 0.0f);
        *reinterpret_cast<uint16_t *>(codes + r * ((int64_t)I / 2) + c[j] / 2) =
            nz ? (uint16_t)(cvt_e2m1x8(w0, w1, z, z) & 0xFFFFu) : (uint16_t)0;
      }
      if (act[j] && (lane & 7) == 0) scales[r * ((int64_t)I / 32) + c[j] / 32] = (uint8_t)sc;
    }
  }
}

// Persistent over warp units: warp w takes units w, w + warps, ... of the
// rows * U units (U = ceil(I / 512) per row); (row, unit) advance by
// (step_rows, step_cols) = divmod(warps, U).  The row_src test is per warp.
// MXFP8 is held to 4 resident CTAs per SM (64 registers), the others to 3
// (measured on B200: MXFP8 230 -> 217 us; MXFP4 209 -> 215 us with 4).
template <int FORMAT, bool INTERLEAVED>
__global__ void __launch_bounds__(kThreads, FORMAT == 1 ? 4 : 3)
    swiglu_split_kernel(const uint4 *__restrict__ gate_up, const int32_t *__restrict__ row_src,
                        uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, int64_t units,
                        int32_t I, int32_t U, int64_t step_rows, int32_t step_cols) {
  MOE_TRACE_CTA(MOE_TRACE_SWIGLU_SPLIT, FORMAT);
  allow_dependents();
  __shared__ float tab[kTabSize];
  for (int i = 2 * threadIdx.x; i < kTabSize; i += 2 * kThreads) {
    const float2 v = silu2(make_float2(tab_gate(i), tab_gate(i + 1)));
    tab[i] = v.x;
    tab[i + 1] = v.y;
  }
  __syncthreads();
  grid_dependency_wait();

  const int lane = threadIdx.x % kWarp;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / kWarp);
  int64_t w = (int64_t)blockIdx.x * (kThreads / kWarp) + threadIdx.x / kWarp;
  int64_t row = w / U;
  int32_t cu = (int32_t)(w - row * U);
  [[maybe_unused]] const int64_t rows = units / U;  // for the debug checks
  for (; w < units; w += warps) {
    if (!MOE_IN_RANGE(row, rows, kDbgSwigluRow)) break;
    const bool live = __ldg(row_src + row) >= 0;  // no routed token: zero bytes
    if (INTERLEAVED)
      swiglu_unit_interleaved<FORMAT>(tab, gate_up, live, codes, scales, row, cu * kUnitCols, I,
                                      lane);
    else
      swiglu_unit_split<FORMAT>(tab, gate_up, live, codes, scales, row, cu * kUnitCols, I, lane);
    row += step_rows;
    cu += step_cols;
    if (cu >= U) {
      cu -= U;
      ++row;
    }
  }
}

// Persistent: thread t of the grid takes groups t, t + stride, ... of the
// rows * G groups (G = I / 32 per row); (row, group) advance by
// (step_rows, step_cols) = divmod(stride, G).
template <int FORMAT, bool INTERLEAVED, int COLS>
__global__ void __launch_bounds__(kThreads, 3)
    swiglu_quant_kernel(const uint4 *__restrict__ gate_up, const int32_t *__restrict__ row_src,
                        const float *__restrict__ global_scale, uint8_t *__restrict__ codes,
                        uint8_t *__restrict__ scales, int64_t groups, int32_t I, int32_t G,
                        int64_t step_rows, int32_t step_cols) {
  MOE_TRACE_CTA(MOE_TRACE_SWIGLU_QUANT, FORMAT);
  allow_dependents();
  __shared__ float tab[kTabSize];
  // the table needs no global memory: it is built while the previous kernel
  // on the stream may still be running
  for (int i = 2 * threadIdx.x; i < kTabSize; i += 2 * kThreads) {
    const float2 v = silu2(make_float2(tab_gate(i), tab_gate(i + 1)));
    tab[i] = v.x;
    tab[i + 1] = v.y;
  }
  __syncthreads();
  grid_dependency_wait();

  const float gs = FORMAT == 0 ? __ldg(global_scale) : 0.0f;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t t = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  int64_t row = t / G;
  int32_t cg = (int32_t)(t - row * G);
  [[maybe_unused]] const int64_t rows = groups / G;  // for the debug checks
  for (; t < groups; t += stride) {
    if (!MOE_IN_RANGE(row, rows, kDbgSwigluRow)) break;
    if constexpr (COLS == 16 && FORMAT == 0)
      swiglu_nvfp4_block<INTERLEAVED>(tab, gate_up, row_src, gs, codes, scales, row, cg * 16, I);
    else if constexpr (COLS == 16)
      swiglu_mxfp6_half<FORMAT, INTERLEAVED>(tab, gate_up, row_src, codes, scales, row, cg * 16,
                                             I, threadIdx.x % kWarp);
    else
      swiglu_group<FORMAT, INTERLEAVED>(tab, gate_up, row_src, gs, codes, scales, row,
                                        cg * kGroupCols, I);
    row += step_rows;
    cg += step_cols;
    if (cg >= G) {
      cg -= G;
      ++row;
    }
  }
}

template <int FORMAT, bool INTERLEAVED>
cudaError_t launch_split(const uint4 *in, const int32_t *row_src, uint8_t *codes,
                         uint8_t *scales, int64_t rows, int32_t I, cudaStream_t stream) {
  auto kernel = swiglu_split_kernel<FORMAT, INTERLEAVED>;
  static OccupancyCache occupancy;
  const int cap = resident_ctas(occupancy, reinterpret_cast<const void *>(kernel), kThreads, 0);
  const int32_t U = (I + kUnitCols - 1) / kUnitCols;
  const int64_t units = rows * U;
  const int64_t per_block = kThreads / kWarp;
  const int64_t want = (units + per_block - 1) / per_block;
  const int64_t blocks = std::max<int64_t>(
      1, std::min<int64_t>(want, (int64_t)cap * device_sm_count()));
  const int64_t warps = blocks * per_block;
  return launch_pdl(kernel, dim3((unsigned)blocks), dim3(kThreads), 0, stream, in, row_src,
                    codes, scales, units, I, U, warps / U, (int32_t)(warps % U));
}

template <int FORMAT, bool INTERLEAVED>
cudaError_t launch(const uint4 *in, const int32_t *row_src, const float *gs, uint8_t *codes,
                   uint8_t *scales, int64_t rows, int32_t I, cudaStream_t stream) {
  if (FORMAT == 1 || FORMAT == 2 || FORMAT == 3)
    return launch_split<(FORMAT == 1 || FORMAT == 2) ? FORMAT : 3, INTERLEAVED>(
        in, row_src, codes, scales, rows, I, stream);
  // NVFP4: one 16-column block per lane; MXFP6: half of a 32-column MX
  // block per lane (the other half in the neighbouring lane)
  constexpr int kCols = (FORMAT == 0 || FORMAT >= 4) ? 16 : kGroupCols;
  auto kernel = swiglu_quant_kernel<FORMAT, INTERLEAVED, kCols>;
  static OccupancyCache occupancy;
  const int cap = resident_ctas(occupancy, reinterpret_cast<const void *>(kernel), kThreads, 0);
  const int32_t G = I / kCols;
  const int64_t groups = rows * G;
  const int64_t want = (groups + kThreads - 1) / kThreads;
  const int64_t blocks = std::max<int64_t>(
      1, std::min<int64_t>(want, (int64_t)cap * device_sm_count()));
  const int64_t stride = blocks * kThreads;
  return launch_pdl(kernel, dim3((unsigned)blocks), dim3(kThreads), 0, stream, in, row_src, gs,
                    codes, scales, groups, I, G, stride / G, (int32_t)(stride % G));
}

}  // namespace

uint32_t debug_violations_swiglu(bool reset) { return read_debug_violations(reset); }

#ifdef MOE_TRACE
cudaError_t trace_attach_swiglu(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                              cudaStream_t stream) {
  return trace_attach_tu(records, count, capacity, stream);
}
#endif

cudaError_t launch_swiglu_quant(const Shape &s, int32_t I, uint32_t format, bool interleaved,
                                const void *gate_up, const int32_t *row_src,
                                const float *global_scale, uint8_t *codes, uint8_t *scales,
                                cudaStream_t stream) {
  if (s.rows == 0) return cudaSuccess;
  const uint4 *in = static_cast<const uint4 *>(gate_up);
#define MOE_SWIGLU_CASE(F)                                                                 \
  case 2 * F:                                                                              \
    return launch<F, false>(in, row_src, global_scale, codes, scales, s.rows, I, stream);   \
  case 2 * F + 1:                                                                          \
    return launch<F, true>(in, row_src, global_scale, codes, scales, s.rows, I, stream);
  switch (format * 2 + (interleaved ? 1 : 0)) {
    MOE_SWIGLU_CASE(0)
    MOE_SWIGLU_CASE(1)
    MOE_SWIGLU_CASE(2)
    MOE_SWIGLU_CASE(3)
    MOE_SWIGLU_CASE(4)
    MOE_SWIGLU_CASE(5)
    default:
      return cudaErrorInvalidValue;
  }
#undef MOE_SWIGLU_CASE
}

}  // namespace moe
