// common.cuh -- device helpers shared by the libmoedc kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- debug build
// Built with -DMOE_DEBUG_CHECKS (libmoedc_debug.so), the kernels check every
// computed row index and scale offset before they use it: an index outside
// its buffer ORs the check's bit into this translation unit's debug word and
// the access is skipped (no trap: the context stays usable), and
// moe_debug_violations() reports the bits.  In normal builds the checks
// compile to nothing.
enum : uint32_t {
  kDbgLayoutRow = 1u,    // a pair's row in the layout's row_src
  kDbgPermuteRow = 2u,   // a permute's destination row
  kDbgScaleOffset = 4u,  // a block-scale byte in the atom layout
  kDbgCombineRow = 8u,   // a combine / backward source row
  kDbgSwigluRow = 16u,   // a SwiGLU row
};
#ifdef MOE_DEBUG_CHECKS
static __device__ uint32_t g_debug_violations;  // one per translation unit
__device__ __forceinline__ bool debug_in_range(int64_t i, int64_t n, uint32_t bit) {
  if (i >= 0 && i < n) return true;
  atomicOr(&g_debug_violations, bit);
  return false;
}
// This translation unit's debug word (and zero it when `reset`); host only.
static inline uint32_t read_debug_violations(bool reset) {
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_debug_violations, sizeof(v)) != cudaSuccess) return ~0u;
  if (reset) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_debug_violations, &zero, sizeof(zero)) != cudaSuccess) return ~0u;
  }
  return v;
}
#define MOE_IN_RANGE(i, n, bit) ::moe::debug_in_range((int64_t)(i), (int64_t)(n), (bit))
#else
static inline uint32_t read_debug_violations(bool) { return 0u; }
#define MOE_IN_RANGE(i, n, bit) true
#endif

// Programmatic dependent launch (sm_90 and later).  The library's kernels
// after the first of a step are launched with programmatic stream
// serialisation allowed (launch_pdl in internal.h), so their CTAs may be
// scheduled while the previous kernel on the stream drains its last wave.
// Each kernel executes grid_dependency_wait() before its first global
// memory access: it returns once the previous kernel has completed and its
// writes are visible, so stream order is kept for every load and store.
// allow_dependents() lets the next kernel be scheduled once every CTA of
// this one has started.  Both are no-ops for a kernel launched normally.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- memory
// 4-byte store whose L2 line is kept in preference to others (evict_last):
// the block-scale atom layout scatters 4-byte groups of different tokens
// into the same 32-byte sectors, and keeping those lines resident until
// they are complete saves partial-sector write-backs (measured on B200,
// NVFP4 dispatch with 128-padded experts: 158 -> 129 us).
__device__ __forceinline__ void st_u32_evict_last(void *p, uint32_t v) {
  asm volatile(
      "{\n\t.reg .b64 pol;\n\tcreatepolicy.fractional.L2::evict_last.b64 pol, 1.0;\n\t"
      "st.global.L2::cache_hint.b32 [%0], %1, pol;\n\t}" ::"l"(p),
      "r"(v)
      : "memory");
}

// Streaming 16-byte load that bypasses L1 (data is read once).
__device__ __forceinline__ uint4 ld_stream_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16-byte store.
__device__ __forceinline__ void st_v4(uint4 *p, const uint4 &v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint64_t ld_relaxed_gpu_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu_u64(uint64_t *p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---------------------------------------------------------------- formats
// bf16 pair (packed in a uint32, element 0 in the low half) -> two floats.
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two floats -> bf16 pair, round to nearest even; `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Two floats -> two E4M3 codes (round to nearest even, saturating to +-448);
// `lo` lands in bits 0-7, `hi` in bits 8-15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// floor(log2(a)) of a finite a > 0, subnormals included.
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = (int)((b >> 23) & 0xFFu);
  if (e != 0) return e - 127;
  return (31 - __clz((int)(b & 0x7FFFFFu))) - 149;
}

// 2^n as a float for n in [-126, 127].
__device__ __forceinline__ float pow2i(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }

// E8M0 code of the OCP MX shared scale of a block with largest magnitude
// amax > 0 (finite): X = floor(log2(amax)) - emax, code clamp(X + 127, 0, 254).
// For every emax >= 2 used here, 2^(127 - code) is a normal float, so the
// element scaling y * 2^-X is a single multiply.
__device__ __forceinline__ uint32_t mx_scale_code(float amax, int emax) {
  return (uint32_t)min(254, max(0, floor_log2(amax) - emax + 127));
}

// max(a, |b|, |c|) in one three-input maximum
__device__ __forceinline__ float max_abs3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
  return r;
}

// Eight floats -> eight E2M1 codes (nearest even, saturating to +-6), the
// first in bits 0-3.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t r;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
  return r;
}

// Four floats -> four E4M3 codes (nearest even, saturating to +-448), the
// first in bits 0-7.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float2 a, float2 b) {
  uint32_t r;
  asm("{\n\t.reg .b16 t0, t1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t1, %4, %3;\n\t"
      "mov.b32 %0, {t0, t1};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// RN(a / d) of both halves from rd = RN(1/d), by two steps of Markstein's
// correction q + (a - d q) * rd (P. Markstein, Computation of elementary
// functions on the IBM RISC System/6000 processor, IBM J. Res. Dev. 34(1),
// 1990: if rd is within half an ulp of 1/d and q within one ulp of a/d, the
// corrected q rounds correctly).  q0 = RN(a rd) is within two ulps of a/d,
// the first step brings it within one, the second rounds correctly.  The
// caller guarantees d in [2^-90, 2^124] (kQuotientMinDivisor,
// kQuotientMaxDivisor) and |a / d| <= 2^24.  Then every remainder is exact
// (no underflow) for quotients >= 2^-13 and the result is RN(a / d); a
// smaller quotient comes out below 2^-12 in magnitude with the sign of a,
// which every 8- and 4-bit code here rounds to the same signed zero.  A zero
// quotient takes the sign of a, as IEEE division does.
constexpr float kQuotientMinDivisor = 0x1p-90f;
constexpr float kQuotientMaxDivisor = 0x1p124f;
__device__ __forceinline__ float2 rn_quotient2(float2 a, float d, float rd) {
  const float2 nd = make_float2(-d, -d), r2 = make_float2(rd, rd);
  float2 q = __fmul2_rn(a, r2);
  q = __ffma2_rn(__ffma2_rn(nd, q, a), r2, q);
  q = __ffma2_rn(__ffma2_rn(nd, q, a), r2, q);
  return make_float2(copysignf(q.x, a.x), copysignf(q.y, a.y));
}

// One E4M3 code -> float (exact): through the f16x2 conversion.
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  uint32_t h2;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
      : "=r"(h2)
      : "r"(code & 0xFFu));
  __half_raw hr;
  hr.x = (unsigned short)(h2 & 0xFFFFu);
  return __half2float(__half(hr));
}

}  // namespace moe
