// cvt_check.cu -- test-only harness (built by tests/test_gpu_cvt_exhaustive.py,
// never linked into libmoedc.so): runs the library's own conversion and
// quotient helpers from csrc/common.cuh over caller-given inputs so that the
// test can compare every result with the CPU oracle.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace {

// Codes of the fp32 bit patterns start + i, i in [0, n), one byte each:
// E4M3 through cvt_e4m3x4 (four patterns per thread).
__global__ void e4m3_patterns_kernel(uint32_t start, int64_t n, uint32_t *out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 4 patterns
  if (i * 4 >= n) return;
  const uint32_t b = start + (uint32_t)(i * 4);
  const float2 lo = make_float2(__uint_as_float(b), __uint_as_float(b + 1));
  const float2 hi = make_float2(__uint_as_float(b + 2), __uint_as_float(b + 3));
  out[i] = moe::cvt_e4m3x4(lo, hi);
}

// E2M1 through cvt_e2m1x8 (eight patterns per thread, one nibble each,
// written out as eight bytes).
__global__ void e2m1_patterns_kernel(uint32_t start, int64_t n, uint2 *out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 8 patterns
  if (i * 8 >= n) return;
  const uint32_t b = start + (uint32_t)(i * 8);
  float2 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    v[j] = make_float2(__uint_as_float(b + 2 * j), __uint_as_float(b + 2 * j + 1));
  const uint32_t c = moe::cvt_e2m1x8(v[0], v[1], v[2], v[3]);
  uint32_t w[2] = {0, 0};
#pragma unroll
  for (int j = 0; j < 8; ++j) w[j / 4] |= ((c >> (4 * j)) & 0xFu) << (8 * (j % 4));
  out[i] = make_uint2(w[0], w[1]);
}

// q = rn_quotient2 of (a[2i], a[2i+1]) by d[i] with rd = RN(1/d[i]).
__global__ void quotient_kernel(const float *a, const float *d, float *q, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float dv = d[i];
  const float2 r = moe::rn_quotient2(make_float2(a[2 * i], a[2 * i + 1]), dv, __frcp_rn(dv));
  q[2 * i] = r.x;
  q[2 * i + 1] = r.y;
}

}  // namespace

extern "C" {

// n must be a multiple of 4 (E4M3) or 8 (E2M1); out holds n bytes.
int cvt_check_e4m3(uint32_t start, int64_t n, void *out, cudaStream_t stream) {
  const int64_t threads = n / 4;
  e4m3_patterns_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(
      start, n, static_cast<uint32_t *>(out));
  return (int)cudaGetLastError();
}

int cvt_check_e2m1(uint32_t start, int64_t n, void *out, cudaStream_t stream) {
  const int64_t threads = n / 8;
  e2m1_patterns_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(
      start, n, static_cast<uint2 *>(out));
  return (int)cudaGetLastError();
}

// a: 2n floats, d: n floats, q: 2n floats
int cvt_check_quotient(const float *a, const float *d, float *q, int64_t n,
                       cudaStream_t stream) {
  quotient_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(a, d, q, n);
  return (int)cudaGetLastError();
}

}  // extern "C"
