/*
 * oracle.c -- CPU oracle for MoE dispatch layout, permute (bf16 / block FP8
 * / NVFP4) and combine.  TEST INFRASTRUCTURE ONLY: see oracle.h for who may
 * call it and for the sources each part follows.
 *
 * Written as the plain definitions: one sequential pass over the pairs in
 * ascending (token, k) order, one output row at a time, one block at a
 * time.  No tiling, no reordering, no shared tables with the GPU path.
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math (IEEE binary32 with
 * round-to-nearest-even; fused multiply-add only where fmaf is written).
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

static uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

static float f32_from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* bfloat16 keeps the sign, the 8 exponent bits and the top 7 fraction bits
 * of binary32.  Rounding to nearest, ties to even, on the dropped 16 bits:
 * add 0x7FFF plus the lowest kept bit, then truncate.  A carry out of the
 * fraction increments the exponent, which is the correct rounding (and
 * yields infinity past the largest finite value).  NaN stays a quiet NaN. */
uint16_t orc_bf16_from_f32(float f) {
  uint32_t u = f32_bits(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
    return (uint16_t)((u >> 16) | 0x0040u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* Round a non-negative double that holds an exact value to the nearest
 * integer, ties to even (rint under the default rounding mode). */
static double rne_int(double v) { return rint(v); }

/* OCP 8-bit FP, E4M3 ("fn": no infinities; S.1111.111 is NaN).
 * Exponent bias 7.  Normal: (1 + m/8) * 2^(e-7), e in 1..15, with
 * (e,m) = (15,7) reserved for NaN, so the largest finite value is
 * 1.75 * 2^8 = 448.  Subnormal (e = 0): m/8 * 2^-6 = m * 2^-9.
 * Conversion: round to nearest, ties to even code; magnitudes beyond 448
 * saturate to 448 (the satfinite rule).  Sign is kept, also for zero. */
uint8_t orc_e4m3_from_f32(float f) {
  uint8_t sign = signbit(f) ? 0x80 : 0x00;
  if (isnan(f)) return (uint8_t)(sign | 0x7F);
  double a = fabs((double)f);
  if (a > 448.0) return (uint8_t)(sign | 0x7E);
  uint32_t code;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: integer multiples of 2^-9; 8 * 2^-9 is the
     * smallest normal and gets code 8 = (e=1, m=0) automatically */
    code = (uint32_t)rne_int(a * 512.0);
  } else {
    int e2;
    double fr = frexp(a, &e2); /* a = fr * 2^e2, fr in [0.5, 1) */
    int e = e2 - 1;            /* a = (2*fr) * 2^e, 2*fr in [1, 2) */
    double m = rne_int((2.0 * fr - 1.0) * 8.0);
    if (m >= 8.0) {
      m = 0.0;
      e += 1;
    }
    code = (uint32_t)(((e + 7) << 3) | (int)m);
    if (code > 0x7E) code = 0x7E;
  }
  return (uint8_t)(sign | code);
}

float orc_e4m3_to_f32(uint8_t c) {
  int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return (float)(s ? -v : v);
}

/* OCP MX E2M1: exponent bias 1.  Normal: (1 + m/2) * 2^(e-1), e in 1..3;
 * subnormal (e = 0): m * 0.5.  Values {0, .5, 1, 1.5, 2, 3, 4, 6}; no inf
 * or NaN.  Round to nearest, ties to even code; saturate beyond 6. */
uint8_t orc_e2m1_from_f32(float f) {
  uint8_t sign = signbit(f) ? 0x8 : 0x0;
  if (isnan(f)) return (uint8_t)(sign | 0x7);
  double a = fabs((double)f);
  if (a > 6.0) return (uint8_t)(sign | 0x7);
  uint32_t code;
  if (a < 1.0) {
    code = (uint32_t)rne_int(a * 2.0); /* 0, 1 (=0.5) or 2 (=1.0) */
  } else {
    int e2;
    double fr = frexp(a, &e2);
    int e = e2 - 1;
    double m = rne_int((2.0 * fr - 1.0) * 2.0);
    if (m >= 2.0) {
      m = 0.0;
      e += 1;
    }
    code = (uint32_t)(((e + 1) << 1) | (int)m);
    if (code > 0x7) code = 0x7;
  }
  return (uint8_t)(sign | code);
}

float orc_e2m1_to_f32(uint8_t c) {
  int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double v = (e == 0) ? 0.5 * m : ldexp(1.0 + m / 2.0, e - 1);
  return (float)(s ? -v : v);
}

/* OCP MX v1.0 FP6 element formats, no infinities or NaN:
 *   E2M3: exponent bias 1; normal (1 + m/8) * 2^(e-1), e in 1..3; subnormal
 *         m/8; largest 7.5.
 *   E3M2: exponent bias 3; normal (1 + m/4) * 2^(e-3), e in 1..7; subnormal
 *         m/16; largest 28.
 * Code layout: sign in bit 5, then the exponent, then the mantissa.        */
static double fp6_magnitude(int code, int ebits) {
  const int mbits = 5 - ebits, bias = ebits == 2 ? 1 : 3;
  const int e = code >> mbits, m = code & ((1 << mbits) - 1);
  if (e == 0) return ldexp((double)m, 1 - bias - mbits);
  return ldexp(1.0 + (double)m / (double)(1 << mbits), e - bias);
}

/* Round to the nearest of the 32 magnitudes (searched one by one), ties to
 * the even code, anything above the largest to the largest (saturation);
 * the sign is kept, NaN maps to the signed largest value. */
static uint8_t fp6_from_f32(float f, int ebits) {
  const uint8_t sign = signbit(f) ? 0x20 : 0x00;
  if (isnan(f)) return (uint8_t)(sign | 0x1F);
  const double a = fabs((double)f);
  if (a >= fp6_magnitude(31, ebits)) return (uint8_t)(sign | 31); /* saturate */
  int best = 0;
  for (int c = 1; c < 32; ++c) {
    const double dc = fabs(a - fp6_magnitude(c, ebits));
    const double db = fabs(a - fp6_magnitude(best, ebits));
    if (dc < db || (dc == db && (c & 1) == 0)) best = c;
  }
  return (uint8_t)(sign | best);
}

uint8_t orc_e2m3_from_f32(float f) { return fp6_from_f32(f, 2); }
uint8_t orc_e3m2_from_f32(float f) { return fp6_from_f32(f, 3); }
float orc_e2m3_to_f32(uint8_t c) {
  const double v = fp6_magnitude(c & 0x1F, 2);
  return (float)((c & 0x20) ? -v : v);
}
float orc_e3m2_to_f32(uint8_t c) {
  const double v = fp6_magnitude(c & 0x1F, 3);
  return (float)((c & 0x20) ? -v : v);
}
void orc_e2m3_from_f32_n(const float *in, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m3_from_f32(in[i]);
}
void orc_e3m2_from_f32_n(const float *in, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e3m2_from_f32(in[i]);
}

/* Four 6-bit codes in three bytes: code i at bits [6i, 6i + 6) of the
 * little-endian 24-bit group. */
void orc_pack_fp6(const uint8_t *codes, int64_t n, uint8_t *out) {
  for (int64_t g = 0; g < n / 4; ++g) {
    uint32_t w = 0;
    for (int i = 0; i < 4; ++i) w |= (uint32_t)(codes[4 * g + i] & 0x3F) << (6 * i);
    out[3 * g] = (uint8_t)(w & 0xFF);
    out[3 * g + 1] = (uint8_t)((w >> 8) & 0xFF);
    out[3 * g + 2] = (uint8_t)((w >> 16) & 0xFF);
  }
}

void orc_bf16_from_f32_n(const float *in, uint16_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_f32(in[i]);
}
void orc_e4m3_from_f32_n(const float *in, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_f32(in[i]);
}
void orc_e2m1_from_f32_n(const float *in, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_from_f32(in[i]);
}

/* ------------------------------------------------------------------ */
/* Dispatch layout                                                     */
/* ------------------------------------------------------------------ */

/* Counting sort of the routed pairs by expert, stable in pair order.
 *
 * A pair p = t*k + j routes token t to expert ids[p].  Id -1 means the
 * pair is masked out (NeMo token_dispatcher, _indices_to_multihot and
 * _HybridEPMetadataProcessor.forward: invalid slots contain -1); any other
 * id outside [0, E) is reported and treated as masked.
 *
 * Packed (dropless) mode, NKI permute_a2av: rows are packed expert-major
 * (hence destination-segment-major, since segment s holds experts
 * [s*L, (s+1)*L)); expert e's rows start at the exclusive cumulative sum of
 * the counts; within an expert, rows follow ascending pair index.  Rows
 * [total, C) are padding.  A pair whose row would be >= C gets no row
 * (status CAPACITY); the counts stay the true counts.
 *
 * Capacity mode, DeepSpeed capacity dispatch ([e, c, m] buffer) with the
 * capacity of NeMo's moe_expert_capacity_factor: the r-th pair routed to
 * expert e (in ascending pair order) takes row e*Ce + r when r < Ce and is
 * dropped otherwise.
 *
 * Per-expert padding (NeMo moe_router_expert_pad_multiple, packed mode):
 * expert e's block of rows is its count rounded up to a multiple of pad, so
 * every expert starts at a multiple of pad; the rows past the count are
 * padding like the rows past the total.
 *
 * send_counts / send_displs / recv_counts / recv_displs (NKI [4, EP]
 * uint32 metadata, in elements): per destination segment its rows times H
 * -- the expert blocks, per-expert padding included, in packed mode; the
 * kept rows in capacity mode -- and where they start: the exclusive
 * cumulative sum (packed) or the static segment start s*L*Ce*H (capacity).
 * On one device the receive rows equal the send rows. */
uint32_t orc_layout(int32_t N, int32_t k, int32_t E, int32_t S, int64_t C,
                    int32_t Ce, int32_t pad, uint32_t flags, int32_t H,
                    const int32_t *ids, int32_t *expert_counts,
                    int32_t *expert_offsets, uint32_t *meta, int32_t *row_src,
                    int32_t *pair_slot, uint8_t *drop_mask) {
  uint32_t status = 0;
  const int64_t P = (int64_t)N * k;
  const int capacity_mode = Ce > 0;
  const int64_t rows = capacity_mode ? (int64_t)E * Ce : C;
  const int32_t L = E / S;

  int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
  int64_t *seen = (int64_t *)calloc((size_t)E, sizeof(int64_t));
  int64_t *off = (int64_t *)calloc((size_t)E + 1, sizeof(int64_t));

  /* 1. count the routed pairs per expert (tokens per expert, NeMo
   *    get_number_of_tokens_per_expert) */
  for (int64_t p = 0; p < P; ++p) {
    int32_t e = ids[p];
    if (e == -1) continue;
    if (e < 0 || e >= E) {
      status |= ORC_STATUS_ID_RANGE;
      continue;
    }
    cnt[e] += 1;
  }

  /* optional: a token naming one expert twice (NKI recv_capacity note:
   * duplicates invalidate the dropless bound) */
  if (flags & ORC_FLAG_CHECK_DUPLICATES) {
    for (int32_t t = 0; t < N; ++t)
      for (int32_t a = 0; a < k; ++a)
        for (int32_t b = a + 1; b < k; ++b) {
          int32_t ea = ids[(int64_t)t * k + a], eb = ids[(int64_t)t * k + b];
          if (ea >= 0 && ea < E && ea == eb) status |= ORC_STATUS_DUP_ID;
        }
  }

  /* 2. expert start rows: exclusive cumulative sum of the (padded) counts
   *    (packed) or e*Ce */
  for (int32_t e = 0; e < E; ++e) {
    int64_t block = cnt[e];
    if (!capacity_mode && pad > 1) block = (cnt[e] + pad - 1) / pad * pad;
    off[e + 1] = off[e] + (capacity_mode ? (int64_t)Ce : block);
  }
  for (int32_t e = 0; e <= E; ++e) expert_offsets[e] = (int32_t)off[e];
  for (int32_t e = 0; e < E; ++e)
    expert_counts[e] = (int32_t)(capacity_mode && cnt[e] > Ce ? Ce : cnt[e]);

  /* 3. every row starts as padding (source -1) */
  for (int64_t r = 0; r < rows; ++r) row_src[r] = -1;

  /* 4. place the pairs in ascending pair order */
  for (int64_t p = 0; p < P; ++p) {
    int32_t e = ids[p];
    int32_t slot = -1;
    int dropped = 0;
    if (e >= 0 && e < E) {
      int64_t r = seen[e]++;
      int64_t row;
      if (capacity_mode) {
        row = (r < Ce) ? (int64_t)e * Ce + r : -1;
      } else {
        row = off[e] + r;
        if (row >= C) {
          row = -1;
          status |= ORC_STATUS_CAPACITY;
        }
      }
      if (row >= 0) {
        slot = (int32_t)row;
        row_src[row] = (int32_t)(p / k);
      } else {
        dropped = 1;
      }
    }
    pair_slot[p] = slot;
    if (drop_mask) drop_mask[p] = (uint8_t)dropped;
  }

  /* 5. [4, S] uint32 metadata in elements (rows * H): per segment its rows
   *    (the kept rows in capacity mode; the expert blocks, padding included,
   *    in packed mode) and where they start */
  for (int32_t s = 0; s < S; ++s) {
    int64_t seg_rows = 0, start;
    if (capacity_mode) {
      for (int32_t e = s * L; e < (s + 1) * L; ++e) seg_rows += expert_counts[e];
      start = (int64_t)s * L * Ce;
    } else {
      seg_rows = off[(s + 1) * L] - off[s * L];
      start = off[s * L];
    }
    uint32_t count_el = (uint32_t)(seg_rows * H);
    uint32_t displ_el = (uint32_t)(start * H);
    meta[0 * S + s] = count_el;
    meta[1 * S + s] = displ_el;
    meta[2 * S + s] = count_el;
    meta[3 * S + s] = displ_el;
  }

  free(cnt);
  free(seen);
  free(off);
  return status;
}

/* ------------------------------------------------------------------ */
/* Permute                                                             */
/* ------------------------------------------------------------------ */

/* NKI permute_a2av return value: [C, H] rows, packed, followed by
 * deterministic zero padding.  Mojo ep_comm BF16TokenFormat: the full row
 * in bfloat16.  Row r is hidden row row_src[r]; a padding row is zeros. */
void orc_permute_bf16(int64_t rows, int32_t H, const uint16_t *hidden,
                      const int32_t *row_src, uint16_t *out) {
  for (int64_t r = 0; r < rows; ++r) {
    uint16_t *dst = out + r * H;
    int32_t t = row_src[r];
    if (t < 0) {
      for (int32_t h = 0; h < H; ++h) dst[h] = 0;
    } else {
      const uint16_t *src = hidden + (int64_t)t * H;
      for (int32_t h = 0; h < H; ++h) dst[h] = src[h];
    }
  }
}

/* Mojo ep_comm BlockwiseFP8TokenFormat: FP8 with block-wise scales.  Each
 * 1x128 block of a row gets one fp32 scale = amax / 448 (the decode
 * multiplier: x ~ q * scale); every element is x / scale rounded to E4M3
 * (nearest even, saturating).  A block whose amax is 0 gets scale 0 and
 * zero codes.  Padding rows: zero codes and zero scales. */
void orc_permute_fp8(int64_t rows, int32_t H, const uint16_t *hidden,
                     const int32_t *row_src, uint8_t *q, float *scales) {
  const int32_t nb = H / 128;
  for (int64_t r = 0; r < rows; ++r) {
    int32_t t = row_src[r];
    for (int32_t b = 0; b < nb; ++b) {
      uint8_t *qd = q + r * H + (int64_t)b * 128;
      float *sd = scales + r * nb + b;
      if (t < 0) {
        memset(qd, 0, 128);
        *sd = 0.0f;
        continue;
      }
      const uint16_t *src = hidden + (int64_t)t * H + (int64_t)b * 128;
      float amax = 0.0f;
      for (int32_t i = 0; i < 128; ++i) {
        float a = fabsf(orc_bf16_to_f32(src[i]));
        if (a > amax) amax = a;
      }
      if (amax == 0.0f) {
        memset(qd, 0, 128);
        *sd = 0.0f;
        continue;
      }
      float sc = amax / 448.0f;
      *sd = sc;
      for (int32_t i = 0; i < 128; ++i)
        qd[i] = orc_e4m3_from_f32(orc_bf16_to_f32(src[i]) / sc);
    }
  }
}

/* Mojo ep_comm NVBlockScaledTokenFormat and the
 * ep.dispatch_async.block.scaled.nv op (global input scales supplied by the
 * caller): E2M1 codes, one E4M3 scale per 16 elements, one fp32 global
 * scale gs per tensor.  Per block: amax; block scale code
 * sq = e4m3((amax / 6) / gs); decode scale d = float(sq) * gs; each
 * element is x / d rounded to E2M1 (nearest even, saturating), or 0 when
 * d == 0.  Two codes per byte, element 2m in the low nibble of byte m.
 * Scales are stored row-major [rows, H/16].  Padding rows are all zero. */
void orc_permute_nvfp4(int64_t rows, int32_t H, const uint16_t *hidden,
                       const int32_t *row_src, float global_scale,
                       uint8_t *q, uint8_t *scales) {
  const int32_t nb = H / 16;
  for (int64_t r = 0; r < rows; ++r) {
    int32_t t = row_src[r];
    for (int32_t b = 0; b < nb; ++b) {
      uint8_t *qd = q + r * (H / 2) + (int64_t)b * 8;
      uint8_t *sd = scales + r * nb + b;
      if (t < 0) {
        memset(qd, 0, 8);
        *sd = 0;
        continue;
      }
      const uint16_t *src = hidden + (int64_t)t * H + (int64_t)b * 16;
      float amax = 0.0f;
      for (int32_t i = 0; i < 16; ++i) {
        float a = fabsf(orc_bf16_to_f32(src[i]));
        if (a > amax) amax = a;
      }
      uint8_t sq = orc_e4m3_from_f32((amax / 6.0f) / global_scale);
      float d = orc_e4m3_to_f32(sq) * global_scale;
      *sd = sq;
      for (int32_t m = 0; m < 8; ++m) {
        uint8_t lo = 0, hi = 0;
        if (d > 0.0f) {
          lo = orc_e2m1_from_f32(orc_bf16_to_f32(src[2 * m]) / d);
          hi = orc_e2m1_from_f32(orc_bf16_to_f32(src[2 * m + 1]) / d);
        }
        qd[m] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

/* E8M0 code of the OCP MX shared scale of a block with largest magnitude
 * amax > 0 (finite): X = floor(log2(amax)) - emax_elem, code = X + 127
 * clamped to [0, 254]. */
static uint8_t mx_scale_code(float amax, int32_t emax) {
  int e;
  frexpf(amax, &e); /* amax = f * 2^e, f in [0.5, 1) */
  int32_t c = (e - 1) - emax + 127;
  if (c < 0) c = 0;
  if (c > 254) c = 254;
  return (uint8_t)c;
}

/* y * 2^(127 - code): the MX scaling of an element (one rounding).  The
 * codes of mx_scale_code are at most 252 (floor(log2 amax) <= 127 for a
 * float, emax >= 2), so 2^(127 - code) is a normal float: biased exponent
 * 254 - code in [2, 254]. */
static float mx_scale_down(float y, uint8_t code) {
  return y * f32_from_bits((uint32_t)(254 - code) << 23);
}

/* Mojo MAX ep_comm MXTokenFormat (MX FP4 token format): OCP MX v1.0 MXFP4,
 * blocks of 32 along H, E2M1 codes two per byte (element 2m in the low
 * nibble of byte m), one E8M0 scale per block: X = floor(log2(amax)) - 2,
 * code = E2M1 of x * 2^-X (nearest even, saturating); an all-zero block
 * has scale code 0 and codes 0.  Scales row-major [rows, H/32].  Padding
 * rows are all zero. */
void orc_permute_mxfp4(int64_t rows, int32_t H, const uint16_t *hidden,
                       const int32_t *row_src, uint8_t *q, uint8_t *scales) {
  const int32_t nb = H / 32;
  for (int64_t r = 0; r < rows; ++r) {
    int32_t t = row_src[r];
    for (int32_t b = 0; b < nb; ++b) {
      uint8_t *qd = q + r * (H / 2) + (int64_t)b * 16;
      uint8_t *sd = scales + r * nb + b;
      memset(qd, 0, 16);
      *sd = 0;
      if (t < 0) continue;
      const uint16_t *src = hidden + (int64_t)t * H + (int64_t)b * 32;
      float amax = 0.0f;
      for (int32_t i = 0; i < 32; ++i) {
        float a = fabsf(orc_bf16_to_f32(src[i]));
        if (a > amax) amax = a;
      }
      if (amax == 0.0f) continue;
      const uint8_t sc = mx_scale_code(amax, 2);
      *sd = sc;
      for (int32_t i = 0; i < 32; ++i) {
        const uint8_t c = orc_e2m1_from_f32(mx_scale_down(orc_bf16_to_f32(src[i]), sc));
        qd[i / 2] |= (uint8_t)(i % 2 ? c << 4 : c);
      }
    }
  }
}

/* Scale-factor atom layout: see oracle.h. */
void orc_swizzle_scales(int64_t rows, int32_t nsf, const uint8_t *linear,
                        uint8_t *out) {
  const int32_t atom_rows = 32 * 4;            /* SF_ATOM_M[0] * 4 row groups */
  const int32_t atom_cols = 4;                 /* SF_ATOM_M[1]                */
  const int32_t row_stride = atom_cols * 4;    /* SF_ROW_STRIDE_LOCAL = 16    */
  const int32_t atom_bytes = 32 * row_stride;  /* SF_ATOM_ELEMS_LOCAL = 512   */
  const int64_t row_tiles = (rows + atom_rows - 1) / atom_rows;
  const int64_t col_tiles = (nsf + atom_cols - 1) / atom_cols;
  memset(out, 0, (size_t)(row_tiles * col_tiles * atom_bytes));
  for (int64_t m = 0; m < rows; ++m)
    for (int32_t c = 0; c < nsf; ++c) {
      int64_t atom = (m / atom_rows) * col_tiles + c / atom_cols;
      int64_t inner = (m % 32) * row_stride + ((m / 32) % 4) * 4 + c % atom_cols;
      out[atom * atom_bytes + inner] = linear[m * nsf + c];
    }
}

/* ------------------------------------------------------------------ */
/* Combine                                                             */
/* ------------------------------------------------------------------ */

/* DeepSpeed combine: gather each token's expert results back and weight
 * them by the gate values.  NeMo moe_router_dtype = 'fp32': weights and
 * the weighted average in fp32.  Mojo ep_comm router_weights_wrapper_type:
 * one fp32 weight per (token, k).  For token t the accumulator starts at
 * +0 and takes acc = fma(w[t,j], x[slot(t,j)], acc) for j = 0..k-1 in
 * order, skipping a pair without a row (masked, dropped, or a slot outside
 * [0, rows)); the result is rounded once to bfloat16. */
void orc_combine(int32_t N, int32_t k, int32_t H, int64_t rows,
                 const uint16_t *expert_out, const float *gates,
                 const int32_t *pair_slot, uint16_t *y) {
  for (int32_t t = 0; t < N; ++t) {
    for (int32_t h = 0; h < H; ++h) {
      float acc = 0.0f;
      for (int32_t j = 0; j < k; ++j) {
        int32_t s = pair_slot[(int64_t)t * k + j];
        if (s < 0 || s >= rows) continue;
        float x = orc_bf16_to_f32(expert_out[(int64_t)s * H + h]);
        acc = fmaf(gates[(int64_t)t * k + j], x, acc);
      }
      y[(int64_t)t * H + h] = orc_bf16_from_f32(acc);
    }
  }
}

/* ------------------------------------------------------------------ */
/* Backward                                                            */
/* ------------------------------------------------------------------ */

/* The dispatch copies token t's row to the rows of its pairs, so the
 * token's gradient is the sum of those rows' gradients (fp32, j in order,
 * one rounding to bfloat16). */
void orc_permute_backward(int32_t N, int32_t k, int32_t H, int64_t rows,
                          const uint16_t *grad_out, const int32_t *pair_slot,
                          uint16_t *grad_hidden) {
  for (int32_t t = 0; t < N; ++t)
    for (int32_t h = 0; h < H; ++h) {
      float acc = 0.0f;
      for (int32_t j = 0; j < k; ++j) {
        int32_t s = pair_slot[(int64_t)t * k + j];
        if (s < 0 || s >= rows) continue;
        acc = acc + orc_bf16_to_f32(grad_out[(int64_t)s * H + h]);
      }
      grad_hidden[(int64_t)t * H + h] = orc_bf16_from_f32(acc);
    }
}

/* y[t] = sum_j w[t,j] * x[slot(t,j)] (DeepSpeed combine), so
 * d y / d x[slot(t,j)] = w[t,j] and d y / d w[t,j] = x[slot(t,j)]. */
void orc_combine_backward(int32_t N, int32_t k, int32_t H, int64_t rows,
                          const uint16_t *grad_y, const uint16_t *expert_out,
                          const float *gates, const int32_t *pair_slot,
                          uint16_t *grad_expert_out, float *grad_gates) {
  for (int64_t i = 0; i < rows * H; ++i) grad_expert_out[i] = 0;
  for (int32_t t = 0; t < N; ++t)
    for (int32_t j = 0; j < k; ++j) {
      int64_t p = (int64_t)t * k + j;
      int32_t s = pair_slot[p];
      if (s < 0 || s >= rows) {
        grad_gates[p] = 0.0f;
        continue;
      }
      double dot = 0.0;
      for (int32_t h = 0; h < H; ++h) {
        float g = orc_bf16_to_f32(grad_y[(int64_t)t * H + h]);
        float x = orc_bf16_to_f32(expert_out[(int64_t)s * H + h]);
        grad_expert_out[(int64_t)s * H + h] = orc_bf16_from_f32(gates[p] * g);
        dot += (double)g * (double)x;
      }
      grad_gates[p] = (float)dot;
    }
}

/* DeepSpeed "pre-multiply token representations by router scores before
 * expert compute": every row starts as zeros; pair (t, j) with a row writes
 * its token scaled by its gate, one fp32 product and one rounding to bf16
 * per element. */
void orc_permute_premultiplied(int32_t N, int32_t k, int32_t H, int64_t rows,
                               const uint16_t *hidden, const float *gates,
                               const int32_t *pair_slot, uint16_t *out) {
  for (int64_t i = 0; i < rows * H; ++i) out[i] = 0;
  for (int32_t t = 0; t < N; ++t)
    for (int32_t j = 0; j < k; ++j) {
      const int64_t p = (int64_t)t * k + j;
      const int32_t s = pair_slot[p];
      if (s < 0 || s >= rows) continue;
      for (int32_t h = 0; h < H; ++h) {
        const float x = orc_bf16_to_f32(hidden[(int64_t)t * H + h]);
        out[(int64_t)s * H + h] = orc_bf16_from_f32(gates[p] * x);
      }
    }
}

/* ------------------------------------------------------------------ */
/* SwiGLU + requantisation                                             */
/* ------------------------------------------------------------------ */

/* 2^n as a float for n in [-126, 127]. */
static float pow2i(int n) { return f32_from_bits((uint32_t)(n + 127) << 23); }

float orc_exp(float x) {
  const float log2e = 1.44269504f;          /* RN(log2 e)                      */
  const float ln2_hi = 0.693145751953125f;  /* ln 2 to 16 significant bits     */
  const float ln2_lo = 1.42860682e-06f;     /* RN(ln 2 - ln2_hi)               */
  if (isnan(x)) return x;
  if (x > 88.75f) return INFINITY;
  if (x < -104.0f) return 0.0f;
  const float n = rintf(x * log2e);
  float r = fmaf(-n, ln2_hi, x);
  r = fmaf(-n, ln2_lo, r);
  /* e^r = sum r^i / i!, i = 0..7, Horner */
  float p = 1.98412698e-04f;                /* 1/7! */
  p = fmaf(p, r, 1.38888889e-03f);          /* 1/6! */
  p = fmaf(p, r, 8.33333333e-03f);          /* 1/5! */
  p = fmaf(p, r, 4.16666667e-02f);          /* 1/4! */
  p = fmaf(p, r, 1.66666667e-01f);          /* 1/3! */
  p = fmaf(p, r, 0.5f);                     /* 1/2! */
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  const int ni = (int)n;
  if (ni > 127) return (p * pow2i(127)) * pow2i(ni - 127);
  if (ni < -126) return (p * pow2i(ni + 64)) * pow2i(-64);
  return p * pow2i(ni);
}

void orc_exp_n(const float *in, float *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_exp(in[i]);
}

float orc_silu(float g) { return g / (1.0f + orc_exp(-g)); }

uint8_t orc_e8m0_from_exponent(int32_t e) {
  int32_t c = e + 127;
  if (c < 0) c = 0;
  if (c > 254) c = 254;
  return (uint8_t)c;
}

/* floor(log2 a) of a finite a > 0 (subnormals included) */
static int32_t floor_log2(float a) {
  int e;
  frexpf(a, &e); /* a = f * 2^e, f in [0.5, 1) */
  return e - 1;
}

void orc_swiglu_quant(int64_t rows, int32_t I, const uint16_t *gate_up,
                      int interleaved, const int32_t *row_src, int format,
                      float global_scale, uint8_t *codes, uint8_t *scales) {
  const int64_t code_row = format == 0 || format == 2 ? I / 2
                           : format == 1               ? I
                           : format == 3               ? 2 * (int64_t)I
                                                       : 3 * (int64_t)I / 4;
  const int64_t scale_row = format == 0 ? I / 16 : format == 3 ? 0 : I / 32;
  float *y = (float *)malloc(sizeof(float) * (size_t)I);
  for (int64_t r = 0; r < rows; ++r) {
    uint8_t *cd = codes + r * code_row;
    uint8_t *sd = scales + r * scale_row;
    if (row_src[r] < 0) {
      memset(cd, 0, (size_t)code_row);
      if (scale_row) memset(sd, 0, (size_t)scale_row);
      continue;
    }
    const uint16_t *in = gate_up + r * 2 * (int64_t)I;
    for (int32_t i = 0; i < I; ++i) {
      float g = orc_bf16_to_f32(interleaved ? in[2 * i] : in[i]);
      float u = orc_bf16_to_f32(interleaved ? in[2 * i + 1] : in[I + i]);
      y[i] = orc_silu(g) * u;
    }
    if (format == 3) {
      /* bf16, rounded to nearest even, little-endian */
      for (int32_t i = 0; i < I; ++i) {
        const uint16_t b = orc_bf16_from_f32(y[i]);
        cd[2 * i] = (uint8_t)(b & 0xFF);
        cd[2 * i + 1] = (uint8_t)(b >> 8);
      }
    } else if (format == 4 || format == 5) {
      /* MXFP6: E2M3 (emax 2) or E3M2 (emax 4) codes, E8M0 scale per 32,
       * 24 bytes of packed codes per block */
      const int32_t emax = format == 4 ? 2 : 4;
      uint8_t c6[32];
      for (int32_t b = 0; b < I / 32; ++b) {
        float amax = 0.0f;
        for (int32_t i = 0; i < 32; ++i) {
          float a = fabsf(y[32 * b + i]);
          if (a > amax) amax = a;
        }
        uint8_t sc = 0;
        memset(c6, 0, sizeof c6);
        if (amax > 0.0f) {
          sc = mx_scale_code(amax, emax);
          for (int32_t i = 0; i < 32; ++i) {
            const float v = mx_scale_down(y[32 * b + i], sc);
            c6[i] = format == 4 ? orc_e2m3_from_f32(v) : orc_e3m2_from_f32(v);
          }
        }
        sd[b] = sc;
        orc_pack_fp6(c6, 32, cd + 24 * b);
      }
    } else if (format == 0) {
      /* NVFP4, exactly the dispatch's rule on the fp32 values */
      for (int32_t b = 0; b < I / 16; ++b) {
        float amax = 0.0f;
        for (int32_t i = 0; i < 16; ++i) {
          float a = fabsf(y[16 * b + i]);
          if (a > amax) amax = a;
        }
        uint8_t sq = orc_e4m3_from_f32((amax / 6.0f) / global_scale);
        float d = orc_e4m3_to_f32(sq) * global_scale;
        sd[b] = sq;
        for (int32_t m = 0; m < 8; ++m) {
          uint8_t lo = 0, hi = 0;
          if (d > 0.0f) {
            lo = orc_e2m1_from_f32(y[16 * b + 2 * m] / d);
            hi = orc_e2m1_from_f32(y[16 * b + 2 * m + 1] / d);
          }
          cd[8 * b + m] = (uint8_t)(lo | (hi << 4));
        }
      }
    } else {
      const int32_t emax = format == 1 ? 8 : 2;
      for (int32_t b = 0; b < I / 32; ++b) {
        float amax = 0.0f;
        for (int32_t i = 0; i < 32; ++i) {
          float a = fabsf(y[32 * b + i]);
          if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
          sd[b] = 0;
          if (format == 1) memset(cd + 32 * b, 0, 32);
          else memset(cd + 16 * b, 0, 16);
          continue;
        }
        const uint8_t sc = orc_e8m0_from_exponent(floor_log2(amax) - emax);
        sd[b] = sc;
        const int32_t X = (int32_t)sc - 127;
        for (int32_t i = 0; i < 32; ++i) {
          /* y * 2^-X: X in [-127, 125] (sc <= 252: floor(log2 amax) <= 127
           * for a float and emax >= 2), so 2^-X is a normal float */
          float v = y[32 * b + i] * pow2i(-X);
          if (format == 1) {
            cd[32 * b + i] = orc_e4m3_from_f32(v);
          } else if (i % 2 == 0) {
            cd[16 * b + i / 2] = orc_e2m1_from_f32(v);
          } else {
            cd[16 * b + i / 2] |= (uint8_t)(orc_e2m1_from_f32(v) << 4);
          }
        }
      }
    }
  }
  free(y);
}
