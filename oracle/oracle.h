/*
 * oracle.h -- plain, slow, single-threaded CPU oracle for MoE token
 * dispatch (layout + permute, bf16 / block FP8 / NVFP4 payloads) and
 * combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load or call this code.  It shares no
 * source, header, table or helper with the CUDA library; the two agree
 * only because both follow the same definitions.
 *
 * Sources the functions follow (cited by page title and section):
 *   [NKI]  AWS Neuron NKI "Permute A2AV Kernel API Reference", permute_a2av
 *          parameters (packed_source_indices, send_counts, recv_capacity)
 *          and return values ([C,H] packed rows + deterministic zero
 *          padding; [4,EP] uint32 counts/displacements in elements).
 *   [NEMO] NeMo AutoModel token_dispatcher API: _indices_to_multihot
 *          ("-1 means masked out"), get_number_of_tokens_per_expert,
 *          TokenDispatcherConfig.moe_expert_capacity_factor and
 *          moe_router_dtype (fp32 routing weights and weighted averaging).
 *   [DS]   DeepSpeed v0.19.4 function list: the combine docstring (gather
 *          each token's expert results and weight them by the gates) and
 *          the capacity dispatch docstring ([e, c, m] expert-slot buffer).
 *   [EPC]  Mojo MAX ep_comm module: BF16TokenFormat,
 *          BlockwiseFP8TokenFormat, NVBlockScaledTokenFormat,
 *          router_weights_wrapper_type (fp32 gate per (token, k)).
 *   [EPD]  Mojo MAX Struct_ep_dispatch_async_block_scaled_nv: NVFP4
 *          payload with a global input scale supplied by the caller.
 * Format definitions written out from the public specifications:
 *   IEEE 754 binary32; bfloat16 = top half of binary32 rounded to nearest
 *   even; OCP 8-bit floating point (E4M3, "fn" variant: no infinities,
 *   max 448); OCP Microscaling v1.0 (E2M1: max 6, no inf/NaN).
 *
 * Parity status: every function here is pinned by tests/test_oracle_*.py
 * to something other than itself (library sorts, torch casts, brute-force
 * nearest-value search over the format tables, an arithmetic
 * round-half-even for FP6, the OCP value tables, closed forms, adjoint
 * identities, invariants the pages state).  The block-scale conventions of
 * the FP8 and NVFP4 quantisers (divide by the stored scale; scale =
 * amax/448; NVFP4 block scale = e4m3((amax/6)/global_scale)), the MX shared
 * scale rule, the MXFP6 packing, the fixed e^x sequence of the SwiGLU and
 * the scale-factor atom layout are readings of the pages, which print no
 * worked example; the arithmetic under those readings is pinned.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status bits reported by orc_layout (same meaning as the library's). */
#define ORC_STATUS_ID_RANGE 1u  /* an id outside [-1, E)                  */
#define ORC_STATUS_DUP_ID 2u    /* a token names one expert twice          */
#define ORC_STATUS_CAPACITY 4u  /* packed mode: more routed rows than C    */
#define ORC_FLAG_CHECK_DUPLICATES 1u

/* ---- number formats -------------------------------------------------- */
uint16_t orc_bf16_from_f32(float f);
float orc_bf16_to_f32(uint16_t b);
uint8_t orc_e4m3_from_f32(float f); /* RNE, saturate to +-448 */
float orc_e4m3_to_f32(uint8_t c);
uint8_t orc_e2m1_from_f32(float f); /* RNE, saturate to +-6, 4-bit code */
float orc_e2m1_to_f32(uint8_t c);

void orc_bf16_from_f32_n(const float *in, uint16_t *out, int64_t n);
void orc_e4m3_from_f32_n(const float *in, uint8_t *out, int64_t n);
void orc_e2m1_from_f32_n(const float *in, uint8_t *out, int64_t n);
/* OCP MX v1.0 FP6: E2M3 (max 7.5) and E3M2 (max 28), 6-bit codes with the
 * sign in bit 5; RNE, saturating, by nearest-value search over the codes. */
uint8_t orc_e2m3_from_f32(float f);
uint8_t orc_e3m2_from_f32(float f);
float orc_e2m3_to_f32(uint8_t c);
float orc_e3m2_to_f32(uint8_t c);
void orc_e2m3_from_f32_n(const float *in, uint8_t *out, int64_t n);
void orc_e3m2_from_f32_n(const float *in, uint8_t *out, int64_t n);
/* n (a multiple of 4) 6-bit codes -> 3n/4 bytes: code i at bits [6i, 6i+6)
 * of each little-endian 24-bit group of four. */
void orc_pack_fp6(const uint8_t *codes, int64_t n, uint8_t *out);

/* ---- dispatch layout --------------------------------------------------
 * ids[N*k] int32 (row-major [N,k]); E experts in S contiguous segments of
 * L = E/S experts.  expert_capacity Ce == 0 selects packed (dropless) mode
 * with C = recv_capacity rows; Ce > 0 selects the capacity layout [E,Ce].
 * pad > 1 (packed mode only) starts every expert's rows at a multiple of pad
 * (NeMo TokenDispatcherConfig.moe_router_expert_pad_multiple).
 * Outputs: expert_counts[E], expert_offsets[E+1], meta[4*S] (row-major
 * [4,S]), row_src[rows] (rows = C, or E*Ce), pair_slot[N*k], drop_mask[N*k]
 * (may be NULL).  Returns status bits.                                   */
uint32_t orc_layout(int32_t N, int32_t k, int32_t E, int32_t S, int64_t C,
                    int32_t Ce, int32_t pad, uint32_t flags, int32_t H,
                    const int32_t *ids, int32_t *expert_counts,
                    int32_t *expert_offsets, uint32_t *meta, int32_t *row_src,
                    int32_t *pair_slot, uint8_t *drop_mask);

/* ---- block-scale atom layout ------------------------------------------
 * Mojo MAX ep_comm: SF_ROW_STRIDE_LOCAL = SF_ATOM_M[1] * 4 and
 * SF_ATOM_ELEMS_LOCAL = SF_ATOM_M[0] * SF_ROW_STRIDE_LOCAL, with SF_ATOM_M
 * read as (32, 4): an atom holds the scales of 128 rows x 4 scale columns in
 * 512 bytes.  Scale (m, c) of a [rows, nsf] matrix goes to atom
 * (m / 128, c / 4) -- atoms row-tile-major, ceil(nsf / 4) per row tile --
 * at byte (m % 32) * 16 + ((m / 32) % 4) * 4 + c % 4 of the atom.
 * out has ceil(rows/128)*128 * ceil(nsf/4)*4 bytes; bytes no scale maps to
 * are zero.                                                              */
void orc_swizzle_scales(int64_t rows, int32_t nsf, const uint8_t *linear,
                        uint8_t *out);

/* ---- permute: out row r = hidden row row_src[r], or zeros ------------- */
void orc_permute_bf16(int64_t rows, int32_t H, const uint16_t *hidden,
                      const int32_t *row_src, uint16_t *out);
void orc_permute_fp8(int64_t rows, int32_t H, const uint16_t *hidden,
                     const int32_t *row_src, uint8_t *q, float *scales);
void orc_permute_nvfp4(int64_t rows, int32_t H, const uint16_t *hidden,
                       const int32_t *row_src, float global_scale,
                       uint8_t *q, uint8_t *scales);
/* MX token format (OCP MXFP4): E2M1 codes [rows, H/2], E8M0 scales
 * [rows, H/32]; X = floor(log2(amax)) - 2 per block of 32, codes of
 * x * 2^-X; an all-zero block has scale code 0. */
void orc_permute_mxfp4(int64_t rows, int32_t H, const uint16_t *hidden,
                       const int32_t *row_src, uint8_t *q, uint8_t *scales);

/* ---- combine ---------------------------------------------------------- */
void orc_combine(int32_t N, int32_t k, int32_t H, int64_t rows,
                 const uint16_t *expert_out, const float *gates,
                 const int32_t *pair_slot, uint16_t *y);

/* ---- SwiGLU + requantisation (Mojo MAX ep_comm fused_silu_*_kernel and
 * MXTokenFormat) -----------------------------------------------------------
 * e^x: Cody-Waite range reduction (n = rint(x * log2 e), r = x - n*ln2 with
 * ln2 split in two constants) and the degree-7 Taylor polynomial of e^r in
 * Horner form with fmaf, then scaling by 2^n; one fixed fp32 operation
 * sequence, written from the mathematics (Cody & Waite, Software Manual for
 * the Elementary Functions, 1980).  x < -104 gives 0, x > 88.75 gives inf.
 * silu(g) = g / (1 + e^-g);  swiglu(g, u) = silu(g) * u  (fp32, no fused
 * multiply-add except inside e^x).
 * E8M0 (OCP MX v1.0 shared scale): code c means 2^(c-127), 255 is NaN.     */
float orc_exp(float x);
float orc_silu(float g);
uint8_t orc_e8m0_from_exponent(int32_t e); /* 2^e -> code, clamped to [0,254] */
void orc_exp_n(const float *in, float *out, int64_t n);

/* rows x I SwiGLU of bf16 gate/up rows (split: columns [0,I) gate and
 * [I,2I) up; interleaved: gate at even, up at odd columns), quantised:
 *   format 0 NVFP4: E2M1 codes [rows, I/2], E4M3 scales [rows, I/16] as in
 *            the dispatch (global scale gs)
 *   format 1 MXFP8: E4M3 codes [rows, I], E8M0 scales [rows, I/32]
 *   format 2 MXFP4: E2M1 codes [rows, I/2], E8M0 scales [rows, I/32]
 *   format 3 BF16:  bf16 [rows, I] (2I bytes a row, little-endian), no scales
 *   format 4 MXFP6 E2M3: packed 6-bit codes [rows, 3I/4], E8M0 [rows, I/32]
 *   format 5 MXFP6 E3M2: packed 6-bit codes [rows, 3I/4], E8M0 [rows, I/32]
 * MX block of 32: X = floor(log2(amax)) - emax (8 for E4M3, 2 for E2M1 and
 * E2M3, 4 for E3M2),
 * scale code E8M0(X), element code = E(y * 2^-X) rounded to nearest even with
 * saturation; an all-zero block gets scale code 0 and codes 0.  Rows whose
 * row_src is -1 (no routed token) are all-zero bytes and are not read.     */
void orc_swiglu_quant(int64_t rows, int32_t I, const uint16_t *gate_up,
                      int interleaved, const int32_t *row_src, int format,
                      float global_scale, uint8_t *codes, uint8_t *scales);

/* ---- backward -----------------------------------------------------------
 * The gradients of the two data movements (training, NeMo token_dispatcher
 * top-k probabilities [T, K] whose gradient flows back through combine):
 *   permute backward: grad_hidden[t] = bf16(sum over j of grad_out[slot(t,j)])
 *     in fp32, j in order, pairs without a row skipped;
 *   combine backward: grad_expert_out[slot(t,j)] = bf16(w[t,j] * grad_y[t])
 *     (fp32 product), rows no pair owns are zero; grad_gates[t,j] =
 *     sum over h of grad_y[t,h] * expert_out[slot(t,j),h], evaluated in
 *     float64 and rounded once to fp32 (0 for a pair without a row).      */
void orc_permute_backward(int32_t N, int32_t k, int32_t H, int64_t rows,
                          const uint16_t *grad_out, const int32_t *pair_slot,
                          uint16_t *grad_hidden);
void orc_combine_backward(int32_t N, int32_t k, int32_t H, int64_t rows,
                          const uint16_t *grad_y, const uint16_t *expert_out,
                          const float *gates, const int32_t *pair_slot,
                          uint16_t *grad_expert_out, float *grad_gates);

/* ---- pre-multiplied gates ---------------------------------------------
 * DeepSpeed v0.19.4 function list: token representations pre-multiplied by
 * their router scores before expert compute.  The dispatch then writes each
 * pair's row scaled by its gate,
 *   out[slot(t,j)] = bf16(w[t,j] * hidden[t])  (fp32 product, one rounding),
 * rows no pair owns are zero; the combine of this variant is the unweighted
 * sum (orc_permute_backward's arithmetic) and its backward is the weighted
 * combine (grad of hidden) and a dot product (grad of the gates).           */
void orc_permute_premultiplied(int32_t N, int32_t k, int32_t H, int64_t rows,
                               const uint16_t *hidden, const float *gates,
                               const int32_t *pair_slot, uint16_t *out);

#ifdef __cplusplus
}
#endif
#endif
