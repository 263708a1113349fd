/*
 * moe_dc.h -- C ABI of libmoedc.so: the single-GPU core of Mixture-of-Experts
 * token dispatch and combine on NVIDIA B200 (sm_100a).
 *
 * Five calls follow one another on one CUDA stream:
 *
 *   moe_dispatch_layout      topk_ids [N,k] -> per-expert counts and start
 *                            rows, the [4,S] counts/displacements table, the
 *                            source-row map row_src and the per-pair rows
 *                            pair_slot
 *   moe_permute              hidden_states [N,H] bf16 -> [rows,H] bf16,
 *                            expert-major, zero padding rows
 *   moe_permute_quant_fp8    same rows, E4M3 codes + one fp32 scale per 1x128
 *   moe_permute_quant_nvfp4  same rows, E2M1 codes (2 per byte) + one E4M3
 *                            scale per 16 elements + caller's global scale
 *   moe_combine              expert outputs [rows,H] bf16 + gates [N,k] fp32
 *                            -> [N,H] bf16, fp32 weighted sum in fixed k order
 *
 * Further calls: moe_permute_quant_mxfp4 (the MX token format: E2M1 codes +
 * one E8M0 scale per 32 elements), moe_swiglu_quant (silu(gate) * up of the
 * expert rows that hold a token, as bf16 or requantised), the gradients
 * moe_permute_backward and moe_combine_backward, moe_permute_premultiplied
 * (the dispatch with each pair's row scaled by its gate), moe_permute_to_peers
 * and its FP8 / NVFP4 forms (the dispatch written straight into the receive
 * buffers of the ranks that own the experts), moe_combine_from_peers (the
 * combine reading the expert outputs where those ranks computed them), and moe_dispatch_layout_noalloc (the layout without a
 * caller workspace).  Two builds of the same sources add checks and records:
 * device index checks (moe_debug_violations) and per-CTA trace records
 * (moe_trace_attach).
 *
 * Notation: N tokens, H hidden size, E experts, k = top_k choices per token,
 * S destination segments of L = E/S consecutive experts, P = N*k pairs; pair
 * p = t*k + j routes token t to expert topk_ids[p].  rows = recv_capacity in
 * packed mode, E*expert_capacity in capacity mode (moe_output_rows()).
 *
 * Conventions for every call:
 *   - Pointers named *_ids, *_states, out*, scales*, gates, pair_slot,
 *     row_src, expert_*, meta, status and workspace are DEVICE pointers
 *     owned by the caller; the library allocates no memory.  moe_problem is
 *     a HOST pointer, read during the call only.
 *   - bf16 data is passed as void* to 16-byte-aligned buffers of IEEE
 *     bfloat16 (the layout of __nv_bfloat16), row-major with no padding.
 *   - int32, uint32 and fp32 arrays (ids, maps, counts, meta, status, gates,
 *     fp32 scales) are 4-byte aligned; each call checks every pointer's
 *     alignment on the host and returns MOE_ERR_INVALID_ARG, launching
 *     nothing, for a misaligned one.
 *   - Every call only enqueues kernels on `stream` (a cudaStream_t) and
 *     returns; nothing synchronises with the host.
 *   - A moe_status return reports argument errors found on the host before
 *     anything is launched (nothing is launched then) and launch errors
 *     (MOE_ERR_CUDA).  Data-dependent conditions found on the device are
 *     reported in the `status` word of moe_dispatch_layout (MOE_STATUS_*).
 *   - Results are deterministic: identical for identical inputs, whatever
 *     the grid size or scheduling.
 */
#ifndef MOE_DC_H
#define MOE_DC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported entry points keep default visibility even when the library is
 * built with hidden visibility. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* cudaStream_t without pulling in the CUDA headers (same type). */
typedef struct CUstream_st *moe_stream_t;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, negative size, misaligned */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside the supported limits     */
  MOE_ERR_CUDA = 3,              /* a CUDA launch or runtime error          */
  MOE_ERR_NOT_BUILT = 4          /* the call needs a build option that this
                                    library was built without               */
} moe_status;

/* Bits of the device status word written by moe_dispatch_layout. */
enum {
  MOE_STATUS_ID_RANGE = 1u, /* an id outside [-1, E): treated as masked     */
  MOE_STATUS_DUP_ID = 2u,   /* a token names one expert (an id in [0, E))
                               twice; repeated -1 or out-of-range ids are
                               not duplicates (checked only with
                               MOE_FLAG_CHECK_DUPLICATES)                  */
  MOE_STATUS_CAPACITY = 4u, /* packed mode: more routed pairs than
                               recv_capacity; the excess pairs get no row  */
  MOE_STATUS_TIMEOUT = 8u   /* a bounded wait of the scan gave up (about one
                               second); counts and rows are then invalid   */
};

/* Problem flags. */
enum {
  MOE_FLAG_CHECK_DUPLICATES = 1u,
  /* The layout picks one of three equivalent kernels by size: one
   * thread-block cluster when the pairs fit in at most 16 tiles of 8192
   * pairs (8 where the device cannot schedule 16-CTA clusters) and the rows
   * number at most 2^18; else one cooperative launch with a decoupled
   * look-back scan up to 128 tiles of 4096 pairs; else a scan kernel and an
   * emit kernel.  These two flags force the latter kernels.  Results are
   * identical; for testing and tuning. */
  MOE_FLAG_LAYOUT_TWO_PASS = 2u,
  /* moe_permute_quant_nvfp4 writes the E4M3 scales in the block-scale atom
   * layout of NVIDIA block-scaled tensor-core operands instead of row-major
   * (see moe_permute_quant_nvfp4). */
  MOE_FLAG_NVFP4_SWIZZLED_SCALES = 4u,
  /* Run the layout as the one-launch look-back kernel even where the cluster
   * kernel applies (see MOE_FLAG_LAYOUT_TWO_PASS). */
  MOE_FLAG_LAYOUT_LOOKBACK = 8u,
  /* Test hook: the first scan tile never publishes its counts, so every
   * later tile's bounded wait runs out and MOE_STATUS_TIMEOUT is reported.
   * Results are invalid; used only to test the timeout path.  Implies the
   * look-back kernels (the cluster kernel has no bounded wait). */
  MOE_FLAG_TEST_STALL_SCAN = 0x80000000u
};

/* Supported limits (MOE_ERR_UNSUPPORTED_SHAPE beyond them). */
#define MOE_MAX_EXPERTS 2048
#define MOE_MAX_TOPK 16

typedef struct moe_problem {
  int32_t num_tokens;      /* N >= 0                                       */
  int32_t hidden;          /* H > 0; H % 8 == 0 (bf16 permute, combine),
                              H % 128 == 0 (FP8), H % 32 == 0 (NVFP4)      */
  int32_t num_experts;     /* E, 1..MOE_MAX_EXPERTS                        */
  int32_t top_k;           /* k, 1..MOE_MAX_TOPK                           */
  int32_t num_segments;    /* S >= 1 with E % S == 0                       */
  int32_t expert_capacity; /* Ce: 0 = packed dropless layout with
                              recv_capacity rows; > 0 = capacity layout
                              [E, Ce] rows, overflow dropped               */
  int64_t recv_capacity;   /* C rows of the packed layout (ignored when
                              Ce > 0)                                      */
  uint32_t flags;          /* MOE_FLAG_*                                   */
  int32_t expert_pad_multiple; /* packed mode: 0 or 1 = experts packed back
                              to back; m > 1 = every expert's block of rows
                              is its count rounded up to a multiple of m
                              (NeMo moe_router_expert_pad_multiple), so each
                              expert starts at a multiple of m; must be 0
                              in capacity mode                             */
} moe_problem;

/* Rows of the dispatch output: recv_capacity, or E * expert_capacity.
 * Returns -1 for an invalid problem. */
MOE_API int64_t moe_output_rows(const moe_problem *problem);

/* Bytes of device workspace moe_dispatch_layout needs for this problem
 * (control counters, per-expert totals, scan tile states).  The workspace
 * must be zero-filled once before its first use (e.g. cudaMemset); every
 * completed layout call returns all of it to zero, so a workspace sized for
 * the largest problem can serve any later call on the same stream.  Calls
 * sharing one workspace must not overlap on the GPU.  Returns 0 for an
 * invalid problem. */
MOE_API size_t moe_workspace_bytes(const moe_problem *problem);

/* Dispatch layout: a stable counting sort of the pairs by expert.
 *
 * Defines (NKI "Permute A2AV Kernel API Reference", permute_a2av):
 * packed_source_indices (here row_src) lists source tokens in
 * destination-major order; send_counts / displacements form a [4, EP]
 * uint32 table "all measured in elements"; recv_capacity is the static row
 * count of the packed buffer, padded with zeros.  Id -1 means masked (NeMo
 * AutoModel token_dispatcher, _indices_to_multihot).  Tokens per expert:
 * NeMo get_number_of_tokens_per_expert.  Capacity layout: DeepSpeed capacity
 * dispatch ([e, c, m] expert-slot buffer) with NeMo's expert capacity.
 *
 * Inputs:
 *   topk_ids       int32 [N, k] row-major.  Entries in [0, E) route a pair,
 *                  -1 masks it; anything else sets MOE_STATUS_ID_RANGE and
 *                  is treated as masked.
 * Outputs (all fully overwritten):
 *   expert_counts  int32 [E]: routed pairs per expert (packed: the true
 *                  count, even past recv_capacity; capacity: min(count, Ce)).
 *   expert_offsets int32 [E+1]: first row of each expert (packed: exclusive
 *                  cumulative sum of expert_counts, each rounded up to
 *                  expert_pad_multiple when that is > 1, [E] = total;
 *                  capacity: e*Ce).
 *   meta           uint32 [4, S] row-major, in elements (rows * H): row 0
 *                  send counts per segment (packed: the segment's expert
 *                  blocks, padding included; capacity: kept rows), row 1
 *                  send displacements (packed: exclusive cumulative sum of
 *                  row 0; capacity: s*L*Ce*H), rows 2-3 the receive counts /
 *                  displacements, equal to rows 0-1 on one GPU.
 *   row_src        int32 [rows]: source token of each row, -1 for padding
 *                  (rows past the total and, with expert_pad_multiple > 1,
 *                  the tail of each expert's block).  Within an expert rows
 *                  follow ascending pair index t*k+j.
 *   pair_slot      int32 [N, k]: row of each pair, -1 when the pair is
 *                  masked, out of range, dropped (capacity mode) or beyond
 *                  recv_capacity (packed mode).
 *   drop_mask      uint8 [N, k] or NULL: 1 for a pair with a valid id that
 *                  got no row, else 0.
 *   status         uint32 device word, overwritten with this call's
 *                  MOE_STATUS_* bits when the call's kernels complete.
 *   workspace      moe_workspace_bytes() bytes, see there.
 * Host checks: sizes within limits, E % S == 0, rows*H and (N*k +
 * E*(expert_pad_multiple-1))*H fit in uint32 (the metadata is uint32
 * elements), required pointers non-null. */
MOE_API moe_status moe_dispatch_layout(const moe_problem *problem, const int32_t *topk_ids,
                               int32_t *expert_counts, int32_t *expert_offsets,
                               uint32_t *meta, int32_t *row_src, int32_t *pair_slot,
                               uint8_t *drop_mask, uint32_t *status, void *workspace,
                               moe_stream_t stream);

/* Size of the static scratch of moe_dispatch_layout_noalloc (1 MiB). */
#define MOE_NOALLOC_SCRATCH_BYTES 1048576

/* moe_dispatch_layout for callers that cannot allocate device memory.  The
 * pages have no counterpart: this entry point exists for callers that may not
 * call cudaMalloc or any allocating routine -- for example code whose device
 * memory is wholly owned by a framework's caching allocator or a fixed
 * up-front memory plan, or plugin code with no handle to an allocator -- and
 * so cannot provide the workspace buffer.
 *
 * Same arguments, outputs, checks and results as moe_dispatch_layout, minus
 * `workspace`: the scratch is a static device array of
 * MOE_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.  Nothing is allocated or freed.
 *   - A problem whose moe_workspace_bytes() exceeds MOE_NOALLOC_SCRATCH_BYTES
 *     is rejected with MOE_ERR_UNSUPPORTED_SHAPE before anything is launched
 *     (at E = 256 that is above about 2 million pairs); use
 *     moe_dispatch_layout with a workspace for such problems.
 *   - The first call on a device looks up the array's device address on that
 *     device (it must be the current device); make that first call before any
 *     stream capture.  The address is kept for the life of the process, so
 *     do not call this entry point on a device after cudaDeviceReset() of
 *     that device (the reset unloads the library's device code and the kept
 *     address no longer names the array).
 *   - Every call shares the one array and finds what the previous call left
 *     in it; each call zero-fills the part it uses on its own stream before
 *     launching.  Calls that overlap on the GPU (other streams, other host
 *     threads) race on the array: serialise them. */
MOE_API moe_status moe_dispatch_layout_noalloc(const moe_problem *problem,
                                               const int32_t *topk_ids, int32_t *expert_counts,
                                               int32_t *expert_offsets, uint32_t *meta,
                                               int32_t *row_src, int32_t *pair_slot,
                                               uint8_t *drop_mask, uint32_t *status,
                                               moe_stream_t stream);

/* Permute, bf16 payload: out[r, :] = hidden_states[row_src[r], :], or zeros
 * when row_src[r] == -1.  NKI permute_a2av return value ([C, H] packed rows
 * followed by deterministic zero padding); Mojo MAX ep_comm BF16TokenFormat.
 *   hidden_states  bf16 [N, H], 16-byte aligned
 *   row_src        int32 [rows] and pair_slot int32 [N, k] from the layout
 *   out            bf16 [rows, H], 16-byte aligned, fully overwritten
 * Requires H % 8 == 0.  Each token row is read from HBM once and written to
 * its k rows; pair_slot entries outside [0, rows) are skipped. */
MOE_API moe_status moe_permute(const moe_problem *problem, const void *hidden_states,
                       const int32_t *row_src, const int32_t *pair_slot, void *out,
                       moe_stream_t stream);

/* Dispatch permute fused with the expert-parallel send: each segment's rows
 * are stored straight into the receive buffer of the rank that owns its
 * experts (peer stores over NVLink / NVSwitch) instead of into a local send
 * buffer that an all-to-all then ships.  NKI "Permute A2AV Kernel API
 * Reference" (the [4, EP] table: segment s of the packed buffer is the block
 * for rank s, at its send displacement); Mojo MAX ep_comm (dispatch kernels
 * that write tokens into the remote ranks' receive buffers).
 * Segment s = experts [sL, (s+1)L): packed mode, local rows [meta[1][s]/H,
 * + meta[0][s]/H) (expert blocks with their padding); capacity mode, rows
 * [s*L*Ce, (s+1)*L*Ce).  Row r of segment s is written, as moe_permute would
 * write it (padding rows as zeros), to row put_offsets[s] + r of the bf16
 * [*, H] buffer peer_out[s]; rows past the last segment are not written, nor
 * are segment rows at or past `rows` (a padded layout whose recv_capacity
 * cuts the last expert block short: meta still counts the whole block).
 *   hidden_states  bf16 [N, H], 16-byte aligned
 *   row_src, pair_slot, meta   from moe_dispatch_layout (meta may be NULL in
 *                  capacity mode)
 *   peer_out       DEVICE array of S device pointers (8-byte aligned array;
 *                  every pointer 16-byte aligned and writable from this GPU:
 *                  a peer mapping, or this rank's own receive buffer)
 *   put_offsets    DEVICE int64 [S]: first row of this rank's block in rank
 *                  s's receive buffer (rank s's receive displacement of this
 *                  source, in rows)
 * Requires H % 8 == 0.  The call only enqueues the stores: the receivers may
 * read after a barrier that follows the kernel's completion. */
MOE_API moe_status moe_permute_to_peers(const moe_problem *problem, const void *hidden_states,
                                        const int32_t *row_src, const int32_t *pair_slot,
                                        const uint32_t *meta, void *const *peer_out,
                                        const int64_t *put_offsets, moe_stream_t stream);

/* The FP8 and NVFP4 dispatches fused with the expert-parallel send, as
 * moe_permute_to_peers is for bf16 rows: the codes and scales that
 * moe_permute_quant_fp8 / moe_permute_quant_nvfp4 would write to local row r
 * of segment s are stored to row put_offsets[s] + (r - start of segment s)
 * of rank s's receive buffers peer_codes[s] and peer_scales[s] (padding
 * rows inside a segment as zeros; rows past the last segment are not
 * written).  Mojo MAX ep.dispatch_async.block.scaled.nv (the EP dispatch
 * with an NVFP4 payload and a per-tensor global input scale) and ep_comm
 * (BlockwiseFP8TokenFormat, NVBlockScaledTokenFormat); segments as in
 * moe_permute_to_peers.  Receive layouts, per rank s (rows = that rank's
 * receive rows):
 *   FP8    peer_codes[s]  E4M3 [rows, H], 16-byte aligned
 *          peer_scales[s] fp32 [rows, H/128] (row-major), 4-byte aligned
 *   NVFP4  peer_codes[s]  E2M1 [rows, H/2] (element 2m in the low nibble of
 *                         byte m), 16-byte aligned
 *          peer_scales[s] E4M3 [rows, H/16] row-major, 2-byte aligned
 *   peer_codes, peer_scales  DEVICE arrays of S device pointers (8-byte
 *                  aligned arrays; every pointer writable from this GPU)
 *   put_offsets    DEVICE int64 [S], rows, as in moe_permute_to_peers
 *   global_scale   NVFP4: DEVICE fp32 scalar, as in moe_permute_quant_nvfp4
 * Requires H % 128 == 0 (FP8) or H % 32 == 0 (NVFP4);
 * MOE_FLAG_NVFP4_SWIZZLED_SCALES is not supported here (rejected with
 * MOE_ERR_UNSUPPORTED_SHAPE): the atom layout tiles a receive buffer by 128
 * rows, which the receiver arranges over all of its sources. */
MOE_API moe_status moe_permute_quant_fp8_to_peers(const moe_problem *problem,
                                                  const void *hidden_states,
                                                  const int32_t *row_src,
                                                  const int32_t *pair_slot, const uint32_t *meta,
                                                  void *const *peer_codes,
                                                  void *const *peer_scales,
                                                  const int64_t *put_offsets, moe_stream_t stream);
MOE_API moe_status moe_permute_quant_nvfp4_to_peers(const moe_problem *problem,
                                                    const void *hidden_states,
                                                    const int32_t *row_src,
                                                    const int32_t *pair_slot,
                                                    const uint32_t *meta,
                                                    const float *global_scale,
                                                    void *const *peer_codes,
                                                    void *const *peer_scales,
                                                    const int64_t *put_offsets,
                                                    moe_stream_t stream);

/* Permute with pre-multiplied gates: out[slot(t,j), :] = bf16(gates[t,j] *
 * hidden_states[t, :]) -- one fp32 product and one rounding to nearest even
 * per element -- and zeros in the rows no pair owns.  DeepSpeed v0.19.4
 * function list: token representations pre-multiplied by their router
 * scores before expert compute.  The combine of this variant is then the
 * unweighted sum, moe_permute_backward's operation; its backward is
 * moe_combine (gradient of hidden_states) and the gate gradient of
 * moe_combine_backward with grad_y = hidden_states and expert_out = the
 * rows' gradient.
 *   hidden_states  bf16 [N, H], 16-byte aligned
 *   row_src        int32 [rows] and pair_slot int32 [N, k] from the layout
 *   gates          fp32 [N, k] (4-byte aligned)
 *   out            bf16 [rows, H], 16-byte aligned, fully overwritten
 * Requires H % 8 == 0; pair_slot entries outside [0, rows) are skipped. */
MOE_API moe_status moe_permute_premultiplied(const moe_problem *problem,
                                             const void *hidden_states, const int32_t *row_src,
                                             const int32_t *pair_slot, const float *gates,
                                             void *out, moe_stream_t stream);

/* Permute with block FP8 quantisation (Mojo MAX ep_comm
 * BlockwiseFP8TokenFormat).  For each output row and each 1x128 block:
 * amax = max |x|; scale = amax / 448 (fp32, round to nearest); code =
 * E4M3(x / scale) rounded to nearest even with saturation to +-448; a block
 * with amax == 0 gets scale 0 and codes 0.  Padding rows: codes 0, scales 0.
 *   out_e4m3  uint8 [rows, H] (16-byte aligned), scales fp32 [rows, H/128]
 * Requires H % 128 == 0. */
MOE_API moe_status moe_permute_quant_fp8(const moe_problem *problem, const void *hidden_states,
                                 const int32_t *row_src, const int32_t *pair_slot,
                                 uint8_t *out_e4m3, float *scales, moe_stream_t stream);

/* Permute with NVFP4 quantisation (Mojo MAX ep_comm NVBlockScaledTokenFormat
 * and Struct_ep_dispatch_async_block_scaled_nv: the global input scale is an
 * input).  global_scale is a device fp32 scalar gs (the decode global scale,
 * positive and finite).  Per 16-element block: amax; scale code sq =
 * E4M3((amax / 6) / gs); d = float(sq) * gs; code_i = E2M1(x_i / d) rounded
 * to nearest even with saturation to +-6, or 0 when d == 0.  Element 2m is
 * the low nibble of byte m.  Padding rows are all zero.
 *   out_e2m1     uint8 [rows, H/2] (16-byte aligned)
 *   scales_e4m3  uint8 [rows, H/16] (2-byte aligned), linear row-major; or,
 *                with MOE_FLAG_NVFP4_SWIZZLED_SCALES, the block-scale atom
 *                layout (Mojo MAX ep_comm SF_ATOM_M, SF_ROW_STRIDE_LOCAL,
 *                SF_ATOM_ELEMS_LOCAL, with SF_ATOM_M = (32, 4)): atoms of
 *                128 rows x 4 scale columns in 512 bytes, atoms row-tile
 *                major, ceil(H/64) atoms per 128-row tile; scale (m, c) at
 *                byte ((m/128)*ceil(H/64) + c/4)*512 + (m%32)*16 +
 *                ((m/32)%4)*4 + c%4.  The buffer then holds
 *                ceil(rows/128)*128 * ceil(H/64)*4 bytes (4-byte aligned),
 *                every one of them written (zero where no scale maps).
 * Requires H % 32 == 0. */
MOE_API moe_status moe_permute_quant_nvfp4(const moe_problem *problem, const void *hidden_states,
                                   const int32_t *row_src, const int32_t *pair_slot,
                                   const float *global_scale, uint8_t *out_e2m1,
                                   uint8_t *scales_e4m3, moe_stream_t stream);

/* MX token format (Mojo MAX ep_comm MXTokenFormat: MX FP4 quantisation of
 * the dispatched tokens; OCP Microscaling v1.0 MXFP4).  Same rows as
 * moe_permute; per block of 32 elements along H:
 *   X = floor(log2(amax)) - 2,  scale code = clamp(X + 127, 0, 254) (E8M0),
 *   code_i = E2M1_rne_satfinite(x_i * 2^-X);
 * an all-zero block has scale code 0 and codes 0.
 *   out_e2m1     uint8 [rows, H/2], element 2m in the low nibble of byte m,
 *                16-byte aligned, fully overwritten (padding rows 0)
 *   scales_e8m0  uint8 [rows, H/32] row-major, or, with
 *                MOE_FLAG_NVFP4_SWIZZLED_SCALES, the block-scale atom layout
 *                of moe_permute_quant_nvfp4 with H/32 scale columns
 *                (4-byte aligned then); fully overwritten
 * Requires H % 32 == 0. */
MOE_API moe_status moe_permute_quant_mxfp4(const moe_problem *problem, const void *hidden_states,
                                   const int32_t *row_src, const int32_t *pair_slot,
                                   uint8_t *out_e2m1, uint8_t *scales_e8m0,
                                   moe_stream_t stream);

/* Combine (DeepSpeed: gather each token's expert results back and weight
 * them by the gate values; NeMo moe_router_dtype 'fp32'; Mojo MAX ep_comm
 * router_weights_wrapper_type: one fp32 weight per (token, k)).
 *   expert_out  bf16 [rows, H], 16-byte aligned
 *   gates       fp32 [N, k]
 *   pair_slot   int32 [N, k] from the layout
 *   out         bf16 [N, H], 16-byte aligned, fully overwritten
 * out[t,:] = bf16_rne(acc) with acc = +0 then acc = fmaf(gates[t,j],
 * expert_out[pair_slot[t,j],:], acc) for j = 0..k-1 in order, skipping
 * pairs whose slot is outside [0, rows).  No renormalisation after drops.
 * Requires H % 8 == 0. */
MOE_API moe_status moe_combine(const moe_problem *problem, const void *expert_out,
                       const float *gates, const int32_t *pair_slot, void *out,
                       moe_stream_t stream);

/* The combine fused with the expert-parallel return: instead of shipping
 * the expert outputs back to this rank first, the expert output of local row
 * r of segment s is read straight from rank s's expert-output buffer
 * peer_expert_out[s], at row get_offsets[s] + (r - start of segment s) --
 * where rank s received row r through a fused send (moe_permute_to_peers
 * with put_offsets = get_offsets) and wrote its expert's output.  Segments
 * as in moe_permute_to_peers.  The result is the one moe_combine gives on the
 * returned rows, bit for bit.  DeepSpeed combine docstring; Mojo MAX ep_comm
 * (combine kernels reading the remote ranks' expert outputs).
 *   peer_expert_out  DEVICE array of S device pointers (8-byte aligned
 *                    array) to bf16 [*, H] buffers, each 16-byte aligned
 *                    and readable from this GPU (a peer mapping, or this
 *                    rank's own buffer for its own segment)
 *   get_offsets      DEVICE int64 [S]: first row of this rank's block in
 *                    rank s's buffer (ep.put_offsets)
 *   meta             from moe_dispatch_layout (may be NULL in capacity mode)
 *   gates, pair_slot, out   as in moe_combine
 * Requires H % 8 == 0.  The caller orders the read after the experts'
 * writes (a barrier); the kernel does not wait on other GPUs. */
MOE_API moe_status moe_combine_from_peers(const moe_problem *problem,
                                          const void *const *peer_expert_out,
                                          const int64_t *get_offsets, const uint32_t *meta,
                                          const float *gates, const int32_t *pair_slot,
                                          void *out, moe_stream_t stream);

/* ---- fused SwiGLU + requantisation -----------------------------------------
 * The step after the experts' gate/up projection (Mojo MAX ep_comm:
 * fused_silu_kernel, fused_silu_mx_kernel, fused_silu_nvfp4_kernel,
 * fused_silu_nvfp4_interleaved_kernel, fused_silu_mxfp8_interleaved_kernel,
 * fused_silu_mxfp6_kernel).  The host does not know
 * how many rows each expert received, so the kernel takes the layout's
 * row_src: a row without a routed token (-1) is written as zero bytes and its
 * input is not read.  For the other rows, per column i < I:
 *   y = silu(g) * u,  silu(g) = g / (1 + e^-g)   in fp32
 * where e^x is one fixed fp32 sequence (Cody-Waite reduction with ln 2 split
 * as 0.693145751953125 + 1.42860682e-06, n = rint(x * 1.44269504), the
 * Taylor polynomial of degree 7 in Horner form with fmaf, scaling by 2^n;
 * x < -104 gives 0, x > 88.75 gives inf), and y is quantised:
 *   MOE_QUANT_NVFP4  codes E2M1 [rows, I/2], scales E4M3 [rows, I/16]: the
 *                    rule of moe_permute_quant_nvfp4 (global_scale needed)
 *   MOE_QUANT_MXFP8  codes E4M3 [rows, I], scales E8M0 [rows, I/32]
 *   MOE_QUANT_MXFP4  codes E2M1 [rows, I/2] (element 2m low nibble), scales
 *                    E8M0 [rows, I/32]
 *   MOE_QUANT_BF16   y rounded to bf16 (nearest even) [rows, I]; no scales
 *                    (scales may be NULL)
 *   MOE_QUANT_MXFP6_E2M3, MOE_QUANT_MXFP6_E3M2
 *                    OCP MX FP6 codes (6 bits: sign, exponent, mantissa;
 *                    E2M3 max 7.5, E3M2 max 28) packed densely [rows, 3I/4]:
 *                    code i of a row at bits [6i, 6i+6) of the row's
 *                    little-endian bit stream (4 codes in 3 bytes); scales
 *                    E8M0 [rows, I/32]
 * MX (OCP Microscaling v1.0): per block of 32, X = floor(log2(amax)) - emax
 * (emax 8 for E4M3, 2 for E2M1 and E2M3, 4 for E3M2), scale code
 * clamp(X + 127, 0, 254), code = E(y * 2^-X) rounded to nearest even,
 * saturating; an all-zero block gets scale code 0 and codes 0.
 *   gate_up  bf16 [rows, 2*I], 16-byte aligned: MOE_GATE_UP_SPLIT = columns
 *            [0, I) gate and [I, 2I) up; MOE_GATE_UP_INTERLEAVED = gate at
 *            even and up at odd columns
 *   row_src  int32 [rows] from the layout
 *   codes    16-byte aligned (8 for MXFP6); scales 2-byte aligned (NVFP4);
 *            both fully overwritten
 * Requires I % 32 == 0. */
enum {
  MOE_QUANT_NVFP4 = 0,
  MOE_QUANT_MXFP8 = 1,
  MOE_QUANT_MXFP4 = 2,
  MOE_QUANT_BF16 = 3,
  MOE_QUANT_MXFP6_E2M3 = 4,
  MOE_QUANT_MXFP6_E3M2 = 5
};
enum { MOE_GATE_UP_SPLIT = 0, MOE_GATE_UP_INTERLEAVED = 1 };
MOE_API moe_status moe_swiglu_quant(const moe_problem *problem, int32_t intermediate,
                                    uint32_t format, uint32_t gate_up_layout,
                                    const void *gate_up, const int32_t *row_src,
                                    const float *global_scale, uint8_t *codes,
                                    uint8_t *scales, moe_stream_t stream);

/* ---- backward (training) -------------------------------------------------
 * The gradients of the data movements above, for training with top-k
 * probabilities whose gradient flows back through the combine (NeMo
 * AutoModel token_dispatcher: token_probs [tokens, top_k] and the router
 * gradient layout).  Same problem, maps and conventions as the forward. */

/* Dispatch backward: the dispatch copies token t's row to the rows of its
 * pairs, so grad_hidden[t,:] = bf16_rne(sum over j of grad_out[slot(t,j),:])
 * in fp32 with j in order, pairs whose slot is outside [0, rows) skipped.
 *   grad_out     bf16 [rows, H], 16-byte aligned
 *   pair_slot    int32 [N, k] from the layout
 *   grad_hidden  bf16 [N, H], 16-byte aligned, fully overwritten
 * Requires H % 8 == 0. */
MOE_API moe_status moe_permute_backward(const moe_problem *problem, const void *grad_out,
                                        const int32_t *pair_slot, void *grad_hidden,
                                        moe_stream_t stream);

/* Combine backward: y[t] = sum_j w[t,j] * x[slot(t,j)] (DeepSpeed combine),
 * so for every pair with a row
 *   grad_expert_out[slot(t,j),:] = bf16_rne(w[t,j] * grad_y[t,:])  (fp32 product)
 *   grad_gates[t,j] = <grad_y[t,:], expert_out[slot(t,j),:]>         (fp32)
 * grad_gates is 0 for a pair without a row, and rows whose row_src is -1
 * get zeros.  The dot product is accumulated in fp32 in a fixed order
 * (deterministic): each of 32 lanes sums its elements in order, then a
 * butterfly over the lanes; it is within 2^-24 * (H/32 + 8) * sum|g*x| of
 * the exact value.
 *   grad_y           bf16 [N, H], 16-byte aligned
 *   expert_out       bf16 [rows, H], 16-byte aligned (the forward input)
 *   gates            fp32 [N, k];  pair_slot int32 [N, k];  row_src int32 [rows]
 *   grad_expert_out  bf16 [rows, H], 16-byte aligned, fully overwritten
 *   grad_gates       fp32 [N, k], fully overwritten
 * Requires H % 8 == 0. */
MOE_API moe_status moe_combine_backward(const moe_problem *problem, const void *grad_y,
                                        const void *expert_out, const float *gates,
                                        const int32_t *pair_slot, const int32_t *row_src,
                                        void *grad_expert_out, float *grad_gates,
                                        moe_stream_t stream);

/* Device index checks.  A build with -DMOE_DEBUG_CHECKS
 * (`python -m combine_topk_ids_scan_b200.build --debug`, libmoedc_debug.so)
 * checks every computed row index and block-scale offset in its kernels
 * before use; an out-of-range one is skipped and recorded (no trap).  Returns
 * the OR of the bits recorded on the current device since the last reset
 * (1 layout row, 2 permute destination row, 4 atom-layout scale offset,
 * 8 combine source row, 16 SwiGLU row; 0 = none), zeroing them when `reset`
 * is non-zero; synchronises with the device.  Returns -1 from a build
 * without the checks (no CUDA call is made then). */
MOE_API int64_t moe_debug_violations(int reset);

/* Per-CTA trace records.  A build with -DMOE_TRACE
 * (`python -m combine_topk_ids_scan_b200.build --trace`, libmoedc_trace.so)
 * has every CTA of every library kernel append one record to the buffer
 * attached with moe_trace_attach: the CTA's start and end on the GPU's
 * global nanosecond timer, the launch it belongs to, its block index and the
 * SM it ran on -- the per-CTA timeline of a step, kernel by kernel (the
 * pages' Mojo ep_comm DispatchTraceSink; NullDispatchTrace, the sink that
 * discards events, is the normal build, whose kernels hold no trace code).
 * Tracing costs one atomic add, one barrier and a 32-byte record per CTA
 * and one atomic max per warp. */
typedef struct moe_trace_record {
  uint64_t start_ns; /* %globaltimer when the CTA started (for a kernel that
                        overlaps its predecessor, before it waits for it)   */
  uint64_t end_ns;   /* %globaltimer when the CTA's last warp finished      */
  uint64_t grid;     /* %gridid, shared by the CTAs of a launch (replays of
                        a captured CUDA graph reuse their kernel node's
                        value; a later replay's CTAs start after the
                        earlier one's have finished)                        */
  uint32_t block;    /* blockIdx.x                                          */
  uint16_t smid;     /* the SM the CTA ran on                               */
  uint8_t kernel;    /* moe_trace_kernel                                    */
  uint8_t variant;   /* the kernel's compile-time variant (below), else 0   */
} moe_trace_record;  /* 32 bytes */

/* moe_trace_record.kernel, with the variant each one records. */
typedef enum moe_trace_kernel {
  MOE_TRACE_LAYOUT_SINGLE = 1,         /* one-CTA layout; variant: pair rounds     */
  MOE_TRACE_LAYOUT_CLUSTER = 2,        /* cluster layout; variant: pair rounds     */
  MOE_TRACE_LAYOUT_LOOKBACK = 3,       /* cooperative look-back layout             */
  MOE_TRACE_LAYOUT_SCAN = 4,           /* two-pass layout, scan kernel             */
  MOE_TRACE_LAYOUT_EMIT = 5,           /* two-pass layout, emit kernel             */
  MOE_TRACE_PERMUTE_BF16 = 6,          /* moe_permute                              */
  MOE_TRACE_PERMUTE_FP8 = 7,           /* moe_permute_quant_fp8                    */
  MOE_TRACE_PERMUTE_NVFP4 = 8,         /* variant: 1 scales stored in the atom
                                          layout, 0 linear (final, or converted
                                          by MOE_TRACE_SCALES_TO_ATOMS)            */
  MOE_TRACE_PERMUTE_MXFP4 = 9,         /* variant as MOE_TRACE_PERMUTE_NVFP4       */
  MOE_TRACE_SCALES_TO_ATOMS = 10,      /* variant: 1 with 16-byte vectors          */
  MOE_TRACE_PERMUTE_PREMULTIPLIED = 11,
  MOE_TRACE_PERMUTE_TO_PEERS = 12,
  MOE_TRACE_COMBINE = 13,              /* variant: the largest top_k it handles    */
  MOE_TRACE_PERMUTE_BACKWARD = 14,     /* variant as MOE_TRACE_COMBINE             */
  MOE_TRACE_COMBINE_BACKWARD = 15,     /* variant as MOE_TRACE_COMBINE             */
  MOE_TRACE_SWIGLU_SPLIT = 16,         /* variant: the MOE_QUANT_* format          */
  MOE_TRACE_SWIGLU_QUANT = 17,         /* variant: the MOE_QUANT_* format          */
  MOE_TRACE_PERMUTE_FP8_TO_PEERS = 18,
  MOE_TRACE_PERMUTE_NVFP4_TO_PEERS = 19,
  MOE_TRACE_COMBINE_FROM_PEERS = 20    /* variant as MOE_TRACE_COMBINE             */
} moe_trace_kernel;

/* Attach the trace record buffer (the build with -DMOE_TRACE): the kernels
 * of every later call on `stream` append one record per CTA.
 *   records   device array of `capacity` records, or NULL to stop tracing
 *   count     device uint32, zeroed by the caller; each CTA adds 1 and
 *             writes records[old value] if that is below `capacity`, so a
 *             count above capacity tells how many records were dropped
 * The attachment is a host-to-device copy from pageable memory enqueued on
 * `stream` (so not a call to make inside a CUDA graph capture; kernels
 * enqueued on other streams see it in no defined order) and lasts until the
 * next call; captured graphs of library calls record when replayed.  The
 * caller owns both buffers and keeps them alive while traced kernels run.
 * Returns MOE_ERR_NOT_BUILT, making no CUDA call, from a build without
 * -DMOE_TRACE; MOE_ERR_INVALID_ARG for records without count, misaligned
 * pointers (records 8 bytes, count 4) or capacity 0 with records. */
MOE_API moe_status moe_trace_attach(moe_trace_record *records, uint32_t capacity,
                                    uint32_t *count, moe_stream_t stream);

/* Static description of a moe_status value. */
MOE_API const char *moe_status_string(moe_status status);

/* Library version string. */
MOE_API const char *moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_DC_H */
