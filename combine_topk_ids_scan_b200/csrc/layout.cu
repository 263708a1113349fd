// layout.cu -- dispatch layout: a stable counting sort of the (token, k)
// pairs by expert.
//
// Scan tiles.  The pairs are cut into tiles of 4096 consecutive pairs; a CTA
// takes the next tile from an atomic ticket, so tiles start in order.  Each of
// its 16 warps owns 256 consecutive pairs and walks them in 8 rounds of 32.
// In a round the warp aggregates its lanes per expert in shared memory: each
// lane ORs its bit into the warp's mask word for its expert, reads the mask
// back (its peers), takes its rank from the popcount of lower peers, and the
// highest peer adds the group's size to the warp's private histogram and
// clears the mask (ranks are in pair order; measured on B200 about 4x cheaper
// per round than __match_any_sync and 2x cheaper than one ballot per id bit).  A scan over the 16 warp histograms gives every
// warp its per-expert base inside the tile, and the tiles chain their
// per-expert counts with a single-pass decoupled look-back (one 64-bit word
// per (tile, expert): flag in the high half, count in the low half; a window
// of predecessors is read per poll), which gives each tile its exclusive
// per-expert prefix.  A pair's rank among all earlier pairs of its expert is
// then prefix + warp base + in-warp rank: stable by (token, k) by
// construction, and independent of scheduling.
//
// Each tile stores its pairs' ranks in pair_slot, and the last tile the
// per-expert totals.  The emit step then scans the totals into expert start
// rows (in shared memory, per CTA) and turns ranks into rows: pair_slot,
// row_src, drop_mask, padding rows, counts and the [4,S] table; the last CTA
// to finish returns the workspace to zero and publishes the status word.
// One-launch path: a cooperative grid of up to one CTA per SM; the first T
// CTAs scan the T tiles, then every CTA waits (bounded) until all tiles are
// done and runs the emit step over its share of the pairs, so the scattered
// row_src stores are spread over all SMs.  Two-kernel path (any size): a scan
// kernel of T CTAs, then an emit kernel.
//
// Layout definitions: NKI "Permute A2AV Kernel API Reference" (permute_a2av
// packed_source_indices, send_counts, recv_capacity, [4, EP] metadata in
// elements); DeepSpeed capacity dispatch ([e, c, m] buffer); NeMo AutoModel
// token_dispatcher (-1 ids are masked; tokens per expert).
#include <cooperative_groups.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "trace.cuh"

namespace moe {

namespace {

constexpr int kScanThreads = 512;
constexpr int kScanWarps = kScanThreads / kWarp;        // 16
constexpr int kScanRounds = 8;                          // pairs per lane
constexpr int kTilePairs = kScanThreads * kScanRounds;  // 4096
constexpr uint64_t kFlagAggregate = 1ull;
constexpr uint64_t kFlagInclusive = 2ull;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // every bounded wait: 1 s
constexpr int kLookWindow = 8;                    // predecessor tiles per poll
constexpr int kFusedMaxTiles = 128;               // last CTA clears <= 128*E words
constexpr int64_t kClusterMaxRows = 1 << 18;      // cluster path: rows per launch
constexpr int kClusterMax = 16;                   // largest cluster the path uses
constexpr int64_t kSingleMaxRows = 1 << 14;       // single-CTA path: rows per launch

constexpr int kEmitThreads = 256;

// control words at the start of the workspace
enum { kCtrlTicket = 0, kCtrlDone = 1, kCtrlStatus = 2, kCtrlTilesDone = 3 };

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// dynamic shared memory of a scan CTA: per-warp counts (u16), per-warp lane
// masks (u32), tile prefix (u32)
__host__ __device__ inline size_t scan_smem_bytes(int E) {
  return align_up((size_t)kScanWarps * E * sizeof(uint16_t), 16) +
         (size_t)kScanWarps * E * sizeof(uint32_t) + align_up((size_t)E * sizeof(uint32_t), 16);
}

struct ScanSmem {
  uint16_t *wcnt;        // [warps][E] counts, then warp bases
  uint32_t *wmask;       // [warps][E] lane masks of the current round, then
                         // the cluster kernel's prefixes, start rows, kept rows
  uint32_t *tile_prefix; // [E] tile aggregate, then tile exclusive prefix
};

__device__ __forceinline__ ScanSmem scan_smem(uint8_t *smem, int32_t E) {
  ScanSmem m;
  m.wcnt = reinterpret_cast<uint16_t *>(smem);
  m.wmask = reinterpret_cast<uint32_t *>(smem + align_up((size_t)kScanWarps * E * 2, 16));
  m.tile_prefix = m.wmask + (size_t)kScanWarps * E;
  return m;
}

// Bounded wait helper: true while the deadline (set on first call) has not
// passed.
__device__ __forceinline__ bool keep_waiting(uint64_t &deadline) {
  const uint64_t now = globaltimer_ns();
  if (deadline == 0) {
    deadline = now + kWaitLimitNs;
    return true;
  }
  return now <= deadline;
}

// Per-CTA state of one scan tile of ROUNDS * 512 pairs (each warp owns
// ROUNDS * 32 consecutive pairs).  pk[r] packs the lane's r-th pair: expert
// id in the low 16 bits (0xFFFF: no expert), rank inside the warp's pairs in
// the high 16 bits.
template <int ROUNDS>
struct TileScanT {
  int tile;
  uint32_t pk[ROUNDS];
  int64_t base;  // first pair of this warp
  __device__ __forceinline__ int32_t expert(int r) const {
    const uint32_t e = pk[r] & 0xFFFFu;
    return e == 0xFFFFu ? -1 : (int32_t)e;
  }
  __device__ __forceinline__ uint32_t rank(int r) const { return pk[r] >> 16; }
};
using TileScan = TileScanT<kScanRounds>;

// Phases 1-2 of tile ts.tile (set by the caller): in-warp stable ranks and
// per-warp histograms, then per expert the exclusive scan over the warps
// (warp bases, left in wcnt; at most 16 * ROUNDS * 32 <= 65535) and the tile
// aggregate (left in tile_prefix).  ORs MOE_STATUS_ID_RANGE into *s_status.
// Called by all threads of the block; ends with a block barrier.
template <int ROUNDS>
__device__ void rank_tile(TileScanT<ROUNDS> &ts, const int32_t *__restrict__ ids, int64_t P,
                          int32_t E, const ScanSmem &sm, uint32_t *s_status) {
  const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
  uint16_t *wcnt = sm.wcnt;
  uint32_t *tile_prefix = sm.tile_prefix;
  // the tile's ids first: their loads are in flight while shared memory is
  // cleared
  ts.base = (int64_t)ts.tile * (kScanThreads * ROUNDS) + (int64_t)warp * (kWarp * ROUNDS);
  int32_t ex[ROUNDS];
#pragma unroll
  for (int r = 0; r < ROUNDS; ++r) {
    const int64_t p = ts.base + r * kWarp + lane;
    ex[r] = p < P ? __ldg(ids + p) : -1;
  }
  {
    // the per-warp counts and lane masks start at zero: 16 * E * (2 + 4)
    // bytes, contiguous from the (16-byte aligned) start of shared memory,
    // cleared with 16-byte stores
    uint4 *z = reinterpret_cast<uint4 *>(wcnt);
    constexpr int kBytesPerExpert = kScanWarps * (int)(sizeof(uint16_t) + sizeof(uint32_t));
    for (int i = tid; i < E * kBytesPerExpert / 16; i += kScanThreads)
      z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  // ---- 1. per-warp stable ranks and histograms
  bool bad_id = false;
  uint16_t *my_cnt = wcnt + (size_t)warp * E;
  uint32_t *my_mask = sm.wmask + (size_t)warp * E;
  // per round, the lanes holding the same expert OR their bits into its mask
  // word (a shared-memory atomic: on B200 the layout ran 12.4 -> 15.4 us at
  // the metric shape with __match_any_sync instead); the highest of them
  // advances the warp's count and clears the word
#pragma unroll
  for (int r = 0; r < ROUNDS; ++r) {
    const int32_t e = ex[r];
    const bool valid = (uint32_t)e < (uint32_t)E;
    bad_id |= (!valid && e != -1);
    if (valid) atomicOr(&my_mask[e], 1u << lane);
    __syncwarp();
    uint32_t peers = 0, before = 0;
    if (valid) {
      peers = my_mask[e];
      before = my_cnt[e];
    }
    __syncwarp();
    uint32_t rank = 0;
    if (valid) {
      rank = before + __popc(peers & lanemask_lt());
      if (lane == 31 - __clz(peers)) {
        my_cnt[e] = (uint16_t)(before + __popc(peers));
        my_mask[e] = 0;
      }
    }
    __syncwarp();
    ts.pk[r] = (rank << 16) | (valid ? (uint32_t)e : 0xFFFFu);
  }
  if (__any_sync(0xFFFFFFFFu, bad_id) && lane == 0) atomicOr(s_status, MOE_STATUS_ID_RANGE);
  __syncthreads();

  // ---- 2. per expert: exclusive scan over the warps, tile aggregate (the
  // 16 counts are loaded before any base is stored, so the loads are in
  // flight together instead of each waiting behind the previous store)
  for (int e = tid; e < E; e += kScanThreads) {
    uint32_t c[kScanWarps];
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) c[w] = wcnt[w * E + e];
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) {
      wcnt[w * E + e] = (uint16_t)run;
      run += c[w];
    }
    tile_prefix[e] = run;
  }
  __syncthreads();
}

// Phases 1-3 of a tile: in-warp ranks, warp bases (left in wcnt), tile
// exclusive prefix per expert (left in tile_prefix); the last tile also
// stores the per-expert totals.  Returns false when the ticket is past the
// last tile (a workspace that was not zero-filled).
__device__ bool scan_tile(TileScan &ts, const int32_t *__restrict__ ids, int64_t P, int32_t E,
                          int32_t num_tiles, uint32_t flags, uint32_t *ctrl, uint64_t *tiles,
                          int32_t *totals, const ScanSmem &sm, int *s_tile, uint32_t *s_status) {
  const int tid = threadIdx.x;
  uint32_t *tile_prefix = sm.tile_prefix;
  if (tid == 0) {
    *s_tile = (int)atomicAdd(&ctrl[kCtrlTicket], 1u);
    *s_status = 0;
  }
  __syncthreads();
  if (*s_tile >= num_tiles) return false;
  ts.tile = *s_tile;
  rank_tile<kScanRounds>(ts, ids, P, E, sm, s_status);

  // ---- 3. decoupled look-back across tiles, one chain per expert
  const int tile = ts.tile;
  const bool withhold = (flags & MOE_FLAG_TEST_STALL_SCAN) && tile == 0;
  bool timed_out = false;
  uint64_t deadline = 0;
  for (int e = tid; e < E; e += kScanThreads) {
    const uint32_t agg = tile_prefix[e];
    uint32_t excl = 0;
    if (tile == 0) {
      if (!withhold) st_relaxed_gpu_u64(&tiles[e], (kFlagInclusive << 32) | agg);
    } else {
      st_relaxed_gpu_u64(&tiles[(size_t)tile * E + e], (kFlagAggregate << 32) | agg);
      // Read a window of predecessors per poll (independent loads: one L2
      // round trip), add aggregates in order until an inclusive prefix ends
      // the chain or an unpublished tile makes us poll again.
      int look = tile - 1;
      while (look >= 0) {
        uint64_t v[kLookWindow];
#pragma unroll
        for (int i = 0; i < kLookWindow; ++i)
          v[i] = look - i >= 0 ? ld_relaxed_gpu_u64(&tiles[(size_t)(look - i) * E + e])
                               : (kFlagInclusive << 32);
        bool stop = false, done = false;
        int advanced = 0;
#pragma unroll
        for (int i = 0; i < kLookWindow; ++i) {
          if (!stop) {
            const uint64_t f = v[i] >> 32;
            if (f == 0) {
              stop = true;
            } else {
              excl += (uint32_t)v[i];
              ++advanced;
              if (f == kFlagInclusive) stop = done = true;
            }
          }
        }
        if (done) break;
        look -= advanced;
        if (advanced < kLookWindow) {
          // tile `look` has not published: it holds an earlier ticket, so it
          // is running; wait for it, but never longer than the limit
          if (!keep_waiting(deadline)) {
            timed_out = true;
            break;
          }
          __nanosleep(32);
        }
      }
      st_relaxed_gpu_u64(&tiles[(size_t)tile * E + e], (kFlagInclusive << 32) | (excl + agg));
    }
    tile_prefix[e] = excl;
    if (tile == num_tiles - 1) totals[e] = (int32_t)(excl + agg);
  }
  if (timed_out) atomicOr(s_status, MOE_STATUS_TIMEOUT);
  __syncthreads();
  return true;
}

// Rank of the lane's r-th pair among all earlier pairs of its expert.
__device__ __forceinline__ int32_t pair_rank_of(const TileScan &ts, int r, const uint16_t *wcnt,
                                                const uint32_t *tile_prefix, int32_t E) {
  const int warp = threadIdx.x / kWarp;
  const int32_t e = ts.expert(r);
  return (int32_t)(tile_prefix[e] + wcnt[(size_t)warp * E + e] + ts.rank(r));
}

// Row of a pair from its expert and rank; -1 with `dropped` set when it gets
// none.  Sets MOE_STATUS_CAPACITY bits for packed overflow.
__device__ __forceinline__ int32_t row_of(int32_t e, int32_t r, const int32_t *s_off, int64_t C,
                                          int32_t Ce, bool capacity, uint8_t &dropped,
                                          uint32_t &bits) {
  dropped = 0;
  if (capacity) {
    if (r >= 0 && r < Ce) return e * Ce + r;
    dropped = 1;
    return -1;
  }
  const int64_t row = (int64_t)s_off[e] + r;
  if (r >= 0 && row >= 0 && row < C) return (int32_t)row;
  dropped = 1;
  bits |= MOE_STATUS_CAPACITY;
  return -1;
}

// Block-wide exclusive scan of n <= PER * THREADS values in place; returns
// the total.  Called by all threads of the block.
template <int THREADS, int PER>
__device__ int32_t block_exclusive_scan(int32_t *v, int n) {
  __shared__ int32_t warp_sums[THREADS / kWarp];
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  int32_t local[PER];
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int idx = tid * PER + i;
    local[i] = idx < n ? v[idx] : 0;
    sum += local[i];
  }
  int32_t incl = sum;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == kWarp - 1) warp_sums[warp] = incl;
  __syncthreads();
  int32_t warp_base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < THREADS / kWarp; ++w) {
    if (w < warp) warp_base += warp_sums[w];
    total += warp_sums[w];
  }
  int32_t run = warp_base + incl - sum;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int idx = tid * PER + i;
    if (idx < n) v[idx] = run;
    run += local[i];
  }
  __syncthreads();
  return total;
}

// Expert start rows s_off[E+1] and kept rows s_kept[E] from the totals
// (packed mode: each expert's block is its count rounded up to `pad`).
template <int THREADS, bool SMEM_TOTALS = false>
__device__ void expert_offsets_from_totals(const int32_t *totals, bool have_totals, int32_t E,
                                           int32_t Ce, int32_t pad, int32_t *s_off,
                                           int32_t *s_kept) {
  const bool capacity = Ce > 0;
  for (int e = threadIdx.x; e < E; e += THREADS) {
    const int32_t t = !have_totals ? 0 : SMEM_TOTALS ? totals[e] : __ldcg(totals + e);
    s_kept[e] = capacity ? min(t, Ce) : t;
    s_off[e] = capacity ? e * Ce : (pad > 1 ? (t + pad - 1) / pad * pad : t);
  }
  if (capacity) {
    if (threadIdx.x == 0) s_off[E] = E * Ce;
    __syncthreads();
    return;
  }
  __syncthreads();
  const int32_t total = block_exclusive_scan<THREADS, (MOE_MAX_EXPERTS + THREADS - 1) / THREADS>(
      s_off, E);
  if (threadIdx.x == 0) s_off[E] = total;
  __syncthreads();
}

// Padding rows of [r0, rows) in steps of `stride` and counts/offsets/meta
// when `write_meta`.
template <int THREADS>
__device__ void emit_common(int64_t r0, int64_t stride, int64_t rows, int32_t E, int32_t S,
                            int32_t Ce, int32_t pad_multiple, int32_t H, const int32_t *s_off,
                            const int32_t *s_kept, int32_t *__restrict__ row_src,
                            bool write_meta, int32_t *__restrict__ expert_counts,
                            int32_t *__restrict__ expert_offsets, uint32_t *__restrict__ meta) {
  const bool capacity = Ce > 0;
  for (int64_t r = r0; r < rows; r += stride) {
    bool pad;
    if (capacity) {
      const int32_t r32 = (int32_t)r;  // rows < 2^31 (host check)
      pad = r32 % Ce >= s_kept[r32 / Ce];
    } else if (r >= (int64_t)s_off[E]) {
      pad = true;
    } else if (pad_multiple > 1) {
      // the expert whose block holds r: last e with s_off[e] <= r
      int lo = 0, hi = E - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if ((int64_t)s_off[mid] <= r) lo = mid;
        else hi = mid - 1;
      }
      pad = r - s_off[lo] >= s_kept[lo];
    } else {
      pad = false;
    }
    if (pad) row_src[r] = -1;
  }
  if (write_meta) {
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += THREADS) expert_counts[e] = s_kept[e];
    for (int e = tid; e <= E; e += THREADS) expert_offsets[e] = s_off[e];
    const int32_t L = E / S;
    // one warp per segment: capacity mode sums the segment's kept rows over
    // its L experts with the lanes and a shuffle reduction (packed mode reads
    // the difference of two start rows)
    const int lane = tid % kWarp;
    for (int s = tid / kWarp; s < S; s += THREADS / kWarp) {
      int64_t seg_rows = 0;
      if (capacity) {
        for (int e = s * L + lane; e < (s + 1) * L; e += kWarp) seg_rows += s_kept[e];
#pragma unroll
        for (int o = kWarp / 2; o > 0; o >>= 1)
          seg_rows += __shfl_xor_sync(0xFFFFFFFFu, seg_rows, o);
      } else {
        seg_rows = (int64_t)s_off[(s + 1) * L] - s_off[s * L];  // blocks incl. padding
      }
      if (lane == 0) {
        const uint32_t count_el = (uint32_t)(seg_rows * H);
        const uint32_t displ_el = capacity ? (uint32_t)((int64_t)s * L * Ce * H)
                                           : (uint32_t)((int64_t)s_off[s * L] * H);
        meta[0 * S + s] = count_el;
        meta[1 * S + s] = displ_el;
        meta[2 * S + s] = count_el;
        meta[3 * S + s] = displ_el;
      }
    }
  }
}

__device__ uint32_t duplicate_bits(const int32_t *__restrict__ ids, int64_t t0, int64_t t1,
                                   int64_t tstride, int32_t k, int32_t E) {
  uint32_t bits = 0;
  for (int64_t t = t0; t < t1; t += tstride) {
    const int32_t *row = ids + t * k;
    for (int a = 0; a < k; ++a) {
      const int32_t ea = __ldg(row + a);
      if ((uint32_t)ea >= (uint32_t)E) continue;
      for (int b = a + 1; b < k; ++b)
        if (__ldg(row + b) == ea) bits |= MOE_STATUS_DUP_ID;
    }
  }
  return bits;
}

// The last block to arrive publishes the status word and returns the
// workspace (tile states, totals, control words) to zero.  Called by all
// threads of every block, last thing in the kernel.  Every block arrives
// after all of its own workspace stores, so the last block runs after every
// store of the launch.  n_states tile states are cleared here always, and
// n_states_on_timeout when a bounded wait gave up: in the one-launch kernel
// a tile whose look-back timed out may publish its state after the other
// blocks, whose grid-wide wait also timed out, cleared the states.
template <int THREADS>
__device__ void finish_and_clean(uint32_t bits, uint32_t *s_status, uint32_t *ctrl,
                                 int32_t *totals, uint64_t *tiles, int64_t n_states,
                                 int64_t n_states_on_timeout, int32_t E, uint32_t *status_out,
                                 uint32_t n_blocks) {
  __shared__ bool s_last;
  __shared__ uint32_t s_final;
  if (bits) atomicOr(s_status, bits);
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*s_status) atomicOr(&ctrl[kCtrlStatus], *s_status);
    __threadfence();
    s_last = atomicAdd(&ctrl[kCtrlDone], 1u) == n_blocks - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) s_final = atomicExch(&ctrl[kCtrlStatus], 0u);
  __syncthreads();
  const int64_t n = (s_final & MOE_STATUS_TIMEOUT) ? max(n_states, n_states_on_timeout)
                                                   : n_states;
  for (int64_t i = threadIdx.x; i < n; i += THREADS) tiles[i] = 0;
  for (int e = threadIdx.x; e < E; e += THREADS) totals[e] = 0;
  if (threadIdx.x == 0) {
    *status_out = s_final;
    ctrl[kCtrlTicket] = 0;
    ctrl[kCtrlTilesDone] = 0;
    atomicExch(&ctrl[kCtrlDone], 0u);
  }
}

// ------------------------------------------------------------ kernels
struct LayoutArgs {
  const int32_t *ids;
  int64_t P;
  int32_t N, k, E, S, Ce, H, pad;
  int64_t C, rows;
  uint32_t flags;
  int32_t num_tiles;
  uint32_t *ctrl;
  int32_t *totals;
  uint64_t *tiles;
  int32_t *expert_counts, *expert_offsets;
  uint32_t *meta;
  int32_t *row_src, *pair_slot;
  uint8_t *drop_mask;
  uint32_t *status_out;
};

// Scan step of one CTA: if it draws a tile, rank the tile's pairs and store
// the ranks in pair_slot (the last tile also stores the totals).
template <bool COUNT_DONE>
__device__ void scan_step(const LayoutArgs &a, uint8_t *smem, uint32_t *s_status) {
  __shared__ int s_tile;
  const ScanSmem sm = scan_smem(smem, a.E);
  TileScan ts;
  if (!scan_tile(ts, a.ids, a.P, a.E, a.num_tiles, a.flags, a.ctrl, a.tiles, a.totals, sm,
                 &s_tile, s_status))
    return;
  const int lane = threadIdx.x % kWarp;
#pragma unroll
  for (int r = 0; r < kScanRounds; ++r) {
    const int64_t p = ts.base + r * kWarp + lane;
    if (p < a.P)
      a.pair_slot[p] = ts.expert(r) >= 0 ? pair_rank_of(ts, r, sm.wcnt, sm.tile_prefix, a.E) : -1;
  }
  if (COUNT_DONE) {
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      atomicAdd(&a.ctrl[kCtrlTilesDone], 1u);
    }
  }
}

// Emit step: ranks -> rows for the pairs [gtid, P) in steps of gstride, the
// padding rows, counts / offsets / meta (block 0), the duplicate check, then
// the last block cleans up.  n_states_on_timeout: tile states the last block
// clears when a bounded wait gave up.
template <int THREADS>
__device__ void emit_step(const LayoutArgs &a, int64_t gtid, int64_t gstride,
                          uint32_t *s_status, int64_t n_states_on_timeout) {
  __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int32_t s_kept[MOE_MAX_EXPERTS];
  expert_offsets_from_totals<THREADS>(a.totals, a.num_tiles > 0, a.E, a.Ce, a.pad, s_off,
                                      s_kept);
  const bool capacity = a.Ce > 0;
  uint32_t bits = 0;
  for (int64_t p = gtid; p < a.P; p += gstride) {
    const int32_t e = __ldg(a.ids + p);
    int32_t slot = -1;
    uint8_t dropped = 0;
    if ((uint32_t)e < (uint32_t)a.E)
      slot = row_of(e, __ldcg(a.pair_slot + p), s_off, a.C, a.Ce, capacity, dropped, bits);
    a.pair_slot[p] = slot;
    if (a.drop_mask) a.drop_mask[p] = dropped;
    if (slot >= 0 && MOE_IN_RANGE(slot, a.rows, kDbgLayoutRow)) a.row_src[slot] = (int32_t)p / a.k;
  }
  emit_common<THREADS>(gtid, gstride, a.rows, a.E, a.S, a.Ce, a.pad, a.H, s_off, s_kept,
                       a.row_src, blockIdx.x == 0, a.expert_counts, a.expert_offsets, a.meta);
  if (a.flags & MOE_FLAG_CHECK_DUPLICATES)
    bits |= duplicate_bits(a.ids, gtid, a.N, gstride, a.k, a.E);
  finish_and_clean<THREADS>(bits, s_status, a.ctrl, a.totals, a.tiles, 0, n_states_on_timeout,
                            a.E, a.status_out, (uint32_t)gridDim.x);
}

// One cooperative launch: scan (first T CTAs), grid-wide wait, emit (all).
__global__ void __launch_bounds__(kScanThreads, 1) layout_fused_kernel(LayoutArgs a) {
  MOE_TRACE_CTA(MOE_TRACE_LAYOUT_LOOKBACK, 0);
  allow_dependents();  // the next kernel may be scheduled; it waits for this grid
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t s_status;
  if (threadIdx.x == 0) s_status = 0;
  __syncthreads();
  scan_step<true>(a, smem, &s_status);
  // wait (bounded) until every tile has stored its ranks and the totals
  if (threadIdx.x == 0) {
    uint64_t deadline = 0;
    while (ld_acquire_gpu_u32(&a.ctrl[kCtrlTilesDone]) < (uint32_t)a.num_tiles) {
      if (!keep_waiting(deadline)) {
        atomicOr(&s_status, MOE_STATUS_TIMEOUT);
        break;
      }
      __nanosleep(20);
    }
  }
  __syncthreads();
  const int64_t gtid = (int64_t)blockIdx.x * kScanThreads + threadIdx.x;
  const int64_t gstride = (int64_t)gridDim.x * kScanThreads;
  // every look-back has finished (unless a wait timed out, see
  // finish_and_clean): the tile states can be cleared by everyone
  for (int64_t i = gtid; i < (int64_t)a.num_tiles * a.E; i += gstride) a.tiles[i] = 0;
  emit_step<kScanThreads>(a, gtid, gstride, &s_status, (int64_t)a.num_tiles * a.E);
}

__global__ void __launch_bounds__(kScanThreads, 1) layout_count_scan_kernel(LayoutArgs a) {
  MOE_TRACE_CTA(MOE_TRACE_LAYOUT_SCAN, 0);
  allow_dependents();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t s_status;
  scan_step<false>(a, smem, &s_status);
  __syncthreads();
  if (threadIdx.x == 0 && s_status) atomicOr(&a.ctrl[kCtrlStatus], s_status);
}

__global__ void __launch_bounds__(kEmitThreads) layout_emit_kernel(LayoutArgs a) {
  MOE_TRACE_CTA(MOE_TRACE_LAYOUT_EMIT, 0);
  allow_dependents();
  grid_dependency_wait();
  __shared__ uint32_t s_status;
  if (threadIdx.x == 0) s_status = 0;
  const int64_t gtid = (int64_t)blockIdx.x * kEmitThreads + threadIdx.x;
  const int64_t gstride = (int64_t)gridDim.x * kEmitThreads;
  // the scan kernel has finished: its tile states can be cleared by everyone
  for (int64_t i = gtid; i < (int64_t)a.num_tiles * a.E; i += gstride) a.tiles[i] = 0;
  emit_step<kEmitThreads>(a, gtid, gstride, &s_status, 0);
}

// One thread-block cluster for the whole layout (P <= cluster size * ROUNDS
// * 512 pairs).  CTA c of the cluster ranks tile c (phases 1-2 above), then
// the CTAs exchange their per-expert tile aggregates through distributed
// shared memory: after a cluster barrier each CTA reads every tile's
// aggregate, which gives its own exclusive prefix (tiles before it) and the
// totals (all tiles) at once -- no look-back chain, no grid-wide wait, no
// workspace.  Each CTA then turns its pairs' ranks (still in registers) into
// rows, writes its share of the padding rows, and ORs its status bits into
// CTA 0's shared word; a second cluster barrier keeps every CTA's shared
// memory alive until the others have read it, and CTA 0 stores the status.
// The barriers are hardware cluster barriers over co-scheduled CTAs: there
// is no spin loop and nothing to time out.  SINGLE: the problem fits one
// tile, the kernel is one ordinary CTA, and block barriers with local reads
// replace the cluster barriers (with their release / acquire fences) and the
// remote reads.
template <int ROUNDS, bool SINGLE>
__global__ void __launch_bounds__(kScanThreads, 1) layout_cluster_kernel(LayoutArgs a) {
  MOE_TRACE_CTA(SINGLE ? MOE_TRACE_LAYOUT_SINGLE : MOE_TRACE_LAYOUT_CLUSTER, ROUNDS);
  namespace cg = cooperative_groups;
  allow_dependents();  // the next kernel may be scheduled; it waits for this grid
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t s_status;
  const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
  const int c = SINGLE ? 0 : (int)cg::this_cluster().block_rank();
  const int nc = SINGLE ? 1 : (int)cg::this_cluster().num_blocks();
  const int32_t E = a.E;
  const ScanSmem sm = scan_smem(smem, E);
  if (tid == 0) s_status = 0;
  TileScanT<ROUNDS> ts;
  ts.tile = c;
  rank_tile<ROUNDS>(ts, a.ids, a.P, E, sm, &s_status);  // ends with a block barrier
  if constexpr (!SINGLE) cg::this_cluster().sync();  // every tile's aggregate is visible

  // the lane-mask words are free now: exclusive prefix, start rows, kept rows
  int32_t *s_excl = reinterpret_cast<int32_t *>(sm.wmask);
  int32_t *s_off = s_excl + E;       // [E + 1]
  int32_t *s_kept = s_off + E + 1;   // [E]: the totals, then the kept rows
  if constexpr (SINGLE) {
    // one tile: its aggregate is the totals, and no tile precedes it
    expert_offsets_from_totals<kScanThreads, true>(
        reinterpret_cast<const int32_t *>(sm.tile_prefix), true, E, a.Ce, a.pad, s_off, s_kept);
  } else {
    for (int e = tid; e < E; e += kScanThreads) {
      // all of the cluster's remote loads in flight at once
      cg::cluster_group cluster = cg::this_cluster();
      uint32_t v[kClusterMax];
#pragma unroll
      for (int q = 0; q < kClusterMax; ++q)
        v[q] = q < nc ? *cluster.map_shared_rank(sm.tile_prefix + e, q) : 0u;
      uint32_t excl = 0, tot = 0;
#pragma unroll
      for (int q = 0; q < kClusterMax; ++q) {
        excl += q < c ? v[q] : 0u;
        tot += v[q];
      }
      s_excl[e] = (int32_t)excl;
      s_kept[e] = (int32_t)tot;
    }
    __syncthreads();
    expert_offsets_from_totals<kScanThreads, true>(s_kept, true, E, a.Ce, a.pad, s_off, s_kept);
  }

  // ranks -> rows for this tile's pairs
  const bool capacity = a.Ce > 0;
  uint32_t bits = 0;
#pragma unroll
  for (int r = 0; r < ROUNDS; ++r) {
    const int64_t p = ts.base + r * kWarp + lane;
    if (p < a.P) {
      const int32_t e = ts.expert(r);
      int32_t slot = -1;
      uint8_t dropped = 0;
      if (e >= 0) {
        const int32_t rank = (SINGLE ? 0 : s_excl[e]) + (int32_t)sm.wcnt[(size_t)warp * E + e] +
                             (int32_t)ts.rank(r);
        slot = row_of(e, rank, s_off, a.C, a.Ce, capacity, dropped, bits);
      }
      a.pair_slot[p] = slot;
      if (a.drop_mask) a.drop_mask[p] = dropped;
      if (slot >= 0 && MOE_IN_RANGE(slot, a.rows, kDbgLayoutRow))
        a.row_src[slot] = (int32_t)(p / a.k);
    }
  }
  const int64_t gtid = (int64_t)c * kScanThreads + tid;
  const int64_t gstride = (int64_t)nc * kScanThreads;
  emit_common<kScanThreads>(gtid, gstride, a.rows, E, a.S, a.Ce, a.pad, a.H, s_off, s_kept,
                            a.row_src, c == 0, a.expert_counts, a.expert_offsets, a.meta);
  if (a.flags & MOE_FLAG_CHECK_DUPLICATES)
    bits |= duplicate_bits(a.ids, gtid, a.N, gstride, a.k, E);
  if (bits) atomicOr(&s_status, bits);
  __syncthreads();
  if constexpr (!SINGLE) {
    cg::cluster_group cluster = cg::this_cluster();
    if (tid == 0 && c != 0 && s_status != 0)
      atomicOr(cluster.map_shared_rank(&s_status, 0), s_status);
    cluster.sync();  // all remote reads and status bits are done
  }
  if (c == 0 && tid == 0) *a.status_out = s_status;
}

// The cluster kernel's instantiations: pairs per lane 1, 2, 4, 8, 16.
constexpr int kClusterRounds[5] = {1, 2, 4, 8, 16};
inline const void *const *cluster_kernels() {
  static const void *const k[5] = {
      (const void *)layout_cluster_kernel<1, false>, (const void *)layout_cluster_kernel<2, false>,
      (const void *)layout_cluster_kernel<4, false>, (const void *)layout_cluster_kernel<8, false>,
      (const void *)layout_cluster_kernel<16, false>};
  return k;
}
// The single-CTA instantiations (one tile of 512, 1024 or 2048 pairs).
constexpr int kSingleRounds[3] = {1, 2, 4};
inline const void *const *single_kernels() {
  static const void *const k[3] = {(const void *)layout_cluster_kernel<1, true>,
                                   (const void *)layout_cluster_kernel<2, true>,
                                   (const void *)layout_cluster_kernel<4, true>};
  return k;
}
struct ClusterKernelList {
  const void *const *begin() const { return cluster_kernels(); }
  const void *const *end() const { return cluster_kernels() + 5; }
};
inline ClusterKernelList cluster_kernel_list() { return {}; }

// Opt the scan kernels in to more than 48 KB of dynamic shared memory, once
// per device.
cudaError_t opt_in_smem() {
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < kMaxDevices && done[dev].load()) return cudaSuccess;
  const int bytes = (int)scan_smem_bytes(MOE_MAX_EXPERTS);
  err = cudaFuncSetAttribute(layout_count_scan_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(layout_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               bytes);
  for (const void *kern : cluster_kernel_list())
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  for (int i = 0; i < 3; ++i)
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(single_kernels()[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 bytes);
  if (err == cudaSuccess && dev < kMaxDevices) done[dev].store(true);
  return err;
}

// Largest cluster of the cluster kernel this device can schedule (16 with
// the non-portable size, else 8, else 0 = no cluster path), queried once per
// device with the largest dynamic shared memory the kernel takes.
int max_cluster_size() {
  static std::atomic<int> cache[kMaxDevices];  // 0 = not queried, else size + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < kMaxDevices) {
    const int v = cache[dev].load();
    if (v > 0) return v - 1;
  }
  if (opt_in_smem() != cudaSuccess) return 0;
  int best = 0;
  const int bytes = (int)scan_smem_bytes(MOE_MAX_EXPERTS);
  for (int size : {16, 8}) {
    bool ok = true;
    for (const void *kern : cluster_kernel_list()) {
      if (size > 8 &&
          cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
              cudaSuccess) {
        ok = false;
        break;
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(size);
      cfg.blockDim = dim3(kScanThreads);
      cfg.dynamicSmemBytes = bytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = size;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1)
        ok = false;
    }
    if (ok) {
      best = size;
      break;
    }
  }
  (void)cudaGetLastError();  // a refused query leaves no sticky error
  if (dev < kMaxDevices) cache[dev].store(best + 1);
  return best;
}

template <int ROUNDS>
cudaError_t launch_cluster_t(const LayoutArgs &a, int nc, size_t smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nc);
  cfg.blockDim = dim3(kScanThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nc;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, layout_cluster_kernel<ROUNDS, false>, a);
}

// One CTA, no cluster (a problem of one tile).
cudaError_t launch_single(int rounds, const LayoutArgs &a, size_t smem, cudaStream_t stream) {
  switch (rounds) {
    case 1: layout_cluster_kernel<1, true><<<1, kScanThreads, smem, stream>>>(a); break;
    case 2: layout_cluster_kernel<2, true><<<1, kScanThreads, smem, stream>>>(a); break;
    default: layout_cluster_kernel<4, true><<<1, kScanThreads, smem, stream>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_cluster(int rounds, const LayoutArgs &a, int nc, size_t smem,
                           cudaStream_t stream) {
  switch (rounds) {
    case 1: return launch_cluster_t<1>(a, nc, smem, stream);
    case 2: return launch_cluster_t<2>(a, nc, smem, stream);
    case 4: return launch_cluster_t<4>(a, nc, smem, stream);
    case 8: return launch_cluster_t<8>(a, nc, smem, stream);
    default: return launch_cluster_t<16>(a, nc, smem, stream);
  }
}

// Largest grid of the fused kernel that is guaranteed co-resident.
int fused_capacity(size_t smem) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layout_fused_kernel, kScanThreads,
                                                    smem) != cudaSuccess)
    return 0;
  return per_sm * device_sm_count();
}

}  // namespace

uint32_t debug_violations_layout(bool reset) { return read_debug_violations(reset); }

#ifdef MOE_TRACE
cudaError_t trace_attach_layout(moe_trace_record *records, uint32_t *count, uint32_t capacity,
                              cudaStream_t stream) {
  return trace_attach_tu(records, count, capacity, stream);
}
#endif

int32_t layout_num_tiles(int64_t P) { return (int32_t)((P + kTilePairs - 1) / kTilePairs); }

size_t layout_workspace_bytes(const Shape &s) {
  const int32_t T = layout_num_tiles(s.P);
  return 256 + align_up((size_t)s.E * sizeof(int32_t), 256) + (size_t)T * s.E * sizeof(uint64_t);
}

LayoutWorkspace layout_workspace_view(const Shape &s, void *workspace) {
  uint8_t *b = static_cast<uint8_t *>(workspace);
  LayoutWorkspace w;
  w.ctrl = reinterpret_cast<uint32_t *>(b);
  w.totals = reinterpret_cast<int32_t *>(b + 256);
  w.tiles = reinterpret_cast<uint64_t *>(b + 256 + align_up((size_t)s.E * sizeof(int32_t), 256));
  w.num_tiles = layout_num_tiles(s.P);
  return w;
}

cudaError_t launch_layout(const Shape &s, const int32_t *ids, int32_t *expert_counts,
                          int32_t *expert_offsets, uint32_t *meta, int32_t *row_src,
                          int32_t *pair_slot, uint8_t *drop_mask, uint32_t *status,
                          const LayoutWorkspace &ws, cudaStream_t stream) {
  LayoutArgs a;
  a.ids = ids;
  a.P = s.P;
  a.N = s.N;
  a.k = s.k;
  a.E = s.E;
  a.S = s.S;
  a.Ce = s.Ce;
  a.H = s.H;
  a.pad = s.pad;
  a.C = s.C;
  a.rows = s.rows;
  a.flags = s.flags;
  a.num_tiles = ws.num_tiles;
  a.ctrl = ws.ctrl;
  a.totals = ws.totals;
  a.tiles = ws.tiles;
  a.expert_counts = expert_counts;
  a.expert_offsets = expert_offsets;
  a.meta = meta;
  a.row_src = row_src;
  a.pair_slot = pair_slot;
  a.drop_mask = drop_mask;
  a.status_out = status;

  const size_t smem = scan_smem_bytes(s.E);
  if (ws.num_tiles > 0 && smem > 32 * 1024) {
    cudaError_t err = opt_in_smem();
    if (err != cudaSuccess) return err;
  }

  // One cluster when the pairs fit in at most max_cluster_size() tiles of
  // 512 * 16 pairs and the rows in a few passes of its threads; the fewest
  // pairs per lane (1, 2, 4, 8 or 16) that fit, so that the ranking rounds,
  // the serial part of a tile, stay short.
  const uint32_t forced = MOE_FLAG_LAYOUT_TWO_PASS | MOE_FLAG_LAYOUT_LOOKBACK |
                          MOE_FLAG_TEST_STALL_SCAN;
  if (!(s.flags & forced) && s.P <= (int64_t)kScanThreads * 4 && s.rows <= kSingleMaxRows) {
    // one tile: one ordinary CTA, the fewest pairs per lane that fit
    for (int rounds : kSingleRounds) {
      if (s.P <= (int64_t)kScanThreads * rounds) {
        if (opt_in_smem() != cudaSuccess) return cudaErrorUnknown;
        return launch_single(rounds, a, smem, stream);
      }
    }
  }
  if (!(s.flags & forced) && s.rows <= kClusterMaxRows) {
    const int maxc = max_cluster_size();
    for (int rounds : kClusterRounds) {
      const int64_t per_tile = (int64_t)kScanThreads * rounds;
      const int64_t tiles = std::max<int64_t>(1, (s.P + per_tile - 1) / per_tile);
      if (maxc > 0 && tiles <= maxc) {
        if (opt_in_smem() != cudaSuccess) return cudaErrorUnknown;
        return launch_cluster(rounds, a, (int)tiles, smem, stream);
      }
    }
  }

  if (ws.num_tiles > 0 && ws.num_tiles <= kFusedMaxTiles &&
      !(s.flags & MOE_FLAG_LAYOUT_TWO_PASS)) {
    // one CTA per tile at least, one thread per pair or row at most, all
    // co-resident (the grid-wide wait needs every CTA running)
    const int capacity = fused_capacity(smem);
    const int64_t work = std::max<int64_t>(s.P, s.rows);
    const int64_t want = std::max<int64_t>(ws.num_tiles, (work + kScanThreads - 1) / kScanThreads);
    const int grid = (int)std::min<int64_t>(want, capacity);
    if (grid >= ws.num_tiles) {
      void *args[] = {&a};
      return cudaLaunchCooperativeKernel((const void *)layout_fused_kernel, dim3(grid),
                                         dim3(kScanThreads), args, smem, stream);
    }
  }
  if (ws.num_tiles > 0) {
    layout_count_scan_kernel<<<ws.num_tiles, kScanThreads, smem, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const int64_t work = std::max<int64_t>(std::max<int64_t>(s.P, s.rows),
                                         (int64_t)ws.num_tiles * s.E);
  const int64_t max_blocks = (int64_t)device_sm_count() * 8;
  const int blocks = (int)std::max<int64_t>(
      1, std::min<int64_t>(max_blocks, (work + kEmitThreads - 1) / kEmitThreads));
  return launch_pdl(layout_emit_kernel, dim3(blocks), dim3(kEmitThreads), 0, stream, a);
}

}  // namespace moe
