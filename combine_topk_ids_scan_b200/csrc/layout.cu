// layout.cu -- dispatch layout: stable counting sort of (token, k) pairs by
// expert, in two kernels.
//
//  count_scan  One CTA per tile of 4096 consecutive pairs, tiles taken in
//              launch order from an atomic ticket.  Each warp owns 256
//              consecutive pairs and walks them in 8 rounds of 32; in a round,
//              lanes naming the same expert find each other with
//              __match_any_sync, take their rank from the popcount of lower
//              peers, and the highest peer bumps the warp's private
//              shared-memory histogram (so the histogram needs no atomics and
//              ranks are in pair order).  A scan over the 16 warp histograms
//              gives each warp its per-expert base inside the tile.  Tiles
//              then chain their per-expert counts with a single-pass
//              decoupled look-back (one 64-bit word per (tile, expert): flag
//              in the high half, count in the low half), giving each tile its
//              exclusive per-expert prefix.  The result per pair is its rank
//              among all earlier pairs of the same expert -- stable by
//              (token, k) by construction.  The last tile stores the totals.
//  emit        Exclusive scan of the per-expert totals (every CTA, in shared
//              memory), then per pair: row = expert start + rank (packed), or
//              e*Ce + rank with rank >= Ce dropped (capacity); writes
//              pair_slot, row_src, drop_mask, padding rows, counts, offsets,
//              the [4,S] table, and returns the workspace to zero.
//
// Layout definitions: NKI "Permute A2AV Kernel API Reference" (permute_a2av
// packed_source_indices, send_counts, recv_capacity, [4, EP] metadata in
// elements); DeepSpeed capacity dispatch ([e, c, m] buffer); NeMo AutoModel
// token_dispatcher (-1 ids are masked; tokens per expert).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kScanThreads = 512;
constexpr int kScanWarps = kScanThreads / kWarp;  // 16
constexpr int kScanRounds = 8;                     // pairs per lane
constexpr int kTilePairs = kScanThreads * kScanRounds;  // 4096
constexpr int kWarpPairs = kWarp * kScanRounds;         // 256
constexpr uint64_t kFlagAggregate = 1ull;
constexpr uint64_t kFlagInclusive = 2ull;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded look-back wait: 1 s

constexpr int kEmitThreads = 256;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline size_t scan_smem_bytes(int E) {
  return align_up((size_t)kScanWarps * E * sizeof(uint16_t), 16) + (size_t)E * sizeof(uint32_t);
}

__global__ void __launch_bounds__(kScanThreads)
    layout_count_scan_kernel(const int32_t *__restrict__ ids, int64_t P, int32_t E,
                             int32_t num_tiles, uint32_t flags, uint32_t *ctrl,
                             int32_t *__restrict__ totals, uint64_t *tiles,
                             int32_t *__restrict__ pair_rank) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t *wcnt = reinterpret_cast<uint16_t *>(smem);  // [warps][E]
  uint32_t *tile_prefix =
      reinterpret_cast<uint32_t *>(smem + align_up((size_t)kScanWarps * E * 2, 16));  // [E]
  __shared__ int s_tile;
  __shared__ uint32_t s_status;

  const int tid = threadIdx.x, warp = tid / kWarp, lane = tid % kWarp;
  if (tid == 0) {
    s_tile = (int)atomicAdd(&ctrl[0], 1u);
    s_status = 0;
  }
  for (int i = tid; i < kScanWarps * E; i += kScanThreads) wcnt[i] = 0;
  __syncthreads();
  const int tile = s_tile;
  // a ticket past the last tile only happens with a workspace that was not
  // zero-filled before first use: do nothing (the other tiles' bounded waits
  // then report MOE_STATUS_TIMEOUT)
  if (tile >= num_tiles) return;

  // ---- 1. per-warp stable ranks and histograms
  const int64_t base = (int64_t)tile * kTilePairs + (int64_t)warp * kWarpPairs;
  int32_t ex[kScanRounds];
#pragma unroll
  for (int r = 0; r < kScanRounds; ++r) {
    const int64_t p = base + r * kWarp + lane;
    ex[r] = p < P ? __ldg(ids + p) : -1;
  }
  uint16_t rank[kScanRounds];
  bool bad_id = false;
  uint16_t *my_cnt = wcnt + (size_t)warp * E;
#pragma unroll
  for (int r = 0; r < kScanRounds; ++r) {
    const int32_t e = ex[r];
    const bool valid = (uint32_t)e < (uint32_t)E;
    bad_id |= (!valid && e != -1);
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, valid ? (uint32_t)e : 0xFFFFFFFFu);
    uint32_t before = 0;
    if (valid) before = my_cnt[e];
    __syncwarp();
    rank[r] = 0;
    if (valid) {
      rank[r] = (uint16_t)(before + __popc(peers & lanemask_lt()));
      if (lane == 31 - __clz(peers)) my_cnt[e] = (uint16_t)(before + __popc(peers));
    }
    __syncwarp();
    ex[r] = valid ? e : -1;
  }
  if (__any_sync(0xFFFFFFFFu, bad_id) && lane == 0) atomicOr(&s_status, MOE_STATUS_ID_RANGE);
  __syncthreads();

  // ---- 2. per expert: exclusive scan over the warps, tile aggregate
  for (int e = tid; e < E; e += kScanThreads) {
    uint32_t run = 0;
#pragma unroll 4
    for (int w = 0; w < kScanWarps; ++w) {
      const uint32_t c = wcnt[w * E + e];
      wcnt[w * E + e] = (uint16_t)run;
      run += c;
    }
    tile_prefix[e] = run;
  }

  // ---- 3. decoupled look-back across tiles, one chain per expert
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
      int look = tile - 1;
      while (look >= 0) {
        const uint64_t v = ld_relaxed_gpu_u64(&tiles[(size_t)look * E + e]);
        const uint64_t f = v >> 32;
        if (f == 0) {
          // predecessor has not published yet: it holds an earlier ticket, so
          // it is running; wait for it, but never longer than the limit
          const uint64_t now = globaltimer_ns();
          if (deadline == 0) {
            deadline = now + kWaitLimitNs;
          } else if (now > deadline) {
            timed_out = true;
            break;
          }
          __nanosleep(64);
          continue;
        }
        excl += (uint32_t)v;
        if (f == kFlagInclusive) break;
        --look;
      }
      st_relaxed_gpu_u64(&tiles[(size_t)tile * E + e], (kFlagInclusive << 32) | (excl + agg));
    }
    tile_prefix[e] = excl;
    if (tile == num_tiles - 1) totals[e] = (int32_t)(excl + agg);
  }
  if (timed_out) atomicOr(&s_status, MOE_STATUS_TIMEOUT);
  __syncthreads();

  // ---- 4. rank of each pair among all earlier pairs of its expert
#pragma unroll
  for (int r = 0; r < kScanRounds; ++r) {
    const int64_t p = base + r * kWarp + lane;
    if (p < P) {
      const int32_t e = ex[r];
      pair_rank[p] = e >= 0 ? (int32_t)(tile_prefix[e] + my_cnt[e] + rank[r]) : -1;
    }
  }
  if (tid == 0 && s_status) atomicOr(&ctrl[2], s_status);
}

// Block-wide exclusive scan of n <= 8 * kEmitThreads values in place.
__device__ void block_exclusive_scan(int32_t *v, int n, int32_t *total_out) {
  __shared__ int32_t warp_sums[kEmitThreads / kWarp];
  constexpr int kPer = 8;
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  int32_t local[kPer];
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = tid * kPer + i;
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
  for (int w = 0; w < kEmitThreads / kWarp; ++w) {
    if (w < warp) warp_base += warp_sums[w];
    total += warp_sums[w];
  }
  int32_t run = warp_base + incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = tid * kPer + i;
    if (idx < n) v[idx] = run;
    run += local[i];
  }
  *total_out = total;
  __syncthreads();
}

__global__ void __launch_bounds__(kEmitThreads)
    layout_emit_kernel(const int32_t *__restrict__ ids, int32_t N, int32_t k, int32_t E,
                       int32_t S, int64_t C, int32_t Ce, int32_t H, uint32_t flags,
                       int32_t num_tiles, uint32_t *ctrl, const int32_t *__restrict__ totals,
                       uint64_t *tiles, int32_t *__restrict__ expert_counts,
                       int32_t *__restrict__ expert_offsets, uint32_t *__restrict__ meta,
                       int32_t *__restrict__ row_src, int32_t *__restrict__ pair_slot,
                       uint8_t *__restrict__ drop_mask, uint32_t *status_out) {
  extern __shared__ __align__(16) int32_t s_emit[];
  int32_t *s_off = s_emit;           // [E + 1] first row per expert
  int32_t *s_kept = s_emit + E + 1;  // [E] rows kept per expert
  __shared__ uint32_t s_status;
  const int tid = threadIdx.x;
  const bool capacity = Ce > 0;
  const int64_t P = (int64_t)N * k;
  const int64_t rows = capacity ? (int64_t)E * Ce : C;
  if (tid == 0) s_status = 0;

  for (int e = tid; e < E; e += kEmitThreads) {
    const int32_t t = num_tiles > 0 ? totals[e] : 0;
    s_kept[e] = capacity ? min(t, Ce) : t;
    s_off[e] = capacity ? e * Ce : t;
  }
  __syncthreads();
  int32_t total = 0;
  if (!capacity) {
    block_exclusive_scan(s_off, E, &total);
    if (tid == 0) s_off[E] = total;
  } else if (tid == 0) {
    s_off[E] = E * Ce;
  }
  __syncthreads();

  const int64_t gtid = (int64_t)blockIdx.x * kEmitThreads + tid;
  const int64_t gstride = (int64_t)gridDim.x * kEmitThreads;
  uint32_t bits = 0;

  // ---- per pair: rank -> row
  for (int64_t p = gtid; p < P; p += gstride) {
    const int32_t e = __ldg(ids + p);
    int32_t slot = -1;
    uint8_t dropped = 0;
    if ((uint32_t)e < (uint32_t)E) {
      const int32_t r = pair_slot[p];
      if (capacity) {
        if (r >= 0 && r < Ce) slot = e * Ce + r;
        else dropped = 1;
      } else {
        const int64_t row = (int64_t)s_off[e] + r;
        if (r >= 0 && row >= 0 && row < C) {
          slot = (int32_t)row;
        } else {
          dropped = 1;
          bits |= MOE_STATUS_CAPACITY;
        }
      }
    }
    pair_slot[p] = slot;
    if (drop_mask) drop_mask[p] = dropped;
    if (slot >= 0) row_src[slot] = (int32_t)(p / k);
  }

  // ---- optional duplicate check, per token
  if (flags & MOE_FLAG_CHECK_DUPLICATES) {
    for (int64_t t = gtid; t < N; t += gstride) {
      const int32_t *row = ids + t * k;
      for (int a = 0; a < k; ++a) {
        const int32_t ea = __ldg(row + a);
        if ((uint32_t)ea >= (uint32_t)E) continue;
        for (int b = a + 1; b < k; ++b)
          if (__ldg(row + b) == ea) bits |= MOE_STATUS_DUP_ID;
      }
    }
  }

  // ---- padding rows
  for (int64_t r = gtid; r < rows; r += gstride) {
    bool pad;
    if (capacity) pad = (int32_t)(r % Ce) >= s_kept[r / Ce];
    else pad = r >= (int64_t)s_off[E];
    if (pad) row_src[r] = -1;
  }

  // ---- counts, offsets, [4, S] metadata (block 0)
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += kEmitThreads) expert_counts[e] = s_kept[e];
    for (int e = tid; e <= E; e += kEmitThreads) expert_offsets[e] = s_off[e];
    const int32_t L = E / S;
    for (int s = tid; s < S; s += kEmitThreads) {
      int64_t seg_rows = 0;
      for (int e = s * L; e < (s + 1) * L; ++e) seg_rows += s_kept[e];
      const uint32_t count_el = (uint32_t)(seg_rows * H);
      const uint32_t displ_el = capacity ? (uint32_t)((int64_t)s * L * Ce * H)
                                         : (uint32_t)((int64_t)s_off[s * L] * H);
      meta[0 * S + s] = count_el;
      meta[1 * S + s] = displ_el;
      meta[2 * S + s] = count_el;
      meta[3 * S + s] = displ_el;
    }
    if (tid == 0) ctrl[0] = 0;  // the scan kernel has finished: reset its ticket
  }

  // ---- return the scan tile states to zero for the next call
  const int64_t n_states = (int64_t)num_tiles * E;
  for (int64_t i = gtid; i < n_states; i += gstride) tiles[i] = 0;

  // ---- status: the last block to finish publishes this call's bits
  if (bits) atomicOr(&s_status, bits);
  __syncthreads();
  if (tid == 0) {
    if (s_status) atomicOr(&ctrl[2], s_status);
    __threadfence();
    const uint32_t done = atomicAdd(&ctrl[1], 1u);
    if (done == gridDim.x - 1) {
      __threadfence();
      *status_out = atomicExch(&ctrl[2], 0u);
      atomicExch(&ctrl[1], 0u);
    }
  }
}

}  // namespace

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
  if (ws.num_tiles > 0) {
    const size_t smem = scan_smem_bytes(s.E);
    if (smem > 48 * 1024) {
      cudaError_t err = cudaFuncSetAttribute(layout_count_scan_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
      if (err != cudaSuccess) return err;
    }
    layout_count_scan_kernel<<<ws.num_tiles, kScanThreads, smem, stream>>>(
        ids, s.P, s.E, ws.num_tiles, s.flags, ws.ctrl, ws.totals, ws.tiles, pair_slot);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const int64_t work = std::max<int64_t>(std::max<int64_t>(s.P, s.rows),
                                         (int64_t)ws.num_tiles * s.E);
  const int64_t max_blocks = (int64_t)device_sm_count() * 4;
  const int blocks = (int)std::max<int64_t>(
      1, std::min<int64_t>(max_blocks, (work + kEmitThreads * 4 - 1) / (kEmitThreads * 4)));
  const size_t smem = (size_t)(2 * s.E + 1) * sizeof(int32_t);
  layout_emit_kernel<<<blocks, kEmitThreads, smem, stream>>>(
      ids, s.N, s.k, s.E, s.S, s.C, s.Ce, s.H, s.flags, ws.num_tiles, ws.ctrl, ws.totals,
      ws.tiles, expert_counts, expert_offsets, meta, row_src, pair_slot, drop_mask, status);
  return cudaGetLastError();
}

}  // namespace moe
