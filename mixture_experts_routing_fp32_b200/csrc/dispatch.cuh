// Dispatch: counting-sort permutation of the (token, k) slots by expert,
// capacity drop, sentinel slots, and the gather of token rows.
//
// Follows the "8-MoE" lecture notes (MoE 高效推理: group tokens by expert so
// each expert's tokens are contiguous, then gather; Expert Capacity and
// GShard: assignments beyond capacity are dropped), the STA324 notes "08 MoE"
// §8.5 (capacity ceil(c*T*K/E); padding must not pollute load statistics)
// and §8.8 (gather per expert), and the transformers batched_mm issue
// (sentinel slots with no local expert contribute nothing).
//
// Slots are ranked within their expert in flat slot order j = t*K + k, so
// the permutation is the stable counting sort; it is deterministic.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kDispWarps = 8;
constexpr int kDispIters = 16;                                // 32-slot groups per warp
constexpr int kDispChunk = kDispWarps * kDispIters * 32;      // slots per block
// single-block dispatch (histogram, scan and rank in one kernel) up to
// kSmallWarps * kDispIters * 32 slots
constexpr int kSmallWarps = 32;
constexpr int kSmallSlots = kSmallWarps * kDispIters * 32;

__device__ __forceinline__ int slot_expert(const int32_t* idx, const uint8_t* mask,
                                           int64_t j, int E) {
  int e = idx[j];
  if (mask != nullptr && mask[j]) e = -1;
  if (e < -1 || e >= E) {
    set_dev_error(MOE_DEVERR_EXPERT_ID);
    e = -1;
  }
  return e;
}

// Expert ids of one warp's n_it groups of 32 consecutive slots starting at
// slot j0 (-1 sentinel, -2 past the end), every load issued up front.
__device__ __forceinline__ void warp_load_slots(const int32_t* idx, const uint8_t* mask,
                                                int64_t n_slots, int E, int64_t j0, int n_it,
                                                int (&ev)[kDispIters]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int it = 0; it < kDispIters; ++it) {
    const int64_t j = j0 + it * 32 + lane;
    ev[it] = (it < n_it && j < n_slots) ? slot_expert(idx, mask, j, E) : -2;
  }
}

// Adds this warp's slots to row[e] (shared memory, one row per warp or per
// block) with one update per distinct expert of each group; returns the
// number of sentinel slots (same value in every lane).
__device__ __forceinline__ int warp_count(const int (&ev)[kDispIters], int32_t* row,
                                          bool shared_row) {
  const unsigned lt = (1u << (threadIdx.x & 31)) - 1u;
  int sent = 0;
#pragma unroll
  for (int it = 0; it < kDispIters; ++it) {
    const int e = ev[it];
    if (__all_sync(0xffffffffu, e == -2)) break;   // past this warp's slots
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) {
      if (shared_row) atomicAdd(&row[e], __popc(peers));
      else row[e] += __popc(peers);
    }
    sent += __popc(__ballot_sync(0xffffffffu, e == -1));
    __syncwarp();
  }
  return sent;
}

// Stable rank of this warp's slots (row[e] holds the rank of the warp's
// first slot of expert e, and is advanced), capacity drop, slot <-> row maps.
__device__ __forceinline__ void warp_rank(const int (&ev)[kDispIters], int64_t j0,
                                          int64_t n_slots, int64_t C, int64_t rows_max,
                                          int32_t* row, const int32_t* seg_off, int ebase,
                                          int El, int32_t* __restrict__ slot_row,
                                          int32_t* __restrict__ row_slot) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int it = 0; it < kDispIters; ++it) {
    const int64_t j = j0 + it * 32 + lane;
    const int e = ev[it];
    if (__all_sync(0xffffffffu, e == -2)) break;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int32_t rank = 0;
    if (e >= 0) rank = row[e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) row[e] += __popc(peers);
    __syncwarp();
    if (e != -2) {
      // -2: sentinel or another shard's expert, -1: dropped
      const bool local = e >= ebase && e < ebase + El;
      int32_t r = (e == -1 || (e >= 0 && !local)) ? -2 : -1;
      if (local && (C < 0 || rank < C)) {
        r = seg_off[e - ebase] + rank;
        if (r < rows_max) row_slot[r] = (int32_t)j;
        else { set_dev_error(MOE_DEVERR_ROWS); r = -1; }
      }
      slot_row[j] = r;
    }
  }
}

// Block-wide: from per-expert totals (tot[e], shared, over all E experts)
// derive counts (all E), and for the local experts [ebase, ebase + El):
// kept (capacity), segment offsets aligned to `align` rows (seg[l], shared,
// and offsets[] in global memory), the tile -> local expert map and the
// stats words.  Valid slots of other experts count as sentinels here.
// Called by every thread of the block; ends with a __syncthreads.
__device__ void finish_layout(const int32_t* tot, int32_t* seg, int E, int ebase, int El, int T,
                              int n_shared, int64_t C, int64_t rows_max, int align,
                              int32_t sentinels, int32_t* __restrict__ counts,
                              int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
                              int32_t* __restrict__ tile_expert, int32_t* __restrict__ stats,
                              int32_t* __restrict__ row_slot) {
  __shared__ unsigned long long drop_s;
  __shared__ unsigned long long remote_s;
  __shared__ int32_t total_s;
  if (threadIdx.x == 0) { drop_s = 0; remote_s = 0; }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t run = tot[e];
    counts[e] = run;
    if (e < ebase || e >= ebase + El) {
      if (run) atomicAdd(&remote_s, (unsigned long long)run);
      continue;
    }
    const int l = e - ebase;
    const int32_t k = (C >= 0 && run > C) ? (int32_t)C : run;
    kept[l] = k;
    if (run > k) atomicAdd(&drop_s, (unsigned long long)(run - k));
    seg[l] = (k + align - 1) / align * align;
  }
  __syncthreads();
  // exclusive scan of the padded sizes by warp 0 (El <= 512: 16 per lane)
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (El + 31) / 32;
    const int e0 = lane * per, e1 = min(El, e0 + per);
    int64_t local = 0;
    for (int e = e0; e < e1; ++e) local += seg[e];
    int64_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int64_t run = incl - local;
    for (int e = e0; e < e1; ++e) { const int64_t v = seg[e]; seg[e] = (int32_t)run; run += v; }
    if (lane == 31) {
      const int64_t routed = incl;
      const int64_t shared_rows = n_shared ? ((int64_t)T + align - 1) / align * align : 0;
      int64_t total = routed + shared_rows;
      if (total > rows_max) { set_dev_error(MOE_DEVERR_ROWS); total = rows_max; }
      offsets[El] = (int32_t)routed;
      offsets[El + 1] = (int32_t)total;
      stats[0] = (int32_t)drop_s;
      stats[1] = sentinels + (int32_t)remote_s;
      stats[2] = (int32_t)total;
      stats[3] = (int32_t)(total / kRowTile);
      seg[El] = (int32_t)routed;
      total_s = (int32_t)total;
    }
  }
  __syncthreads();
  const int64_t total = total_s;
  for (int e = threadIdx.x; e <= El; e += blockDim.x) {
    const int64_t beg = seg[e];
    const int64_t end = (e < El) ? seg[e + 1] : total;
    if (e < El) offsets[e] = (int32_t)beg;
    for (int64_t r = beg; r < end && r < total; r += kRowTile) tile_expert[r / kRowTile] = e;
  }
  // rows that hold no routed slot (each expert's padding, the shared
  // expert's rows) get row_slot = -1; the rank pass fills the others
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int e = warp; e < El; e += nw) {
    const int32_t run = tot[ebase + e];
    const int32_t k = (C >= 0 && run > C) ? (int32_t)C : run;
    const int64_t end = seg[e + 1] < total ? (int64_t)seg[e + 1] : total;
    for (int64_t r = seg[e] + k + lane; r < end; r += 32) row_slot[r] = -1;
  }
  for (int64_t r = (int64_t)seg[El] + threadIdx.x; r < total; r += blockDim.x) row_slot[r] = -1;
  __syncthreads();
}

// Pass 1: per-block histograms of valid slots and sentinel counts.
__global__ void __launch_bounds__(256)
disp_hist_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ mask,
                 int64_t n_slots, int E, int32_t* __restrict__ block_hist,
                 int32_t* __restrict__ block_sent) {
  pdl_begin();
  extern __shared__ int32_t hist[];   // [E]
  __shared__ int32_t sent;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  if (threadIdx.x == 0) sent = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int64_t j0 = (int64_t)blockIdx.x * kDispChunk + (int64_t)warp * kDispIters * 32;
  int ev[kDispIters];
  warp_load_slots(idx, mask, n_slots, E, j0, kDispIters, ev);
  const int my_sent = warp_count(ev, hist, true);
  if ((threadIdx.x & 31) == 0 && my_sent) atomicAdd(&sent, my_sent);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    block_hist[(size_t)blockIdx.x * E + e] = hist[e];
  if (threadIdx.x == 0) block_sent[blockIdx.x] = sent;
}

// Pass 2 (one block): per-expert totals, exclusive scan over blocks (block
// bases), then the layout (counts, kept, offsets, tile map, stats).
__global__ void __launch_bounds__(1024)
disp_scan_kernel(int32_t* __restrict__ block_hist, const int32_t* __restrict__ block_sent,
                 int n_blocks, int E, int ebase, int El, int T, int n_shared, int64_t C,
                 int64_t rows_max, int align, int32_t* __restrict__ counts,
                 int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
                 int32_t* __restrict__ tile_expert, int32_t* __restrict__ stats,
                 int32_t* __restrict__ row_slot) {
  pdl_begin();
  extern __shared__ int32_t sh[];     // tot[E], seg[El + 1]
  int32_t* tot = sh;
  int32_t* seg = sh + E;
  __shared__ int32_t sent_total;
  if (threadIdx.x == 0) sent_total = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
#pragma unroll 8
    for (int b = 0; b < n_blocks; ++b) {
      const int32_t c = block_hist[(size_t)b * E + e];
      block_hist[(size_t)b * E + e] = run;   // becomes the block's base rank
      run += c;
    }
    tot[e] = run;
  }
  int32_t ls = 0;
  for (int b = threadIdx.x; b < n_blocks; b += blockDim.x) ls += block_sent[b];
  if (ls) atomicAdd(&sent_total, ls);
  __syncthreads();
  finish_layout(tot, seg, E, ebase, El, T, n_shared, C, rows_max, align, sent_total, counts, kept,
                offsets, tile_expert, stats, row_slot);
}

// Pass 3: stable rank of every slot inside its expert, capacity drop,
// slot <-> row maps.  Warp w of block b walks its 512 slots in order; peers
// with the same expert inside a 32-slot group are ranked by lane.
__global__ void __launch_bounds__(256)
disp_rank_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ mask,
                 int64_t n_slots, int E, int ebase, int El, int64_t C, int64_t rows_max,
                 const int32_t* __restrict__ block_base,
                 const int32_t* __restrict__ offsets,
                 int32_t* __restrict__ slot_row, int32_t* __restrict__ row_slot) {
  pdl_begin();
  extern __shared__ int32_t wh[];   // [kDispWarps][E] per-warp counters, then seg_off[El]
  int32_t* seg_off = wh + kDispWarps * E;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kDispWarps * E; i += blockDim.x) wh[i] = 0;
  for (int e = threadIdx.x; e < El; e += blockDim.x) seg_off[e] = offsets[e];
  const int64_t j0 = (int64_t)blockIdx.x * kDispChunk + (int64_t)warp * kDispIters * 32;
  int ev[kDispIters];
  warp_load_slots(idx, mask, n_slots, E, j0, kDispIters, ev);
  __syncthreads();
  warp_count(ev, wh + warp * E, false);
  __syncthreads();
  // exclusive scan over warps, seeded with the block's base rank
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = block_base[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < kDispWarps; ++w) {
      const int32_t c = wh[w * E + e];
      wh[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  warp_rank(ev, j0, n_slots, C, rows_max, wh + warp * E, seg_off, ebase, El, slot_row, row_slot);
}

// Passes 1-3 in one block for up to kSmallSlots slots: 32 warps each own
// a run of consecutive slots, so scanning the per-warp counts in warp
// order gives the same stable ranks as the multi-block passes.
__global__ void __launch_bounds__(1024)
disp_small_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ mask,
                  int64_t n_slots, int E, int ebase, int El, int T, int n_shared, int64_t C,
                  int64_t rows_max,
                  int align, int32_t* __restrict__ counts, int32_t* __restrict__ kept,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ tile_expert,
                  int32_t* __restrict__ stats, int32_t* __restrict__ slot_row,
                  int32_t* __restrict__ row_slot) {
  pdl_begin();
  extern __shared__ int32_t wh[];   // [kSmallWarps][E] counters, tot[E], seg[El + 1]
  int32_t* tot = wh + kSmallWarps * E;
  int32_t* seg = tot + E;
  __shared__ int32_t sent_total;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) wh[i] = 0;
  if (threadIdx.x == 0) sent_total = 0;
  const int n_it = (int)((n_slots + kSmallWarps * 32 - 1) / (kSmallWarps * 32));
  const int64_t j0 = (int64_t)warp * n_it * 32;
  int ev[kDispIters];
  warp_load_slots(idx, mask, n_slots, E, j0, n_it, ev);
  __syncthreads();
  const int sent = warp_count(ev, wh + warp * E, false);
  if ((threadIdx.x & 31) == 0 && sent) atomicAdd(&sent_total, sent);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < kSmallWarps; ++w) {
      const int32_t c = wh[w * E + e];
      wh[w * E + e] = run;
      run += c;
    }
    tot[e] = run;
  }
  __syncthreads();
  finish_layout(tot, seg, E, ebase, El, T, n_shared, C, rows_max, align, sent_total, counts, kept,
                offsets, tile_expert, stats, row_slot);
  warp_rank(ev, j0, n_slots, C, rows_max, wh + warp * E, seg, ebase, El, slot_row, row_slot);
}

// Pass 4: gather x rows into expert order; zero padding rows; shared rows.
// A row's source is decided by row_slot alone (-1: padding below the shared
// segment, or a shared row), so each warp's chain is one index load then
// the row copy.
template <typename TX>
__global__ void __launch_bounds__(256)
disp_gather_kernel(const TX* __restrict__ x, int D, int K, int E, int T,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ stats,
                   const int32_t* __restrict__ row_slot, TX* __restrict__ x_perm) {
  pdl_begin();
  const int n_rows = stats[2];
  const int64_t shared0 = offsets[E];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t r = (int64_t)blockIdx.x * 8 + warp; r < n_rows; r += (int64_t)gridDim.x * 8) {
    const int32_t slot = row_slot[r];
    int64_t src = -1;
    if (slot >= 0) src = slot / K;
    else if (r >= shared0 && r - shared0 < T) src = r - shared0;
    TX* dst = x_perm + r * D;
    if (src >= 0) {
      // four 256-column steps' loads in flight before their stores
      const TX* s = x + src * D;
      for (int d0 = 0; d0 < D; d0 += 1024) {
        Raw8<TX> v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int d = d0 + 256 * j + lane * 8;
          v[j].load(s + (d < D ? d : lane * 8));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int d = d0 + 256 * j + lane * 8;
          if (d < D) v[j].store(dst + d);
        }
      }
    } else {
      for (int d = lane * 8; d < D; d += 256) zero8(dst + d);
    }
  }
}

// Padding rows (row_slot < 0 outside the shared expert's rows) of a
// permuted buffer set to zero: each warp checks 32 rows per step.
template <typename TX>
__device__ __forceinline__ void zero_padding_rows(TX* __restrict__ buf, int64_t n_rows, int D,
                                                  const int32_t* __restrict__ row_slot,
                                                  int64_t shared0, int64_t shared_n) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t base = ((int64_t)blockIdx.x * 8 + warp) * 32; base < n_rows;
       base += (int64_t)gridDim.x * 8 * 32) {
    const int64_t r = base + lane;
    const bool pad = r < n_rows && row_slot[r] < 0 && !(r >= shared0 && r < shared0 + shared_n);
    unsigned m = __ballot_sync(0xffffffffu, pad);
    while (m != 0u) {
      const int64_t rr = base + __ffs(m) - 1;
      m &= m - 1u;
      for (int d = lane * 8; d < D; d += 256) zero8(buf + rr * D + d);
    }
  }
}

// Pass 4 in token order (K in {1, 2, 4, 8}): each token's row of x is read
// once and written to the rows of its kept slots (and its shared-expert
// row); then the padding rows are zeroed.  One warp per token, NB
// 256-column steps of loads in flight before their stores.
template <typename TX, int KT>
__global__ void __launch_bounds__(256)
disp_gather_tok_kernel(const TX* __restrict__ x, int D, int El, int T, int n_shared,
                       const int32_t* __restrict__ offsets, const int32_t* __restrict__ stats,
                       const int32_t* __restrict__ slot_row, const int32_t* __restrict__ row_slot,
                       TX* __restrict__ x_perm) {
  pdl_begin();
  constexpr int NB = 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t shared0 = n_shared ? (int64_t)offsets[El] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < T; t += (int64_t)gridDim.x * 8) {
    const int32_t my_row = lane < KT ? slot_row[t * KT + lane] : -1;
    int64_t rows[KT + 1];
#pragma unroll
    for (int k = 0; k < KT; ++k) rows[k] = __shfl_sync(0xffffffffu, my_row, k);
    rows[KT] = n_shared ? shared0 + t : -1;
    const TX* src = x + t * D;
    for (int d0 = lane * 8; d0 < D; d0 += 256 * NB) {
      Raw8<TX> v[NB];
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const int d = d0 + 256 * j;
        v[j].load(src + (d < D ? d : lane * 8));
      }
#pragma unroll
      for (int k = 0; k <= KT; ++k) {
        if (rows[k] >= 0) {
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            const int d = d0 + 256 * j;
            if (d < D) v[j].store(x_perm + rows[k] * D + d);
          }
        }
      }
    }
  }
  zero_padding_rows(x_perm, stats[2], D, row_slot, shared0, n_shared ? T : 0);
}

}  // namespace moe
