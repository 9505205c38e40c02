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

// Pass 1: per-block histograms of valid slots and sentinel counts.
__global__ void __launch_bounds__(256)
disp_hist_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ mask,
                 int64_t n_slots, int E, int32_t* __restrict__ block_hist,
                 int32_t* __restrict__ block_sent) {
  extern __shared__ int32_t hist[];   // [E]
  __shared__ int32_t sent;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  if (threadIdx.x == 0) sent = 0;
  __syncthreads();
  const int64_t j0 = (int64_t)blockIdx.x * kDispChunk;
  const int64_t j1 = min(j0 + kDispChunk, n_slots);
  // every load of this thread first (one memory latency, not one per slot)
  constexpr int kPer = kDispChunk / 256;
  int ev[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int64_t j = j0 + threadIdx.x + (int64_t)k * 256;
    ev[k] = (j < j1) ? slot_expert(idx, mask, j, E) : -2;
  }
  int my_sent = 0;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    if (ev[k] >= 0) atomicAdd(&hist[ev[k]], 1);
    else if (ev[k] == -1) ++my_sent;
  }
  if (my_sent) atomicAdd(&sent, my_sent);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    block_hist[(size_t)blockIdx.x * E + e] = hist[e];
  if (threadIdx.x == 0) block_sent[blockIdx.x] = sent;
}

// Pass 2 (one block): per-expert totals, exclusive scan over blocks (block
// bases), capacity, padded offsets (segments aligned to `align` rows, a
// multiple of the 128-row tile), tile -> expert map, stats.
__global__ void __launch_bounds__(1024)
disp_scan_kernel(int32_t* __restrict__ block_hist, const int32_t* __restrict__ block_sent,
                 int n_blocks, int E, int T, int n_shared, int64_t C,
                 int64_t rows_max, int align, int32_t* __restrict__ counts,
                 int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
                 int32_t* __restrict__ tile_expert, int32_t* __restrict__ stats) {
  extern __shared__ int64_t sh[];     // [E] padded sizes -> offsets
  __shared__ int64_t drop_total;
  __shared__ int32_t sent_total;
  if (threadIdx.x == 0) { drop_total = 0; sent_total = 0; }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
#pragma unroll 8
    for (int b = 0; b < n_blocks; ++b) {
      const int32_t c = block_hist[(size_t)b * E + e];
      block_hist[(size_t)b * E + e] = run;   // becomes the block's base rank
      run += c;
    }
    counts[e] = run;
    const int32_t k = (C >= 0 && run > C) ? (int32_t)C : run;
    kept[e] = k;
    if (run > k) atomicAdd((unsigned long long*)&drop_total,
                           (unsigned long long)(run - k));
    sh[e] = ((int64_t)k + align - 1) / align * align;
  }
  for (int b = threadIdx.x; b < n_blocks; b += blockDim.x)
    atomicAdd(&sent_total, block_sent[b]);
  __syncthreads();
  if (threadIdx.x == 0) {   // E <= 512: a serial scan is negligible
    int64_t run = 0;
    for (int e = 0; e < E; ++e) { const int64_t v = sh[e]; sh[e] = run; run += v; }
    const int64_t shared_rows = n_shared ? ((int64_t)T + align - 1) / align * align : 0;
    int64_t total = run + shared_rows;
    if (total > rows_max) { set_dev_error(MOE_DEVERR_ROWS); total = rows_max; }
    offsets[E] = (int32_t)run;
    offsets[E + 1] = (int32_t)total;
    stats[0] = (int32_t)drop_total;
    stats[1] = sent_total;
    stats[2] = (int32_t)total;
    stats[3] = (int32_t)(total / kRowTile);
  }
  __syncthreads();
  const int64_t total = offsets[E + 1];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    const int64_t beg = (e < E) ? sh[e] : offsets[E];
    const int64_t end = (e + 1 < E) ? sh[e + 1] : (e < E ? offsets[E] : total);
    if (e < E) offsets[e] = (int32_t)beg;
    for (int64_t r = beg; r < end && r < total; r += kRowTile)
      tile_expert[r / kRowTile] = e;
  }
}

// Pass 3: stable rank of every slot inside its expert, capacity drop,
// slot <-> row maps.  Warp w of block b walks its 512 slots in order; peers
// with the same expert inside a 32-slot group are ranked by lane.
__global__ void __launch_bounds__(256)
disp_rank_kernel(const int32_t* __restrict__ idx, const uint8_t* __restrict__ mask,
                 int64_t n_slots, int E, int64_t C, int64_t rows_max,
                 const int32_t* __restrict__ block_base,
                 const int32_t* __restrict__ offsets,
                 int32_t* __restrict__ slot_row, int32_t* __restrict__ row_slot) {
  extern __shared__ int32_t wh[];   // [kDispWarps][E] per-warp counters
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kDispWarps * E; i += blockDim.x) wh[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kDispChunk + (int64_t)warp * kDispIters * 32;
  const unsigned lt = (1u << lane) - 1u;
  // the warp's slots, loaded once up front
  int ev[kDispIters];
#pragma unroll
  for (int it = 0; it < kDispIters; ++it) {
    const int64_t j = base + it * 32 + lane;
    ev[it] = (j < n_slots) ? slot_expert(idx, mask, j, E) : -1;
  }
  // per-warp histogram
#pragma unroll
  for (int it = 0; it < kDispIters; ++it) {
    const int e = ev[it];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) wh[warp * E + e] += __popc(peers);
  }
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
#pragma unroll
  for (int it = 0; it < kDispIters; ++it) {
    const int64_t j = base + it * 32 + lane;
    const int e = ev[it];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int32_t rank = 0;
    if (e >= 0) rank = wh[warp * E + e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) wh[warp * E + e] += __popc(peers);
    __syncwarp();
    if (j < n_slots) {
      int32_t row = -1;
      if (e >= 0 && (C < 0 || rank < C)) {
        row = offsets[e] + rank;
        if (row < rows_max) row_slot[row] = (int32_t)j;
        else { set_dev_error(MOE_DEVERR_ROWS); row = -1; }
      }
      slot_row[j] = row;
    }
  }
}

// Pass 4: gather x rows into expert order; zero padding rows; shared rows.
template <typename TX>
__global__ void __launch_bounds__(256)
disp_gather_kernel(const TX* __restrict__ x, int D, int K, int E, int T,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ kept,
                   const int32_t* __restrict__ tile_expert, const int32_t* __restrict__ stats,
                   int32_t* __restrict__ row_slot, TX* __restrict__ x_perm) {
  const int n_rows = stats[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t r = (int64_t)blockIdx.x * 8 + warp; r < n_rows; r += (int64_t)gridDim.x * 8) {
    const int e = tile_expert[r / kRowTile];
    int64_t src = -1;
    if (e < E) {
      const int64_t local = r - offsets[e];
      if (local < kept[e]) src = row_slot[r] / K;
      else if (lane == 0) row_slot[r] = -1;
    } else {
      const int64_t t = r - offsets[E];
      if (t < T) src = t;
      if (lane == 0) row_slot[r] = -1;
    }
    TX* dst = x_perm + r * D;
    if (src >= 0) {
      const TX* s = x + src * D;
      for (int d = lane * 8; d < D; d += 256) {
        float v[8];
        load8(s + d, v);
        store8(dst + d, v);
      }
    } else {
      for (int d = lane * 8; d < D; d += 256) zero8(dst + d);
    }
  }
}

}  // namespace moe
