// Row gather of the dispatch on the bulk-copy engine ("8-MoE" lecture
// notes, MoE 高效推理: gather each expert's tokens into a contiguous block;
// STA324 notes "08 MoE" §8.8): x_perm[r] = x[token(r)] for routed and shared
// rows, zeros for padding rows.
//
// A permuted row is a whole, 16-byte aligned row of x (D * 2 bytes), so it
// moves with two bulk copies and no register traffic: global -> shared
// (cp.async.bulk, completing on an mbarrier) and shared -> global
// (cp.async.bulk, committed in a bulk group).  One warp per CTA, several
// CTAs per SM; lane 0 drives the copies, the warp resolves the row sources
// and writes the padding rows.  Rows of a CTA are taken in chunks of NB:
// the NB loads of a chunk are in flight together, and the stores of one
// chunk overlap the loads of the next (two buffer sets; before a set is
// reused the stores that read it must have finished reading it).
#pragma once
#include "gemm_tc.cuh"

namespace moe {
namespace bulk {

__device__ __forceinline__ void g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most N committed bulk groups still reading shared memory
template <int N>
__device__ __forceinline__ void wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

constexpr int kCtasPerSm = 3;
constexpr int kBufBytes = 32768;   // per buffer set (NB rows)

__host__ __device__ constexpr uint32_t padded_row_bytes(int D) { return ((uint32_t)D * 2 + 127) & ~127u; }

// Shared memory of gather_kernel<NB>: two sets of NB row buffers, then one
// mbarrier per buffer.
__host__ __device__ constexpr size_t gather_smem(int NB, int D) {
  return 2 * (size_t)NB * padded_row_bytes(D) + 2 * NB * 8 + 128;
}

template <int NB>
__global__ void __launch_bounds__(32)
gather_kernel(const __nv_bfloat16* __restrict__ x, int D, int K, int El, int T,
              const int32_t* __restrict__ offsets, const int32_t* __restrict__ stats,
              const int32_t* __restrict__ row_slot, __nv_bfloat16* __restrict__ x_perm) {
  extern __shared__ uint8_t sm_raw[];
  const int lane = threadIdx.x;
  const uint32_t rb = (uint32_t)D * 2;
  const uint32_t rbp = padded_row_bytes(D);
  const uint32_t buf0 = (tc::smem_u32(sm_raw) + 127u) & ~127u;
  const uint32_t bar0 = buf0 + 2u * NB * rbp;
  auto buf = [&](int b) { return buf0 + (uint32_t)b * rbp; };
  auto bar = [&](int b) { return bar0 + 8u * b; };
  if (lane == 0) {
    for (int b = 0; b < 2 * NB; ++b) tc::mbar_init(bar(b), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  pdl_begin();
  const int64_t n_rows = stats[2];
  const int64_t shared0 = offsets[El];
  const int64_t G = gridDim.x;
  uint32_t ph = 0;            // parity of each buffer's barrier (lane 0)
  uint32_t pend = 0;          // buffers with a load issued and not yet waited for
  int set = 0;
  bool ok = true;
  __shared__ int abort_s;
  if (lane == 0) abort_s = 0;
  __syncwarp();
  for (int64_t j0 = 0; blockIdx.x + j0 * G < n_rows; j0 += NB) {
    // source token of this chunk's rows (lane i < NB: row blockIdx.x + (j0 + i) G);
    // -1: zero row, -2: past the end
    int src = -2;
    if (lane < NB) {
      const int64_t r = blockIdx.x + (j0 + lane) * G;
      if (r < n_rows) {
        const int32_t slot = row_slot[r];
        src = slot >= 0 ? slot / K : (r >= shared0 && r - shared0 < T ? (int)(r - shared0) : -1);
      }
    }
    int si[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) si[i] = __shfl_sync(0xffffffffu, src, i);
    if (lane == 0 && ok) {
      wait_read<1>();   // the stores that last read this buffer set are done reading it
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        if (si[i] >= 0) {
          const int b = set * NB + i;
          tc::mbar_expect_tx(bar(b), rb);
          g2s(buf(b), x + (int64_t)si[i] * D, rb, bar(b));
          pend |= 1u << b;
        }
      }
    }
    // padding rows: zeros, by the whole warp
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      if (si[i] == -1) {
        __nv_bfloat16* dst = x_perm + (blockIdx.x + (j0 + i) * G) * (int64_t)D;
        for (int d = lane * 8; d < D; d += 256) zero8(dst + d);
      }
    }
    if (lane == 0 && ok) {
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        if (si[i] >= 0) {
          const int b = set * NB + i;
          if (!tc::mbar_wait(bar(b), (ph >> b) & 1u, &abort_s)) { ok = false; break; }
          ph ^= 1u << b;
          pend &= ~(1u << b);
          s2g(x_perm + (blockIdx.x + (j0 + i) * G) * (int64_t)D, buf(b), rb);
        }
      }
      commit();
    }
    set ^= 1;
  }
  if (lane == 0) {
    // after a timed-out wait (error recorded): the loads still in flight
    // land before the buffers go away (bounded)
    const uint64_t t0 = tc::global_ns();
    for (int b = 0; b < 2 * NB; ++b)
      if ((pend >> b) & 1u)
        while (!tc::mbar_try(bar(b), (ph >> b) & 1u) && tc::global_ns() - t0 < tc::kWaitLimitNs) {}
    wait_all();   // every store complete before the buffers go away
  }
  __syncwarp();
}

}  // namespace bulk
}  // namespace moe
