// CUDA-core grouped GEMMs for the expert projections: the fp32 layer path
// (tensor cores have no exact-fp32 kind) and a cross-check of the tensor-core
// kernels.  64x64 output tile per block, 4x4 per thread, fp32 accumulation.
//
// ROWS mode (forward and data-gradient GEMMs): C[r, n] = sum_k A[r, k] *
// B_e(n, k) over the permuted rows r, with e the expert owning r's 128-row
// tile ("8-MoE" lecture notes, MoE 高效推理: each expert runs one dense batch
// of its own tokens; STA324 notes "08 MoE" §8.8: grouped GEMM, experts with
// no tokens are skipped).
// WGRAD mode (weight gradients): C_g[m, n] = sum_{r in rows(g)} A[r, m] *
// B[r, n] over the rows of group g (expert or shared).
#pragma once
#include "common.cuh"

namespace moe {

struct SimtGemm {
  // ROWS
  const void* A; int64_t lda;
  const void* B; int64_t sbn, sbk, strideBE;
  const void* Bs;                       // shared expert operand (group E)
  void* C; int64_t ldc;
  int N, Kd;
  const int32_t* tile_expert;
  const int32_t* stats;
  int E;
  // WGRAD
  int64_t ldb;
  int Mo, No;
  const int32_t* offsets;
  const int32_t* kept;
  int T;
  int64_t strideCE;
  void* Cs;
};

template <typename TE>
__global__ void __launch_bounds__(256)
simt_rows_kernel(SimtGemm g) {
  pdl_begin();
  __shared__ __align__(16) float As[16][64 + 4];
  __shared__ __align__(16) float Bs[16][64 + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t r0 = (int64_t)blockIdx.x * 64;
  if (r0 >= g.stats[2]) return;
  const int n0 = blockIdx.y * 64;
  const int e = g.tile_expert[r0 / kRowTile];
  const TE* A = static_cast<const TE*>(g.A);
  const TE* B = (e < g.E) ? static_cast<const TE*>(g.B) + (int64_t)e * g.strideBE
                          : static_cast<const TE*>(g.Bs);
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.Kd; k0 += 16) {
    for (int i = tid; i < 16 * 64; i += 256) {
      const int kk = i & 15, ii = i >> 4;
      As[kk][ii] = (k0 + kk < g.Kd) ? ld_f(A + (r0 + ii) * g.lda + k0 + kk) : 0.f;
      int j, kb;
      if (g.sbk == 1) { kb = i & 15; j = i >> 4; } else { j = i & 63; kb = i >> 6; }
      const int n = n0 + j, k = k0 + kb;
      Bs[kb][j] = (n < g.N && k < g.Kd) ? ld_f(B + (int64_t)n * g.sbn + (int64_t)k * g.sbk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[k][ty * 4 + i]; b[i] = Bs[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  TE* C = static_cast<TE*>(g.C);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < g.N) st_f(C + (r0 + ty * 4 + i) * g.ldc + n, acc[i][j]);
    }
}

template <typename TE>
__global__ void __launch_bounds__(256)
simt_wgrad_kernel(SimtGemm g) {
  pdl_begin();
  __shared__ __align__(16) float As[16][64 + 4];
  __shared__ __align__(16) float Bs[16][64 + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int grp = blockIdx.z;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int64_t row0 = g.offsets[grp];
  const int64_t rows = grp < g.E ? g.kept[grp] : g.T;
  const TE* A = static_cast<const TE*>(g.A);
  const TE* B = static_cast<const TE*>(g.B);
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < rows; k0 += 16) {
    for (int i = tid; i < 16 * 64; i += 256) {
      const int kk = i >> 6, c = i & 63;
      const int64_t r = row0 + k0 + kk;
      const bool rk = k0 + kk < rows;
      As[kk][c] = (rk && m0 + c < g.Mo) ? ld_f(A + r * g.lda + m0 + c) : 0.f;
      Bs[kk][c] = (rk && n0 + c < g.No) ? ld_f(B + r * g.ldb + n0 + c) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[k][ty * 4 + i]; b[i] = Bs[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  TE* C = grp < g.E ? static_cast<TE*>(g.C) + (int64_t)grp * g.strideCE
                    : static_cast<TE*>(g.Cs);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.Mo) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < g.No) st_f(C + (int64_t)m * g.No + n, acc[i][j]);
    }
  }
}

// h = silu(a) * b over the permuted rows (a13 = [a | b], row stride 2F).
template <typename TE>
__global__ void __launch_bounds__(256)
swiglu_fwd_kernel(const TE* __restrict__ a13, TE* __restrict__ h,
                  const int32_t* __restrict__ stats, int F) {
  pdl_begin();
  const int64_t n = (int64_t)stats[2] * F;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / F, j = i % F;
    const float a = ld_f(a13 + r * 2 * F + j), b = ld_f(a13 + r * 2 * F + F + j);
    st_f(h + i, silu_f(a) * b);
  }
}

// [da | db] from dh and the saved pre-activations.
template <typename TE>
__global__ void __launch_bounds__(256)
swiglu_bwd_kernel(const TE* __restrict__ dh, const TE* __restrict__ a13,
                  TE* __restrict__ da13, const int32_t* __restrict__ stats, int F) {
  pdl_begin();
  const int64_t n = (int64_t)stats[2] * F;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / F, j = i % F;
    const float a = ld_f(a13 + r * 2 * F + j), b = ld_f(a13 + r * 2 * F + F + j);
    const float d = ld_f(dh + i);
    const float s = sigmoid_f(a);
    st_f(da13 + r * 2 * F + j, d * b * s * (1.f + a * (1.f - s)));
    st_f(da13 + r * 2 * F + F + j, d * a * s);
  }
}

}  // namespace moe
