// Combine and the memory-bound parts of the backward.
//
// Combine: y_t = sum_{k kept} g_{t,k} o[row(t,k)] (+ shared expert row),
// the weighted sum of the "8-MoE" lecture notes (Router / Gating Network:
// y = sum_i G(x)_i E_i(x)) and STA324 notes "08 MoE" §8.7-§8.8 (a token
// appears K times so its outputs accumulate; the shared expert is added
// unweighted).  A gather in fixed k order: deterministic, no atomics.
//
// Gate gradient: dL/dg_{t,k} = <o_{t,k}, dy_t> for kept slots only.  The
// transformers batched_mm issue (cause analysis) shows why: the gradient of
// a sample weight is the expert output, so a slot with no local expert
// (sentinel) must contribute a zero expert output; dropped slots likewise.
//
// Router backward: STA324 §8.3 (fixed selected set, g differentiable in the
// logits; for K=1 variant B the weight is the constant 1), §8.5 (aux
// gradient alpha*E*f_e/T with f constant), "8-MoE" ST-MoE (z-loss), and the
// MiniMind issue §2 (the gate weight is the router's only differentiable
// path).
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace moe {

template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ o, const int32_t* __restrict__ slot_row,
               const float* __restrict__ topk_w, const int32_t* __restrict__ offsets,
               int n_shared, int Tn, int D, int K, int E, T* __restrict__ y) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < Tn; t += (int64_t)gridDim.x * 8) {
    int64_t rows[kMaxK];
    float g[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
      rows[k] = -1;
      g[k] = 0.f;
      if (k < K) {
        rows[k] = slot_row[t * K + k];
        g[k] = topk_w[t * K + k];
      }
    }
    const int64_t srow = n_shared ? (int64_t)offsets[E] + t : -1;
    for (int d = lane * 8; d < D; d += 256) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {
        if (k < K && rows[k] >= 0) {
          float v[8];
          load8(o + rows[k] * D + d, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(g[k], v[i], acc[i]);
        }
      }
      if (srow >= 0) {
        float v[8];
        load8(o + srow * D + d, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += v[i];
      }
      store8(y + t * D + d, acc);
    }
  }
}

// bf16 combine for a compile-time K: one warp per token, each lane 8
// columns of two 256-column chunks per step, with the K row loads of both
// chunks in flight together (the row indices are read once per token and
// broadcast).  Same fixed k order and fp32 accumulation as combine_kernel.
template <int KT>
__global__ void __launch_bounds__(256)
combine_bf16_kernel(const __nv_bfloat16* __restrict__ o, const int32_t* __restrict__ slot_row,
                    const float* __restrict__ topk_w, const int32_t* __restrict__ offsets,
                    int n_shared, int Tn, int D, int E, __nv_bfloat16* __restrict__ y) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t shared0 = n_shared ? (int64_t)offsets[E] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < Tn; t += (int64_t)gridDim.x * 8) {
    int32_t my_row = -1;
    float my_g = 0.f;
    if (lane < KT) {
      my_row = slot_row[t * KT + lane];
      my_g = topk_w[t * KT + lane];
    }
    int32_t rows[KT];
    float g[KT];
#pragma unroll
    for (int k = 0; k < KT; ++k) {
      rows[k] = __shfl_sync(0xffffffffu, my_row, k);
      g[k] = __shfl_sync(0xffffffffu, my_g, k);
    }
    const int64_t srow = n_shared ? shared0 + t : -1;
    for (int d0 = lane * 8; d0 < D; d0 += 512) {
      const int d1 = d0 + 256;
      const bool has1 = d1 < D;
      uint4 r0[KT + 1], r1[KT + 1];
#pragma unroll
      for (int k = 0; k <= KT; ++k) {
        const int64_t row = k < KT ? (int64_t)rows[k] : srow;
        r0[k] = make_uint4(0, 0, 0, 0);
        r1[k] = make_uint4(0, 0, 0, 0);
        if (row >= 0) {
          r0[k] = *reinterpret_cast<const uint4*>(o + row * D + d0);
          if (has1) r1[k] = *reinterpret_cast<const uint4*>(o + row * D + d1);
        }
      }
      float a0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float a1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < KT; ++k) {
        if (rows[k] >= 0) {
          float v[8];
          const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&r0[k]);
          const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&r1[k]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h0[i]);
            v[2 * i] = f.x; v[2 * i + 1] = f.y;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) a0[i] = fmaf(g[k], v[i], a0[i]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h1[i]);
            v[2 * i] = f.x; v[2 * i + 1] = f.y;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) a1[i] = fmaf(g[k], v[i], a1[i]);
        }
      }
      if (srow >= 0) {
        float v[8];
        const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&r0[KT]);
        const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&r1[KT]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h0[i]);
          v[2 * i] = f.x; v[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) a0[i] += v[i];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h1[i]);
          v[2 * i] = f.x; v[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) a1[i] += v[i];
      }
      store8(y + t * D + d0, a0);
      if (has1) store8(y + t * D + d1, a1);
    }
  }
}

// bf16 combine for K <= 2: as combine_bf16_kernel, with four 256-column
// chunks per step (more row loads in flight per warp for few rows per
// token).  Same fixed k order and fp32 accumulation.
template <int KT>
__global__ void __launch_bounds__(256, 2)
combine_bf16_wide_kernel(const __nv_bfloat16* __restrict__ o, const int32_t* __restrict__ slot_row,
                    const float* __restrict__ topk_w, const int32_t* __restrict__ offsets,
                    int n_shared, int Tn, int D, int E, __nv_bfloat16* __restrict__ y) {
  pdl_begin();
  constexpr int NC = 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t shared0 = n_shared ? (int64_t)offsets[E] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < Tn; t += (int64_t)gridDim.x * 8) {
    int32_t my_row = -1;
    float my_g = 0.f;
    if (lane < KT) {
      my_row = slot_row[t * KT + lane];
      my_g = topk_w[t * KT + lane];
    }
    int64_t rows[KT + 1];
    float g[KT];
#pragma unroll
    for (int k = 0; k < KT; ++k) {
      rows[k] = __shfl_sync(0xffffffffu, my_row, k);
      g[k] = __shfl_sync(0xffffffffu, my_g, k);
    }
    rows[KT] = n_shared ? shared0 + t : -1;
    for (int d0 = lane * 8; d0 < D; d0 += 256 * NC) {
      uint4 r[NC][KT + 1];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int d = d0 + 256 * c;
#pragma unroll
        for (int k = 0; k <= KT; ++k)
          r[c][k] = (rows[k] >= 0 && d < D) ? *reinterpret_cast<const uint4*>(o + rows[k] * D + d)
                                            : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int d = d0 + 256 * c;
        if (d >= D) continue;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < KT; ++k) {
          if (rows[k] >= 0) {
            float v[8];
            bf16x8_to_f32(r[c][k], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = fmaf(g[k], v[i], a[i]);
          }
        }
        if (rows[KT] >= 0) {
          float v[8];
          bf16x8_to_f32(r[c][KT], v);
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] += v[i];
        }
        store8(y + t * D + d, a);
      }
    }
  }
}

// Per permuted row: routed rows -> dg[slot] = <o[r], dy[t]> and
// dO[r] = g * dy[t]; shared rows -> dO[r] = dy[t]; padding -> 0.  A row's
// kind is decided by row_slot alone (the dispatch sets -1 on padding and
// shared rows), so each warp's chain is one index load then the row work.
// 256-column steps of a row whose loads are batched (rows of up to
// 256 * kRowBatch elements need one round trip to memory).
constexpr int kRowBatch = 4;

template <typename T>
__global__ void __launch_bounds__(256)
bwd_rows_kernel(const T* __restrict__ o, const T* __restrict__ dy,
                const float* __restrict__ topk_w, const int32_t* __restrict__ row_slot,
                const int32_t* __restrict__ offsets, const int32_t* __restrict__ stats,
                int K, int E, int Tn, int D, float* __restrict__ dg_slot,
                T* __restrict__ dO) {
  pdl_begin();
  const int n_rows = stats[2];
  const int64_t shared0 = offsets[E];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t r = (int64_t)blockIdx.x * 8 + warp; r < n_rows; r += (int64_t)gridDim.x * 8) {
    const int64_t slot = row_slot[r];
    int64_t t = -1;
    if (slot >= 0) t = slot / K;
    else if (r >= shared0 && r - shared0 < Tn) t = r - shared0;
    T* dst = dO + r * D;
    if (t < 0) {
      for (int d = lane * 8; d < D; d += 256) zero8(dst + d);
      continue;
    }
    const float g = slot >= 0 ? topk_w[slot] : 1.0f;
    float dot = 0.f;
    // kRowBatch 256-column steps per batch: every load of the batch is
    // issued (unconditionally, clamped to the row) before any is used
    for (int d0 = 0; d0 < D; d0 += 256 * kRowBatch) {
      Raw8<T> rd[kRowBatch], ro[kRowBatch];
#pragma unroll
      for (int j = 0; j < kRowBatch; ++j) {
        const int d = d0 + 256 * j + lane * 8;
        const int dc = d < D ? d : lane * 8;
        rd[j].load(dy + t * D + dc);
        ro[j].load(o + r * D + dc);
      }
#pragma unroll
      for (int j = 0; j < kRowBatch; ++j) {
        const int d = d0 + 256 * j + lane * 8;
        if (d < D) {
          float dv[8], ov[8];
          rd[j].widen(dv);
          if (slot >= 0) {
            ro[j].widen(ov);
#pragma unroll
            for (int i = 0; i < 8; ++i) dot = fmaf(ov[i], dv[i], dot);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) dv[i] *= g;
          store8(dst + d, dv);
        }
      }
    }
    if (slot >= 0) {
      dot = warp_sum(dot);
      if (lane == 0) dg_slot[slot] = dot;
    }
  }
}

// The gate-gradient pass in token order (bf16, K in {1, 2, 4, 8}): each
// token's dy row is read once; for each kept slot k, dg[slot] = <o[row_k],
// dy_t> (the same per-row accumulation order as bwd_rows_kernel) and
// dO[row_k] = g_k dy_t; the shared expert's row gets dO = dy_t; then the
// padding rows of dO are zeroed.
template <int KT>
__global__ void __launch_bounds__(256)
bwd_tok_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dy,
               const float* __restrict__ topk_w, const int32_t* __restrict__ slot_row,
               const int32_t* __restrict__ row_slot, const int32_t* __restrict__ offsets,
               const int32_t* __restrict__ stats, int n_shared, int El, int Tn, int D,
               float* __restrict__ dg_slot, __nv_bfloat16* __restrict__ dO) {
  pdl_begin();
  constexpr int NB = KT == 1 ? 4 : KT == 2 ? 2 : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t shared0 = n_shared ? (int64_t)offsets[El] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < Tn; t += (int64_t)gridDim.x * 8) {
    int32_t my_row = -1;
    float my_g = 0.f;
    if (lane < KT) {
      my_row = slot_row[t * KT + lane];
      my_g = topk_w[t * KT + lane];
    }
    int64_t rows[KT];
    float g[KT], dot[KT];
#pragma unroll
    for (int k = 0; k < KT; ++k) {
      rows[k] = __shfl_sync(0xffffffffu, my_row, k);
      g[k] = __shfl_sync(0xffffffffu, my_g, k);
      dot[k] = 0.f;
    }
    const int64_t srow = n_shared ? shared0 + t : -1;
    for (int d0 = lane * 8; d0 < D; d0 += 256 * NB) {
      Raw8<__nv_bfloat16> rd[NB], ro[NB][KT];
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const int d = d0 + 256 * j;
        const int dc = d < D ? d : lane * 8;
        rd[j].load(dy + t * D + dc);
#pragma unroll
        for (int k = 0; k < KT; ++k)
          if (rows[k] >= 0) ro[j][k].load(o + rows[k] * D + dc);
      }
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const int d = d0 + 256 * j;
        if (d >= D) continue;
        float dv[8];
        rd[j].widen(dv);
#pragma unroll
        for (int k = 0; k < KT; ++k) {
          if (rows[k] >= 0) {
            float ov[8], w[8];
            ro[j][k].widen(ov);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              dot[k] = fmaf(ov[i], dv[i], dot[k]);
              w[i] = dv[i] * g[k];
            }
            store8(dO + rows[k] * D + d, w);
          }
        }
        if (srow >= 0) store8(dO + srow * D + d, dv);
      }
    }
#pragma unroll
    for (int k = 0; k < KT; ++k) {
      const float v = warp_sum(dot[k]);
      if (lane == 0 && rows[k] >= 0) dg_slot[t * KT + k] = v;
    }
  }
  zero_padding_rows(dO, stats[2], D, row_slot, shared0, n_shared ? Tn : 0);
}

struct RouterBwdArgs {
  int T, E, K;
  int score_fn, renorm;
  float route_scale, aux_alpha, z_lambda;
  const float* logits;     // [T,E]
  const float* probs;      // [T,E]
  const float* lse;        // [T]
  const int32_t* topk_idx; // [T,K]
  const float* topk_w;     // [T,K]
  const int32_t* slot_row; // [T*K]
  const float* dg_slot;    // [T*K] (valid where slot_row >= 0)
  const int32_t* counts;   // [E]
  float* ds;               // [T,E]
  float* dlogits_out;      // [T,E] or null
  float* dg_out;           // [T,K] or null
  // sequence-wise aux (seq_len > 0): f[s][e] per sequence
  int seq_len;
  const float* seq_f;
  // bf16 splits of ds for the tensor-core router products (or null):
  // dsf [T, 3 Ep] = (hi | mid | lo), dsb [T, 3 Ep] = (hi | hi | mid) (or
  // null: the router part of dx is formed on CUDA cores)
  __nv_bfloat16* dsf;
  __nv_bfloat16* dsb;
  int Ep;
  float Tn;                // tokens the batch aux and z losses average over (T, or the
                           // data-parallel global count)
};

template <int NV>
__global__ void __launch_bounds__(256)
router_bwd_kernel(RouterBwdArgs a) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, K = a.K;
  float cnt_tot = 0.f;
  if (a.aux_alpha != 0.f) {
    for (int e = lane; e < E; e += 32) cnt_tot += (float)a.counts[e];
    cnt_tot = warp_sum(cnt_tot);
  }
  const float rs = a.route_scale;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < a.T; t += (int64_t)gridDim.x * 8) {
    float dgk[kMaxK], gk[kMaxK];
    int ik[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
      dgk[k] = 0.f; gk[k] = 0.f; ik[k] = -1;
      if (k < K) {
        const int64_t j = t * K + k;
        ik[k] = a.topk_idx[j];
        gk[k] = a.topk_w[j];
        dgk[k] = a.slot_row[j] >= 0 ? a.dg_slot[j] : 0.f;
      }
    }
    float p[NV], ds[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      p[i] = e < E ? a.probs[t * E + e] : 0.f;
      ds[i] = 0.f;
    }
    if (a.score_fn == MOE_SOFTMAX) {
      float dp[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (a.aux_alpha != 0.f && a.seq_len > 0)
          dp[i] = e < E ? a.aux_alpha * (float)E * a.seq_f[(t / a.seq_len) * E + e] /
                              (float)a.T
                        : 0.f;
        else
          dp[i] = (a.aux_alpha != 0.f && e < E && cnt_tot > 0.f)
                      ? a.aux_alpha * (float)E * ((float)a.counts[e] / cnt_tot) / a.Tn
                      : 0.f;
      }
      if (!a.renorm) {
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
          if (k < K && ik[k] >= 0 && (ik[k] & 31) == lane) {
#pragma unroll
            for (int i = 0; i < NV; ++i) if (i == (ik[k] >> 5)) dp[i] += rs * dgk[k];
          }
        }
      }
      float inner = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) inner += p[i] * dp[i];
      inner = warp_sum(inner);
#pragma unroll
      for (int i = 0; i < NV; ++i) ds[i] = p[i] * (dp[i] - inner);
      if (a.renorm) {
        float innerB = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxK; ++k)
          if (k < K && ik[k] >= 0) innerB += (gk[k] / rs) * (rs * dgk[k]);
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
          if (k < K && ik[k] >= 0 && (ik[k] & 31) == lane) {
            const float add = (gk[k] / rs) * (rs * dgk[k] - innerB);
#pragma unroll
            for (int i = 0; i < NV; ++i) if (i == (ik[k] >> 5)) ds[i] += add;
          }
        }
      }
    } else {
      float S = 0.f, innerS = 0.f;
      float sp[kMaxK];
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {
        sp[k] = 0.f;
        if (k < K && ik[k] >= 0) {
          sp[k] = a.probs[t * E + ik[k]];
          S += sp[k];
          innerS += dgk[k] * gk[k];
        }
      }
      S += 1e-20f;
      innerS /= rs;
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) {
        if (k < K && ik[k] >= 0 && (ik[k] & 31) == lane) {
          const float dsig = a.renorm ? rs / S * (dgk[k] - innerS) : rs * dgk[k];
          const float add = dsig * sp[k] * (1.f - sp[k]);
#pragma unroll
          for (int i = 0; i < NV; ++i) if (i == (ik[k] >> 5)) ds[i] += add;
        }
      }
    }
    if (a.score_fn != MOE_SOFTMAX && a.aux_alpha != 0.f && a.seq_len > 0) {
      // sequence-wise aux on q = sigma / sum sigma: dq = alpha E f / T,
      // dsigma = (dq - <dq, q>) / sum sigma, ds += dsigma sigma (1 - sigma)
      float S = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) S += p[i];
      S = warp_sum(S);
      float dq[NV], inner = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        dq[i] = e < E ? a.aux_alpha * (float)E * a.seq_f[(t / a.seq_len) * E + e] / (float)a.T
                      : 0.f;
        inner += dq[i] * (p[i] / S);
      }
      inner = warp_sum(inner);
#pragma unroll
      for (int i = 0; i < NV; ++i) ds[i] += (dq[i] - inner) / S * p[i] * (1.f - p[i]);
    }
    if (a.z_lambda != 0.f) {
      const float l = a.lse[t];
      const float c = 2.f * a.z_lambda * l / a.Tn;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (e < E) ds[i] += c * expf(a.logits[t * E + e] - l);
      }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        a.ds[t * E + e] = ds[i];
        if (a.dlogits_out) a.dlogits_out[t * E + e] = ds[i];
      }
    }
    if (a.dsf != nullptr) {
      const int64_t b = t * 3 * (int64_t)a.Ep;
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
          __nv_bfloat16 hi, mid, lo;
          split3_bf16(ds[i], hi, mid, lo);
          a.dsf[b + e] = hi; a.dsf[b + a.Ep + e] = mid; a.dsf[b + 2 * a.Ep + e] = lo;
          if (a.dsb != nullptr) {
            a.dsb[b + e] = hi; a.dsb[b + a.Ep + e] = hi; a.dsb[b + 2 * a.Ep + e] = mid;
          }
        }
      }
      for (int e = E + lane; e < a.Ep; e += 32) {
        a.dsf[b + e] = z; a.dsf[b + a.Ep + e] = z; a.dsf[b + 2 * a.Ep + e] = z;
        if (a.dsb != nullptr) {
          a.dsb[b + e] = z; a.dsb[b + a.Ep + e] = z; a.dsb[b + 2 * a.Ep + e] = z;
        }
      }
    }
    if (a.dg_out != nullptr && lane < K) {
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxK; ++k) if (k == lane) v = dgk[k];
      a.dg_out[t * K + lane] = v;
    }
  }
}

// dW_r partials: part[c][e][d] = sum_{t in chunk c} ds[t,e] x[t,d].
// Block tile BE x BD, thread tile TE x TD, token steps of 32.
template <typename TX, int BE, int BD, int TE, int TD>
__global__ void __launch_bounds__(256)
dwr_partial_kernel(const float* __restrict__ ds, const TX* __restrict__ x,
                   int Tn, int E, int D, int chunk, float* __restrict__ part) {
  pdl_begin();
  static_assert((BE / TE) * (BD / TD) == 256, "thread tile");
  __shared__ __align__(16) float sds[32][BE + 4];
  __shared__ __align__(16) float sx[32][BD + 4];
  const int tid = threadIdx.x;
  const int nd = BD / TD;
  const int td = tid % nd, te = tid / nd;
  const int d0 = blockIdx.x * BD, e0 = blockIdx.y * BE;
  const int64_t t_beg = (int64_t)blockIdx.z * chunk;
  const int64_t t_end = min(t_beg + chunk, (int64_t)Tn);
  float acc[TE][TD] = {};
  for (int64_t tb = t_beg; tb < t_end; tb += 32) {
    for (int i = tid; i < 32 * BE; i += 256) {
      const int r = i / BE, c = i % BE;
      const int64_t t = tb + r;
      sds[r][c] = (t < t_end && e0 + c < E) ? ds[t * E + e0 + c] : 0.f;
    }
    for (int i = tid * 8; i < 32 * BD; i += 256 * 8) {
      const int r = i / BD, c = i % BD;
      const int64_t t = tb + r;
      float v[8];
      if (t < t_end && d0 + c < D) load8(x + t * D + d0 + c, v);
      else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) sx[r][c + j] = v[j];
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 32; ++r) {
      float av[TE], bv[TD];
#pragma unroll
      for (int i = 0; i < TE; ++i) av[i] = sds[r][te * TE + i];
#pragma unroll
      for (int j = 0; j < TD; ++j) bv[j] = sx[r][td * TD + j];
#pragma unroll
      for (int i = 0; i < TE; ++i)
#pragma unroll
        for (int j = 0; j < TD; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TE; ++i) {
    const int e = e0 + te * TE + i;
    if (e >= E) continue;
#pragma unroll
    for (int j = 0; j < TD; ++j) {
      const int d = d0 + td * TD + j;
      if (d < D) part[((size_t)blockIdx.z * E + e) * D + d] = acc[i][j];
    }
  }
}

__global__ void __launch_bounds__(256)
dwr_reduce_kernel(const float* __restrict__ part, int n_chunks, int64_t n,
                  float* __restrict__ dw_r) {
  pdl_begin();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int c = 0; c < n_chunks; ++c) s += part[(size_t)c * n + i];
    dw_r[i] = s;
  }
}

// dx[t,:] = sum_e ds[t,e] W_r[e,:] + sum_{k kept} dXp[row(t,k),:] (+ shared
// row).  64 tokens x 128 columns per block, 4 x 8 per thread.
template <typename T>
__global__ void __launch_bounds__(256)
dx_kernel(const float* __restrict__ ds, const float* __restrict__ w_r,
          const T* __restrict__ dXp, const int32_t* __restrict__ slot_row,
          const int32_t* __restrict__ offsets, int n_shared, int Tn, int D, int E,
          int K, T* __restrict__ dx) {
  pdl_begin();
  constexpr int BT = 64, BD = 128, BK = 16;
  __shared__ __align__(16) float sds[BK][BT + 4];
  __shared__ __align__(16) float sw[BK][BD + 4];
  const int tid = threadIdx.x;
  const int td = tid & 15, tt = tid >> 4;   // 16 x 16 threads: 8 cols, 4 tokens
  const int64_t t0 = (int64_t)blockIdx.x * BT;
  const int d0 = blockIdx.y * BD;
  float acc[4][8] = {};
  for (int k0 = 0; k0 < E; k0 += BK) {
    for (int i = tid; i < BT * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      const int64_t t = t0 + r;
      sds[c][r] = (t < Tn && k0 + c < E) ? ds[t * E + k0 + c] : 0.f;
    }
    for (int i = tid; i < BK * BD; i += 256) {
      const int r = i / BD, c = i % BD;
      sw[r][c] = (k0 + r < E && d0 + c < D) ? w_r[(size_t)(k0 + r) * D + d0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float av[4], bv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = sds[k][tt * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) bv[j] = sw[k][td * 8 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int d = d0 + td * 8;
  if (d >= D) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + tt * 4 + i;
    if (t >= Tn) continue;
    for (int k = 0; k < K; ++k) {
      const int64_t row = slot_row[t * K + k];
      if (row >= 0) {
        float v[8];
        load8(dXp + row * D + d, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] += v[j];
      }
    }
    if (n_shared) {
      float v[8];
      load8(dXp + ((int64_t)offsets[E] + t) * D + d, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] += v[j];
    }
    store8(dx + t * D + d, acc[i]);
  }
}

// ---------------------------------------------------------------------------
// Sequence-wise aux loss and the selection-bias update ([STA324] §8.5-§8.6,
// [TRAIN]).  One block per sequence of S tokens; every sum runs in a fixed
// order (per-warp token strides, then warps in order), so results do not
// depend on timing.
// ---------------------------------------------------------------------------
// Partial sums of one piece of a sequence (block (b, s): tokens
// [s S + b L, s S + (b+1) L) with L = ceil(S / gridDim.x)): slot counts per
// expert, sums of q per expert, sum of lse^2.  q = probs (softmax) or
// probs / sum_e probs (sigmoid); lane l of a warp holds experts l + 32 i.
template <int NV>
__global__ void __launch_bounds__(256)
seq_aux_partial_kernel(const float* __restrict__ probs, const float* __restrict__ lse,
                       const int32_t* __restrict__ topk_idx,
                       const int32_t* __restrict__ slot_row, int S, int K, int E,
                       int normalise, int32_t* __restrict__ cnt_part,
                       float* __restrict__ q_part, float* __restrict__ z_part) {
  pdl_begin();
  __shared__ int32_t cnt_s[kMaxExperts];
  __shared__ float pw[8][kMaxExperts];
  __shared__ float zw[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = gridDim.x, b = blockIdx.x;
  const int64_t s = blockIdx.y;
  const int L = (S + nb - 1) / nb;
  const int64_t t0 = s * S + (int64_t)b * L;
  const int64_t t1 = t0 + L < (s + 1) * S ? t0 + L : (s + 1) * S;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt_s[e] = 0;
  __syncthreads();
  for (int64_t j = t0 * K + threadIdx.x; j < t1 * K; j += blockDim.x) {
    const int e = topk_idx[j];
    if (slot_row[j] != -2 && e >= 0 && e < E) atomicAdd(&cnt_s[e], 1);
  }
  float acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = 0.f;
  float z = 0.f;
  for (int64_t t = t0 + warp; t < t1; t += 8) {
    float q[NV], rs = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      q[i] = e < E ? probs[t * E + e] : 0.f;
      rs += q[i];
    }
    if (normalise) {
      rs = warp_sum(rs);
#pragma unroll
      for (int i = 0; i < NV; ++i) q[i] /= rs;
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[i] += q[i];
    if (lane == 0) z += lse[t] * lse[t];
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    if (e < E) pw[warp][e] = acc[i];
  }
  if (lane == 0) zw[warp] = z;
  __syncthreads();
  const int64_t o = (s * nb + b) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float P = 0.f;
    for (int w = 0; w < 8; ++w) P += pw[w][e];
    q_part[o + e] = P;
    cnt_part[o + e] = cnt_s[e];
  }
  if (threadIdx.x == 0) {
    float zz = 0.f;
    for (int w = 0; w < 8; ++w) zz += zw[w];
    z_part[s * nb + b] = zz;
  }
}

// One block per sequence s: n and P from its pieces (summed in piece
// order), f = n / sum n, part[s] = sum_e f P (fixed-order block sums);
// f [n_seq, E] is written for the backward when f_out is given.
__global__ void __launch_bounds__(256)
seq_aux_seq_kernel(const int32_t* __restrict__ cnt_part, const float* __restrict__ q_part,
                   int nb, int S, int E, float* __restrict__ part,
                   float* __restrict__ f_out) {
  pdl_begin();
  __shared__ int32_t n_s[kMaxExperts];
  __shared__ float p_s[kMaxExperts];
  __shared__ float red[256];
  const int64_t s = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t n = 0;
    float P = 0.f;
#pragma unroll 8
    for (int b = 0; b < nb; ++b) {
      n += cnt_part[(s * nb + b) * E + e];
      P += q_part[(s * nb + b) * E + e];
    }
    n_s[e] = n;
    p_s[e] = P / (float)S;
  }
  __syncthreads();
  float tot = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) tot += (float)n_s[e];
  red[threadIdx.x] = tot;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  const float ntot = red[0];
  __syncthreads();
  float v = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float f = ntot > 0.f ? (float)n_s[e] / ntot : 0.f;
    if (f_out != nullptr) f_out[s * E + e] = f;
    v += f * p_s[e];
  }
  red[threadIdx.x] = v;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[s] = red[0];
}

// losses[0] = alpha E mean_s part[s], losses[1] = lambda mean_t lse^2
// (fixed-order block sums).
__global__ void __launch_bounds__(256)
seq_aux_final_kernel(const float* __restrict__ part, const float* __restrict__ z_part,
                     int n_seq, int n_z, int T, int E, float alpha, float lambda,
                     float* __restrict__ losses) {
  pdl_begin();
  __shared__ float red[2][256];
  float a = 0.f, z = 0.f;
  for (int i = threadIdx.x; i < n_seq; i += blockDim.x) a += part[i];
  for (int i = threadIdx.x; i < n_z; i += blockDim.x) z += z_part[i];
  red[0][threadIdx.x] = a;
  red[1][threadIdx.x] = z;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      red[0][threadIdx.x] += red[0][threadIdx.x + o];
      red[1][threadIdx.x] += red[1][threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    losses[0] = alpha * (float)E * red[0][0] / (float)n_seq;
    losses[1] = lambda * red[1][0] / (float)T;
  }
}

// b_e -= gamma * sign(n_e - mean n), the sign taken exactly on n_e*E - sum n
__global__ void __launch_bounds__(256)
bias_update_kernel(const int32_t* __restrict__ counts, int E, float gamma,
                   float* __restrict__ bias) {
  pdl_begin();
  __shared__ long long tot_s;
  if (threadIdx.x == 0) {
    long long t = 0;
    for (int e = 0; e < E; ++e) t += counts[e];
    tot_s = t;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const long long d = (long long)counts[e] * E - tot_s;
    if (d > 0) bias[e] -= gamma;
    else if (d < 0) bias[e] += gamma;
  }
}

// dx for few experts (E <= 8, bf16): dx_t = sum_e ds[t,e] W_r[e,:] (e
// ascending, fp32) + sum_{k kept} dX_perm[row(t,k),:] (k ascending) + the
// shared row.  A block has 16 warps, one per 256-column slice of the row (8
// columns per lane), and walks its token group; each lane keeps its 8
// columns of every expert's W_r row in registers for the whole launch.  The
// 16 warps take the same tokens in the same order, so the slices of one
// routed row are read close together in time (whole rows, as DRAM pages
// like).  A warp streams its tokens in stages of NB tokens through a ring
// of stages in shared memory filled by cp.async (16 bytes per lane per
// routed row, 4 bytes per ds value, zero-filled for dropped and sentinel
// slots); the slot rows of the stage issued next are loaded one iteration
// ahead.
template <int KT>
struct DxRing {
  static constexpr int NB = KT >= 4 ? 1 : 4 / KT;      // tokens per stage
  static constexpr int S = KT == 8 ? 2 : 4;             // stages per warp
  static constexpr int kRows = NB * KT * 512;           // routed rows, 16 B per lane
  static constexpr int kStage = kRows + NB * 8 * 4;     // + ds [NB][E <= 8] fp32
  static constexpr int kWarps = 16;
  static constexpr int kBytes = kWarps * S * kStage;
};
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async_zfill(uint32_t dst, const void* src, int bytes, bool valid) {
  if (bytes == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 4 : 0) : "memory");
}
// Packed pairs of fp32 lanes (sm_100: one instruction rounds each half as
// its scalar counterpart does, round to nearest, no flush to zero).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int KT>
__global__ void __launch_bounds__(512, 1)
dx_small_kernel(const float* __restrict__ ds, const float* __restrict__ w_r,
                const __nv_bfloat16* __restrict__ dXp, const int32_t* __restrict__ slot_row,
                const int32_t* __restrict__ offsets, int n_shared, int Tn, int D, int E, int El,
                __nv_bfloat16* __restrict__ dx) {
  pdl_begin();
  using R = DxRing<KT>;
  constexpr int kE = 8, NB = R::NB, S = R::S;
  extern __shared__ __align__(16) uint8_t dx_ring[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = blockIdx.x * R::kWarps + warp;
  if (slice * 256 >= D) return;            // a whole warp past the row (no block barrier)
  const int d = slice * 256 + lane * 8;
  const bool live = d < D;                 // (every lane of the warp takes part in its shuffles)
  uint64_t w[kE][4];                       // column pairs (2i, 2i + 1)
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    float f[8];
    if (live && e < E) {
      load8(w_r + (int64_t)e * D + d, f);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) w[e][i] = f2_pack(f[2 * i], f[2 * i + 1]);
  }
  const int64_t shared0 = n_shared ? (int64_t)offsets[El] : -1;
  const int64_t stride = gridDim.y;
  const int64_t first = blockIdx.y;                            // this block's tokens:
  const int64_t nt = first < Tn ? (Tn - 1 - first) / stride + 1 : 0;   // first + n stride
  const int64_t nst = (nt + NB - 1) / NB;                      // stages
  const uint32_t ring = smem_addr(dx_ring) + warp * S * R::kStage;
  // lane l < NB K: the row of slot l % K of the stage's token l / K
  auto stage_row = [&](int64_t st) -> int32_t {
    const int64_t n = st * NB + lane / KT;
    return (st < nst && lane < NB * KT && n < nt)
               ? slot_row[(first + n * stride) * KT + lane % KT] : -1;
  };
  auto issue = [&](int64_t st, int32_t my_row) {
    const uint32_t buf = ring + (uint32_t)(st % S) * R::kStage;
#pragma unroll
    for (int q = 0; q < NB * KT; ++q) {
      const int32_t row = __shfl_sync(0xffffffffu, my_row, q);
      const bool ok = live && row >= 0;
      cp_async_zfill(buf + q * 512 + lane * 16, dXp + (ok ? (int64_t)row * D + d : 0), 16, ok);
    }
    if (lane < NB * kE) {                  // ds of the stage's tokens
      const int j = lane / kE, e = lane % kE;
      const int64_t n = st * NB + j;
      const bool ok = st < nst && n < nt && e < E;
      cp_async_zfill(buf + R::kRows + lane * 4, ds + (ok ? (first + n * stride) * E + e : 0), 4, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // prologue: stages 0 .. S-2 in flight, the rows of stage S-1 loaded
#pragma unroll
  for (int st = 0; st < S - 1; ++st) issue(st, stage_row(st));
  int32_t next_row = stage_row(S - 1);
  for (int64_t st = 0; st < nst; ++st) {
    const int32_t my_row = next_row;
    next_row = stage_row(st + S);          // consumed next iteration
    issue(st + S - 1, my_row);             // (empty groups past the last stage)
    asm volatile("cp.async.wait_group %0;" ::"n"(S - 1) : "memory");
    __syncwarp();                          // every lane's copies of stage st landed
    const uint32_t buf = ring + (uint32_t)(st % S) * R::kStage;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int64_t n = st * NB + j;
      if (n >= nt) break;                  // warp-uniform
      const int64_t t = first + n * stride;
      // fp32 pairs: per column the same operations in the same order as
      // the scalar form acc = fma(ds_e, w_e, acc) (e ascending), acc += row
      // (k ascending)
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};   // (+0, +0)
#pragma unroll
      for (int e = 0; e < kE; ++e) {
        if (e < E) {
          float de;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(de) : "r"(buf + R::kRows + (j * kE + e) * 4));
          const uint64_t de2 = f2_pack(de, de);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc2[i] = f2_fma(de2, w[e][i], acc2[i]);
        }
      }
#pragma unroll
      for (int k = 0; k < KT; ++k) {
        uint4 u;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                     : "r"(buf + (j * KT + k) * 512 + lane * 16));
        float v[8];
        bf16x8_to_f32(u, v);               // dropped / sentinel slots: zeros
#pragma unroll
        for (int i = 0; i < 4; ++i) acc2[i] = f2_add(acc2[i], f2_pack(v[2 * i], v[2 * i + 1]));
      }
      float acc[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = f2_unpack(acc2[i]);
        acc[2 * i] = a.x;
        acc[2 * i + 1] = a.y;
      }
      if (!live) continue;
      if (shared0 >= 0) {                  // the shared expert's row, last
        float v[8];
        load8(dXp + (shared0 + t) * D + d, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += v[i];
      }
      store8(dx + t * D + d, acc);
    }
    __syncwarp();                          // stage st read before it is refilled
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// bf16 dx when the router part R = ds . W_r [T, D] fp32 comes from the
// tensor-core product: dx_t = R_t + sum_k dX_perm[row(t,k)] (k ascending) +
// the shared row.  One warp per token, each lane 8 columns of two
// 256-column chunks per step, every load of both chunks in flight together.
// KT = compile-time K (0: runtime K, up to 16, one chunk per step).
template <int KT>
__global__ void __launch_bounds__(256)
dx_sum_kernel(const float* __restrict__ R, const __nv_bfloat16* __restrict__ dXp,
              const int32_t* __restrict__ slot_row, const int32_t* __restrict__ offsets,
              int n_shared, int Tn, int D, int E, int K, __nv_bfloat16* __restrict__ dx) {
  pdl_begin();
  constexpr int NK = KT > 0 ? KT : 16;
  constexpr int NC = KT > 0 ? 2 : 1;        // 256-column chunks per step
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kk = KT > 0 ? KT : K;
  const int64_t shared0 = n_shared ? (int64_t)offsets[E] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < Tn; t += (int64_t)gridDim.x * 8) {
    const int32_t my_row = lane < kk ? slot_row[t * kk + lane] : -1;
    int32_t rows[NK + 1];
#pragma unroll
    for (int k = 0; k < NK; ++k) rows[k] = __shfl_sync(0xffffffffu, my_row, k);
    rows[NK] = n_shared ? (int32_t)(shared0 + t) : -1;
    for (int d0 = lane * 8; d0 < D; d0 += 256 * NC) {
      uint4 raw[NC][NK + 1];
      float acc[NC][8];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int d = d0 + 256 * c;
        if (d < D) load8(R + t * D + d, acc[c]);
#pragma unroll
        for (int k = 0; k <= NK; ++k) {
          raw[c][k] = make_uint4(0, 0, 0, 0);
          if ((k < kk || k == NK) && rows[k] >= 0 && d < D)
            raw[c][k] = *reinterpret_cast<const uint4*>(dXp + (int64_t)rows[k] * D + d);
        }
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int d = d0 + 256 * c;
        if (d >= D) break;
#pragma unroll
        for (int k = 0; k <= NK; ++k) {
          if ((k < kk || k == NK) && rows[k] >= 0) {
            float v[8];
            bf16x8_to_f32(raw[c][k], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[c][i] += v[i];
          }
        }
        store8(dx + t * D + d, acc[c]);
      }
    }
  }
}

// dW_r from the three partial products of the tensor-core path
// (part [3 Ep, D]: ds_hi^T x | ds_mid^T x | ds_lo^T x), summed in that order,
// for each of the n_split token ranges (partials n_split apart, 3 Ep D
// elements each), the ranges added in order.
__global__ void __launch_bounds__(256)
dwr_reduce3_kernel(const float* __restrict__ part, int E, int Ep, int D, int n_split,
                   float* __restrict__ dw_r) {
  pdl_begin();
  const int64_t n = (int64_t)E * D, stride = (int64_t)Ep * D, sstride = 3 * stride;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc = (part[i] + part[stride + i]) + part[2 * stride + i];
    for (int s = 1; s < n_split; ++s) {
      const float* q = part + s * sstride;
      acc += (q[i] + q[stride + i]) + q[2 * stride + i];
    }
    dw_r[i] = acc;
  }
}

}  // namespace moe
