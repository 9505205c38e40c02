// Expert-choice routing ("08 MoE" STA324 notes §8.4: every expert picks a
// fixed number C of the batch's tokens; a token may be picked by several
// experts or by none).  Scores are the softmax router probabilities; expert
// e takes the C tokens with the largest p[t,e], equal scores going to the
// lower token; the gate weight is p[t,e] itself (no renormalisation).
//
// The layer runs it in the token-choice layout with one slot per (t, e)
// pair (K = E): topk_idx[t,e] = e, topk_w[t,e] = p[t,e], and the pairs an
// expert did not pick are sentinel slots.  The dispatch, the expert GEMMs
// and the weight gradients are then the token-choice ones; the kernels here
// are the choice itself and the per-token passes whose token-choice
// versions hold K values per lane (combine, router backward, dx).
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace moe {

// Per token: logits (from logits, or from the three tensor-core partial
// logit blocks parts [T, 3 Ep]), probs = softmax, lse, and the slot-form
// routing outputs.  Lane l holds experts l + 32 i.
template <int NV>
__global__ void __launch_bounds__(256)
ec_scores_kernel(const float* __restrict__ parts, int Ep, const float* __restrict__ offset,
                 int T, int E, float* __restrict__ logits, float* __restrict__ probs,
                 float* __restrict__ lse, int32_t* __restrict__ topk_idx,
                 float* __restrict__ topk_w) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < T; t += (int64_t)gridDim.x * 8) {
    float s[NV];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      s[i] = -INFINITY;
      if (e < E) {
        if (parts != nullptr) {
          const float* pr = parts + t * 3 * Ep;
          s[i] = (pr[e] + pr[Ep + e]) + pr[2 * Ep + e];
          if (offset != nullptr) s[i] += offset[e];
          logits[t * E + e] = s[i];
        } else {
          s[i] = logits[t * E + e];
        }
        m = fmaxf(m, s[i]);
      }
    }
    m = warp_max(m);
    float z = 0.f, ex[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      ex[i] = (lane + 32 * i < E) ? expf(s[i] - m) : 0.f;
      z += ex[i];
    }
    z = warp_sum(z);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        const float p = ex[i] / z;
        probs[t * E + e] = p;
        topk_w[t * E + e] = p;
        topk_idx[t * E + e] = e;
      }
    }
    if (lane == 0) lse[t] = m + logf(z);
  }
}

// One block per expert: the C-th largest probability v* by a radix select
// on its bits (probabilities are >= 0, so the bits order like the values),
// then the choice: p > v*, plus the first C - #(p > v*) tokens with p = v*
// in token order.  Writes the sentinel mask of the column (1 = not picked)
// and counts a near-tie when the C-th and (C+1)-th values differ by less
// than kNearTie.
constexpr int kEcThreads = 1024;
__global__ void __launch_bounds__(kEcThreads)
ec_select_kernel(const float* __restrict__ probs, int T, int E, int C,
                 uint8_t* __restrict__ sentinel_mask, int32_t* __restrict__ near_ties) {
  pdl_begin();
  __shared__ int32_t hist[256];
  __shared__ uint32_t prefix_s;
  __shared__ int32_t k_s;
  __shared__ int32_t wsum[kEcThreads / 32];
  __shared__ float vmax_w[kEcThreads / 32];
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int k = C;                             // rank (1-based) of v* among the remaining keys
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const uint32_t b = __float_as_uint(probs[(int64_t)t * E + e]);
      if ((b & mask) == prefix) atomicAdd(&hist[(b >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int run = 0, d = 255;
      for (; d > 0; --d) {
        if (run + hist[d] >= k) break;
        run += hist[d];
      }
      k_s = k - run;
      prefix_s = prefix | ((uint32_t)d << shift);
    }
    __syncthreads();
    k = k_s;
    prefix = prefix_s;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t vstar = prefix;         // bits of the C-th largest value
  // ties at v*: the first `k` of them in token order are picked
  int seen = 0;                          // ties before this chunk
  float vmax = -INFINITY;                // largest value below v*
  int n_ge = 0;
  for (int t0 = 0; t0 < T; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    uint32_t b = 0;
    if (t < T) b = __float_as_uint(probs[(int64_t)t * E + e]);
    const bool tie = t < T && b == vstar;
    if (t < T && b < vstar) vmax = fmaxf(vmax, __uint_as_float(b));
    // exclusive count of ties in this chunk before t (warp ballot + warp sums)
    const unsigned bal = __ballot_sync(0xffffffffu, tie);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = seen;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    before += __popc(bal & ((1u << lane) - 1u));
    int chunk = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) chunk += wsum[w];
    if (t < T) {
      const bool pick = b > vstar || (tie && before < k);
      sentinel_mask[(int64_t)t * E + e] = pick ? 0 : 1;
      if (b >= vstar) ++n_ge;
    }
    seen += chunk;
    __syncthreads();
  }
  // near-tie: the (C+1)-th value is v* itself (more than C values >= v*) or
  // the largest value below v*
  vmax = warp_max(vmax);
  if (lane == 0) vmax_w[warp] = vmax;
  int ge = n_ge;
  for (int o = 16; o > 0; o >>= 1) ge += __shfl_xor_sync(0xffffffffu, ge, o);
  if (lane == 0) wsum[warp] = ge;
  __syncthreads();
  if (threadIdx.x == 0 && C < T) {
    float vm = -INFINITY;
    int tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      vm = fmaxf(vm, vmax_w[w]);
      tot += wsum[w];
    }
    const float margin = tot > C ? 0.f : __uint_as_float(vstar) - vm;
    if (margin < kNearTie) atomicAdd(near_ties, 1);
  }
}

// A token's picked slots in increasing e, compacted into the warp's shared
// list (rows, and gate weights when g != nullptr); returns their number.
constexpr int kEcBatch = 8;   // picked rows whose loads are in flight together
__device__ __forceinline__ int ec_picks(const int32_t* __restrict__ slot_row,
                                       const float* __restrict__ g, int64_t t, int E,
                                       int32_t* rows, float* gs) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int n = 0;
  __syncwarp();   // the previous token's list has been read
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const int32_t r = e < E ? slot_row[t * E + e] : -1;
    const unsigned bal = __ballot_sync(0xffffffffu, r >= 0);
    if (r >= 0) {
      const int pos = n + __popc(bal & lt);
      rows[pos] = r;
      if (g != nullptr) gs[pos] = g[t * E + e];
    }
    n += __popc(bal);
  }
  __syncwarp();
  return n;
}

// acc += sum over the n listed rows (in list order) of w_i * src[row_i, d..d+7]
// (w_i = 1 when gs == nullptr).  The loads of kEcBatch rows are issued
// unconditionally (a slot past the list reads the first listed row, or row
// 0) before any is used, so they are in flight together.
template <typename TX>
__device__ __forceinline__ void ec_accumulate(const TX* __restrict__ src, int64_t D, int d,
                                              bool act, int n, const int32_t* rows,
                                              const float* gs, float (&acc)[8]) {
  const int dd = act ? d : 0;
  for (int i0 = 0; i0 < n; i0 += kEcBatch) {
    Raw8<TX> raw[kEcBatch];
#pragma unroll
    for (int j = 0; j < kEcBatch; ++j) {
      const int64_t r = i0 + j < n ? rows[i0 + j] : rows[0];
      raw[j].load(src + r * D + dd);
    }
#pragma unroll
    for (int j = 0; j < kEcBatch; ++j) {
      if (i0 + j < n) {
        float v[8];
        raw[j].widen(v);
        if (gs != nullptr) {
          const float w = gs[i0 + j];
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = fmaf(w, v[k], acc[k]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] += v[k];
        }
      }
    }
  }
}

// y_t = sum over the experts that picked t (increasing e) of p[t,e] o[row]
// (+ the shared row).  One warp per token: its picked slots are compacted
// into a shared list once, then every lane adds 8 columns of each listed
// row, kEcBatch rows' loads at a time.
template <typename TX>
__global__ void __launch_bounds__(256)
ec_combine_kernel(const TX* __restrict__ o, const int32_t* __restrict__ slot_row,
                  const float* __restrict__ topk_w, const int32_t* __restrict__ offsets,
                  int n_shared, int T, int D, int E, TX* __restrict__ y) {
  pdl_begin();
  __shared__ int32_t rows_s[8][kMaxExperts];
  __shared__ float g_s[8][kMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t shared0 = n_shared ? (int64_t)offsets[E] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < T; t += (int64_t)gridDim.x * 8) {
    const int n = ec_picks(slot_row, topk_w, t, E, rows_s[warp], g_s[warp]);
    for (int d0 = 0; d0 < D; d0 += 256) {
      const int d = d0 + lane * 8;
      const bool act = d < D;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      ec_accumulate(o, D, d, act, n, rows_s[warp], g_s[warp], acc);
      if (act) {
        if (shared0 >= 0) {
          float v[8];
          load8(o + (shared0 + t) * D + d, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += v[i];
        }
        store8(y + t * D + d, acc);
      }
    }
  }
}

// dx_t = router term + sum over the rows of the experts that picked t
// (increasing e) + the shared row.  Router term: R[t,:] (fp32, from the
// tensor-core product) when R is given, else sum_e ds[t,e] w_r[e,:].
template <typename TX>
__global__ void __launch_bounds__(256)
ec_dx_kernel(const float* __restrict__ R, const float* __restrict__ ds,
             const float* __restrict__ w_r, const TX* __restrict__ dXp,
             const int32_t* __restrict__ slot_row, const int32_t* __restrict__ offsets,
             int n_shared, int T, int D, int E, TX* __restrict__ dx) {
  pdl_begin();
  __shared__ int32_t rows_s[8][kMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t shared0 = n_shared ? (int64_t)offsets[E] : -1;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < T; t += (int64_t)gridDim.x * 8) {
    const int n = ec_picks(slot_row, nullptr, t, E, rows_s[warp], nullptr);
    for (int d0 = 0; d0 < D; d0 += 256) {
      const int d = d0 + lane * 8;
      const bool act = d < D;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (act) {
        if (R != nullptr) {
          load8(R + t * D + d, acc);
        } else {
          for (int e = 0; e < E; ++e) {
            const float c = ds[t * E + e];
            float w[8];
            load8(w_r + (int64_t)e * D + d, w);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(c, w[i], acc[i]);
          }
        }
      }
      ec_accumulate(dXp, D, d, act, n, rows_s[warp], nullptr, acc);
      if (act) {
        if (shared0 >= 0) {
          float v[8];
          load8(dXp + (shared0 + t) * D + d, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += v[i];
        }
        store8(dx + t * D + d, acc);
      }
    }
  }
}

// Router backward of expert choice: dp[t,e] = dg[t,e] on picked pairs (the
// gate weight is p itself), ds = p (dp - <p, dp>) + the z-loss term; also
// dg_out, dlogits and the bf16 splits of ds for the tensor-core products.
template <int NV>
__global__ void __launch_bounds__(256)
ec_router_bwd_kernel(const float* __restrict__ probs, const float* __restrict__ logits,
                     const float* __restrict__ lse, const int32_t* __restrict__ slot_row,
                     const float* __restrict__ dg_slot, int T, int E, float z_lambda,
                     float* __restrict__ ds_out, float* __restrict__ dlogits_out,
                     float* __restrict__ dg_out, __nv_bfloat16* __restrict__ dsf,
                     __nv_bfloat16* __restrict__ dsb, int Ep) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t t = (int64_t)blockIdx.x * 8 + warp; t < T; t += (int64_t)gridDim.x * 8) {
    float p[NV], dp[NV], inner = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      p[i] = 0.f;
      dp[i] = 0.f;
      if (e < E) {
        p[i] = probs[t * E + e];
        const int64_t j = t * E + e;
        dp[i] = slot_row[j] >= 0 ? dg_slot[j] : 0.f;
        if (dg_out != nullptr) dg_out[j] = dp[i];
      }
      inner += p[i] * dp[i];
    }
    inner = warp_sum(inner);
    float ds[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) ds[i] = p[i] * (dp[i] - inner);
    if (z_lambda != 0.f) {
      const float l = lse[t];
      const float c = 2.f * z_lambda * l / (float)T;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (e < E) ds[i] += c * expf(logits[t * E + e] - l);
      }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        ds_out[t * E + e] = ds[i];
        if (dlogits_out != nullptr) dlogits_out[t * E + e] = ds[i];
      }
    }
    if (dsf != nullptr) {
      const int64_t b = t * 3 * (int64_t)Ep;
      const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
          __nv_bfloat16 hi, mid, lo;
          split3_bf16(ds[i], hi, mid, lo);
          dsf[b + e] = hi; dsf[b + Ep + e] = mid; dsf[b + 2 * Ep + e] = lo;
          dsb[b + e] = hi; dsb[b + Ep + e] = hi; dsb[b + 2 * Ep + e] = mid;
        }
      }
      for (int e = E + lane; e < Ep; e += 32) {
        dsf[b + e] = zero; dsf[b + Ep + e] = zero; dsf[b + 2 * Ep + e] = zero;
        dsb[b + e] = zero; dsb[b + Ep + e] = zero; dsb[b + 2 * Ep + e] = zero;
      }
    }
  }
}

}  // namespace moe
