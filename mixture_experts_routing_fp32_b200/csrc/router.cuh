// Router: fp32 logits, softmax / sigmoid scores, group-limited top-K and
// gate weights (variants A and B).
//
// Follows "08 MoE" (STA324 notes) §8.2 (s = x W_r, TopK on the logits,
// variant A = truncate, variant B = softmax over the selected logits) and
// §8.6 (sigmoid affinities, selection-only bias b_e, weights from the raw
// affinity), the "8-MoE" lecture notes (router in full precision) and the
// MoE training course page (group-limited routing, optional scaling).
//
// One warp routes one token.  Lane l holds experts e = l + 32*i, i < NV.
#pragma once
#include "common.cuh"

namespace moe {

struct RouteArgs {
  int T, E, K;
  int score_fn, renorm;
  int n_groups, topk_groups, group_score;
  float route_scale;
  const float* sel_bias;   // [E] or null
  float* logits;           // [T,E] (written by the fused path only)
  float* probs;            // [T,E]
  float* lse;              // [T]
  int32_t* topk_idx;       // [T,K]
  float* topk_w;           // [T,K]
  int32_t* near_ties;      // [1]
};

constexpr int kMaxK = 16;

// (value, index) argmax across the warp: larger value wins, then lower index.
__device__ __forceinline__ void warp_argmax(float& v, int& e) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, v, o);
    int oe = __shfl_xor_sync(0xffffffffu, e, o);
    if (ov > v || (ov == v && oe < e)) { v = ov; e = oe; }
  }
}

template <int NV>
__device__ __forceinline__ float pick(const float (&a)[NV], int i) {
  float r = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) if (j == i) r = a[j];
  return r;
}

// Routes token t given its logits s[i] (expert lane + 32 i).  `gsm` is
// per-warp shared scratch of at least E floats (group-limited routing).
// KM: compile-time bound on K (the selection arrays are sized by it).
template <int NV, int KM = kMaxK>
__device__ void route_token(int t, float (&s)[NV], const RouteArgs& a,
                            float* gsm, int lane) {
  const int E = a.E;
  const float NEG = -INFINITY;
  // logsumexp (z-loss, and softmax normaliser)
  float m = NEG;
#pragma unroll
  for (int i = 0; i < NV; ++i) if (lane + 32 * i < E) m = fmaxf(m, s[i]);
  m = warp_max(m);
  float ex[NV];
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    ex[i] = (lane + 32 * i < E) ? expf(s[i] - m) : 0.f;
    z += ex[i];
  }
  z = warp_sum(z);
  const float lse = m + logf(z);
  float p[NV], u[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    if (a.score_fn == MOE_SOFTMAX) {
      p[i] = ex[i] / z;
      u[i] = s[i];
    } else {
      p[i] = 1.0f / (1.0f + expf(-s[i]));
      u[i] = p[i] + (a.sel_bias != nullptr && e < E ? a.sel_bias[e] : 0.f);
    }
    if (e >= E) u[i] = NEG;
    else a.probs[(size_t)t * E + e] = p[i];
  }
  if (lane == 0) a.lse[t] = lse;

  // group limit
  float gmargin = INFINITY;
  if (a.n_groups > 1) {
    const int gsz = E / a.n_groups;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E) gsm[e] = u[i];
    }
    __syncwarp();
    float gs = NEG;
    if (lane < a.n_groups) {
      float b1 = NEG, b2 = NEG;
      for (int j = 0; j < gsz; ++j) {
        const float v = gsm[lane * gsz + j];
        if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
      }
      gs = (a.group_score == MOE_GMAX) ? b1 : b1 + b2;
    }
    __syncwarp();
    unsigned keep = 0u;
    bool taken = false;
    float last = NEG;
    for (int r = 0; r <= a.topk_groups && r < a.n_groups; ++r) {
      float v = taken ? NEG : gs;
      int g = (lane < a.n_groups && !taken) ? lane : 0x7fffffff;
      warp_argmax(v, g);
      if (r < a.topk_groups) {
        keep |= 1u << g;
        if (lane == g) taken = true;
        last = v;
      } else {
        gmargin = last - v;
      }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((keep >> (e / gsz)) & 1u)) u[i] = NEG;
    }
  }

  // top-K (+1 round): the near-tie margin is the smallest gap between
  // consecutive selection scores among the top K+1
  int sel_e[KM];
  float sel_s[KM], sel_p[KM];
  unsigned taken = 0u;
  float uk = NEG, margin = INFINITY;
#pragma unroll
  for (int k = 0; k <= KM; ++k) {
    if (k > a.K) break;
    float v = NEG;
    int e = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int ei = lane + 32 * i;
      const bool ok = ei < E && !((taken >> i) & 1u);
      if (ok && (u[i] > v || (u[i] == v && ei < e))) { v = u[i]; e = ei; }
    }
    warp_argmax(v, e);
    if (k > 0 && v != NEG) margin = fminf(margin, uk - v);
    if (k < a.K) {
      const int owner = e & 31, slot = e >> 5;
      const float sv = __shfl_sync(0xffffffffu, pick<NV>(s, slot), owner);
      const float pv = __shfl_sync(0xffffffffu, pick<NV>(p, slot), owner);
      if (lane == owner) taken |= 1u << slot;
      if (k < KM) { sel_e[k] = e; sel_s[k] = sv; sel_p[k] = pv; }
      uk = v;
    }
  }
  if (lane == 0 && (margin < kNearTie || gmargin < kNearTie))
    atomicAdd(a.near_ties, 1);

  // gate weights
  float g[KM];
  float denom = 0.f;
#pragma unroll
  for (int k = 0; k < KM; ++k) {
    if (k >= a.K) break;
    if (a.score_fn == MOE_SOFTMAX) {
      g[k] = a.renorm ? expf(sel_s[k] - sel_s[0]) : sel_p[k];
    } else {
      g[k] = sel_p[k];
    }
    denom += g[k];
  }
  if (a.renorm) denom = (a.score_fn == MOE_SOFTMAX) ? denom : denom + 1e-20f;
#pragma unroll
  for (int k = 0; k < KM; ++k) {
    if (k >= a.K) break;
    float w = a.renorm ? g[k] / denom : g[k];
    w *= a.route_scale;
    if (lane == k) {
      a.topk_idx[(size_t)t * a.K + k] = sel_e[k];
      a.topk_w[(size_t)t * a.K + k] = w;
    }
  }
}

// ---------------------------------------------------------------------------
// Few experts: logits and routing fused, one warp per token, grid-stride
// over tokens.  W_r rows are read through the read-only cache (after the
// first touch they are L1 hits), so the x row loads start at once.
// ---------------------------------------------------------------------------
template <typename TX, int EB, int KM = kMaxK>
__global__ void __launch_bounds__(256)
router_fused_kernel(const TX* __restrict__ x, const float* __restrict__ w_r,
                    const float* __restrict__ offset, int D, RouteArgs a) {
  pdl_begin();
  extern __shared__ __align__(16) float gsm_all[];   // [8 warps, E]
  const int E = a.E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* gsm = gsm_all + warp * E;
  for (int t = blockIdx.x * 8 + warp; t < a.T; t += gridDim.x * 8) {
    const TX* xr = x + (size_t)t * D;
    float acc[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) acc[e] = 0.f;
    // one-slot routing keeps few registers: unroll so that the x and W_r
    // loads of several 256-column steps are in flight together
#pragma unroll (KM == 1 ? 4 : 1)
    for (int d = lane * 8; d < D; d += 256) {
      float xv[8];
      load8(xr + d, xv);
#pragma unroll
      for (int e = 0; e < EB; ++e) {
        if (e < E) {
          const float4* wrow = reinterpret_cast<const float4*>(w_r + (size_t)e * D + d);
          const float4 w0 = __ldg(wrow), w1 = __ldg(wrow + 1);
          acc[e] = fmaf(xv[0], w0.x, acc[e]); acc[e] = fmaf(xv[1], w0.y, acc[e]);
          acc[e] = fmaf(xv[2], w0.z, acc[e]); acc[e] = fmaf(xv[3], w0.w, acc[e]);
          acc[e] = fmaf(xv[4], w1.x, acc[e]); acc[e] = fmaf(xv[5], w1.y, acc[e]);
          acc[e] = fmaf(xv[6], w1.z, acc[e]); acc[e] = fmaf(xv[7], w1.w, acc[e]);
        }
      }
    }
    float s[1];
    s[0] = -INFINITY;
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const float v = warp_sum(acc[e]);
      if (lane == e && e < E) s[0] = v;
    }
    if (lane < E) {
      if (offset != nullptr) s[0] += offset[lane];
      a.logits[(size_t)t * E + lane] = s[0];
    }
    route_token<1, KM>(t, s, a, gsm, lane);
  }
}

// ---------------------------------------------------------------------------
// E > 32: tiled fp32 logits GEMM (64 tokens x 64 experts per block, 4x4 per
// thread), then a routing kernel reading the logits back.
// ---------------------------------------------------------------------------
template <typename TX>
__global__ void __launch_bounds__(256)
router_logits_kernel(const TX* __restrict__ x, const float* __restrict__ w_r,
                     const float* __restrict__ offset, float* __restrict__ logits,
                     int T, int D, int E) {
  pdl_begin();
  constexpr int BT = 64, BE = 64, BK = 32;
  __shared__ __align__(16) float xs[BK][BT + 4];
  __shared__ __align__(16) float wsm[BK][BE + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.x * BT, e0 = blockIdx.y * BE;
  float acc[4][4] = {};
  const int lr = tid >> 2, lc = (tid & 3) * 8;   // loader: row, 8-wide column
  for (int k0 = 0; k0 < D; k0 += BK) {
    {
      float v[8];
      const int t = t0 + lr;
      if (t < T && k0 + lc < D) load8(x + (size_t)t * D + k0 + lc, v);
      else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[lc + j][lr] = v[j];
      const int e = e0 + lr;
      if (e < E && k0 + lc < D) load8(w_r + (size_t)e * D + k0 + lc, v);
      else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) wsm[lc + j][lr] = v[j];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < BK; ++k) {
      const float4 av = *reinterpret_cast<const float4*>(&xs[k][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&wsm[k][tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (offset ? offset[e] : 0.f);
    }
  }
}

template <int NV>
__global__ void __launch_bounds__(256)
router_route_kernel(const float* __restrict__ logits, RouteArgs a) {
  pdl_begin();
  extern __shared__ __align__(16) float gsm_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* gsm = gsm_all + warp * a.E;
  for (int t = blockIdx.x * 8 + warp; t < a.T; t += gridDim.x * 8) {
    float s[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      s[i] = e < a.E ? logits[(size_t)t * a.E + e] : -INFINITY;
    }
    route_token<NV>(t, s, a, gsm, lane);
  }
}

// ---------------------------------------------------------------------------
// Router products on tensor cores.  An fp32 value v is the sum of three bf16
// terms up to 2^-24 |v|: hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi
// - mid) (each difference is exact in fp32).  With x already bf16, the
// logits x . W_r^T are x . W_hi^T + x . W_mid^T + x . W_lo^T: bf16 MMAs
// with fp32 accumulation give fp32-accurate logits.  Ep is E rounded up to
// 64; split rows e >= E are zero.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void split3_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& mid,
                                            __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r1);
  lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
}

// w [E,D] f32 -> wf [3 Ep, D] = (hi; mid; lo) and, if wb, wb = (hi; mid; hi)
// (the latter pairs with (hi | hi | mid) splits of a second fp32 operand).
// One thread per 8 consecutive elements of a row (D % 8 == 0): two 16-byte
// loads (w is 16-byte aligned: the entry points check it) and one 16-byte
// store per split row (wf and wb are 256-byte aligned workspace blocks, Ep D
// elements per split a multiple of 8).
__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

__global__ void __launch_bounds__(256)
split_w_kernel(const float* __restrict__ w, int E, int Ep, int D,
               __nv_bfloat16* __restrict__ wf, __nv_bfloat16* __restrict__ wb) {
  pdl_begin();
  const int64_t n = (int64_t)Ep * D;
  const int64_t nv = n / 8;
  const int dv = D / 8;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nv;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = v * 8;
    float f[8];
    if (v / dv < E) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(w + i));
      const float4 b = __ldg(reinterpret_cast<const float4*>(w + i) + 1);
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
      f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = 0.f;
    }
    uint32_t hi[4], mid[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat16 h0, m0, l0, h1, m1, l1;
      split3_bf16(f[2 * j], h0, m0, l0);
      split3_bf16(f[2 * j + 1], h1, m1, l1);
      hi[j] = pack_bf16x2(h0, h1);
      mid[j] = pack_bf16x2(m0, m1);
      lo[j] = pack_bf16x2(l0, l1);
    }
    const uint4 vh = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    const uint4 vm = make_uint4(mid[0], mid[1], mid[2], mid[3]);
    if (wf != nullptr) {
      *reinterpret_cast<uint4*>(wf + i) = vh;
      *reinterpret_cast<uint4*>(wf + n + i) = vm;
      *reinterpret_cast<uint4*>(wf + 2 * n + i) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (wb != nullptr) {
      *reinterpret_cast<uint4*>(wb + i) = vh;
      *reinterpret_cast<uint4*>(wb + n + i) = vm;
      *reinterpret_cast<uint4*>(wb + 2 * n + i) = vh;
    }
  }
}

// Routing from the three partial logit blocks of the tensor-core product
// (parts [T, 3 Ep]: x W_hi^T | x W_mid^T | x W_lo^T): logits are summed in
// that order, the offset added, written out, and the token routed.
template <int NV>
__global__ void __launch_bounds__(256)
router_route_parts_kernel(const float* __restrict__ parts, int Ep,
                          const float* __restrict__ offset, RouteArgs a) {
  pdl_begin();
  extern __shared__ __align__(16) float gsm_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* gsm = gsm_all + warp * a.E;
  for (int t = blockIdx.x * 8 + warp; t < a.T; t += gridDim.x * 8) {
    const float* pr = parts + (size_t)t * 3 * Ep;
    float s[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      s[i] = -INFINITY;
      if (e < a.E) {
        s[i] = (pr[e] + pr[Ep + e]) + pr[2 * Ep + e];
        if (offset != nullptr) s[i] += offset[e];
        a.logits[(size_t)t * a.E + e] = s[i];
      }
    }
    route_token<NV>(t, s, a, gsm, lane);
  }
}

// (v, e) into a list of N entries kept in selection order (larger score
// first, equal scores by lower expert index).  `first`: v comes from a
// lower expert index than every entry (an equal score goes in front), else
// from a higher one (an equal score stays behind).  Branch-free: position
// j takes max(lu[j], min(lu[j-1], v)) (its entry, v, or the entry pushed
// down from j - 1) and its index follows the comparisons of v with lu[j]
// and lu[j-1]; going down from the last position, only two comparisons are
// live at a time.  v is not NaN; v = -inf is never inserted.
template <int N>
__device__ __forceinline__ void topk_push(float (&lu)[N], int (&le)[N], float v, int e,
                                          bool first = false) {
  const bool real = v != -INFINITY;
  auto beats = [&](float x) { return v > x || (first && real && v == x); };
  bool beats_j = beats(lu[N - 1]);
#pragma unroll
  for (int j = N - 1; j > 0; --j) {
    const bool beats_prev = beats(lu[j - 1]);
    le[j] = beats_j ? (beats_prev ? le[j - 1] : e) : le[j];
    lu[j] = fmaxf(lu[j], fminf(lu[j - 1], v));
    beats_j = beats_prev;
  }
  le[0] = beats_j ? e : le[0];
  lu[0] = fmaxf(lu[0], v);
}

// Routing from the three partial-logit blocks with L = E / 32 lanes per
// token (E a multiple of 32, at most 1024): lane j of a token holds experts
// 32 j .. 32 j + 31 — group j when the group limit has 32 experts per
// group (the DeepSeek-shaped 8 groups of 32).  Each lane sums its logits'
// parts in the partial-logit path's order, writes its logits and scores,
// scores its group, and keeps the top-(K+1) of its experts by a
// branch-free push; the L lanes exchange group scores (rank of each group,
// lower group index first on ties) and merge their lists by shuffles in
// log2 L rounds.  The selection, the near-tie margins (among the top K+1,
// and between the last kept and the first dropped group) and the gate
// weights follow route_token; its warp-wide argmax rounds took 0.1 ms on
// the DeepSeek shape.
template <int L, int KM>
__global__ void __launch_bounds__(256)
router_route_lanes_kernel(const float* __restrict__ parts, int Ep,
                          const float* __restrict__ offset, RouteArgs a) {
  pdl_begin();
  constexpr int N = KM + 1;
  const float NEG = -INFINITY;
  const int lane = threadIdx.x & 31;
  const int j = lane % L;                    // this lane's 32-expert chunk
  const int base = lane - j;                 // the token's first lane
  const int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / L;
  const bool valid = tok < a.T;
  const int64_t t = valid ? tok : (int64_t)a.T - 1;   // whole warps take part in the shuffles
  const int E = a.E;
  const int e0 = 32 * j;
  const bool sigm = a.score_fn != MOE_SOFTMAX;
  // logits: (hi + mid) + lo + offset, as the partial-logit path sums them
  float sv[32];
  const float* pr = parts + t * 3 * (int64_t)Ep + e0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 h = *reinterpret_cast<const float4*>(pr + 4 * q);
    const float4 m = *reinterpret_cast<const float4*>(pr + Ep + 4 * q);
    const float4 l = *reinterpret_cast<const float4*>(pr + 2 * Ep + 4 * q);
    sv[4 * q] = (h.x + m.x) + l.x;
    sv[4 * q + 1] = (h.y + m.y) + l.y;
    sv[4 * q + 2] = (h.z + m.z) + l.z;
    sv[4 * q + 3] = (h.w + m.w) + l.w;
  }
  if (offset != nullptr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) sv[i] += offset[e0 + i];
  }
  // logsumexp over the token's L lanes
  float mx = NEG;
#pragma unroll
  for (int i = 0; i < 32; ++i) mx = fmaxf(mx, sv[i]);
#pragma unroll
  for (int d = 1; d < L; d <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) z += expf(sv[i] - mx);
#pragma unroll
  for (int d = 1; d < L; d <<= 1) z += __shfl_xor_sync(0xffffffffu, z, d);
  const float lse = mx + logf(z);
  // scores and selection scores; logits and scores rows written
  float u[32];
  float* lrow = a.logits + t * E + e0;
  float* prow = a.probs + t * E + e0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float pv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = 4 * q + r;
      pv[r] = sigm ? 1.0f / (1.0f + expf(-sv[i])) : expf(sv[i] - mx) / z;
      u[i] = sigm ? pv[r] + (a.sel_bias != nullptr ? a.sel_bias[e0 + i] : 0.f) : sv[i];
      if (!(u[i] == u[i])) u[i] = NEG;      // NaN never selected
    }
    if (valid) {
      *reinterpret_cast<float4*>(lrow + 4 * q) = make_float4(sv[4 * q], sv[4 * q + 1],
                                                             sv[4 * q + 2], sv[4 * q + 3]);
      *reinterpret_cast<float4*>(prow + 4 * q) = make_float4(pv[0], pv[1], pv[2], pv[3]);
    }
  }
  // group limit: this lane's chunk is one group
  float gmargin = INFINITY;
  if (a.n_groups > 1) {
    float b1 = NEG, b2 = NEG;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float v = u[i];
      if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
    }
    const float gs = (a.group_score == MOE_GMAX) ? b1 : b1 + b2;
    float gall[L];
#pragma unroll
    for (int q = 0; q < L; ++q) gall[q] = __shfl_sync(0xffffffffu, gs, base + q);
    const int tg = a.topk_groups;
    int rank = 0;
    float last = NEG, next = NEG;
#pragma unroll
    for (int q = 0; q < L; ++q) {
      int rq = 0;
#pragma unroll
      for (int q2 = 0; q2 < L; ++q2)
        rq += (gall[q2] > gall[q] || (gall[q2] == gall[q] && q2 < q)) ? 1 : 0;
      if (q == j) rank = rq;
      if (rq == tg - 1) last = gall[q];
      if (rq == tg) next = gall[q];
    }
    if (tg < L) gmargin = last - next;
    if (rank >= tg) {
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = NEG;
    }
  }
  // top-(K+1): this lane's experts in ascending order, then the other lanes'
  float lu[N];
  int le[N];
#pragma unroll
  for (int k = 0; k < N; ++k) { lu[k] = NEG; le[k] = 0x7fffffff; }
#pragma unroll
  for (int i = 0; i < 32; ++i) topk_push<N>(lu, le, u[i], e0 + i);
#pragma unroll
  for (int d = 1; d < L; d <<= 1) {
    float pu[N];
    int pe[N];
#pragma unroll
    for (int k = 0; k < N; ++k) {   // both lists exchanged before either changes
      pu[k] = __shfl_xor_sync(0xffffffffu, lu[k], d);
      pe[k] = __shfl_xor_sync(0xffffffffu, le[k], d);
    }
    const bool lower = (j & d) != 0;   // the partner's experts lie below this lane's
#pragma unroll
    for (int k = 0; k < N; ++k) topk_push<N>(lu, le, pu[k], pe[k], lower);
  }
  const int K = a.K;
  float margin = INFINITY;
#pragma unroll
  for (int k = 1; k < N; ++k)
    if (k <= K && lu[k] != NEG) margin = fminf(margin, lu[k - 1] - lu[k]);
  const bool writer = valid && j == 0;
  const unsigned tie = __ballot_sync(0xffffffffu, writer && (margin < kNearTie || gmargin < kNearTie));
  if (lane == 0 && tie != 0u) atomicAdd(a.near_ties, __popc(tie));
  __syncwarp();   // the logits and scores rows above are visible to the warp
  if (writer) {
    a.lse[t] = lse;
    float g[KM], sel_s0 = 0.f, denom = 0.f;
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      if (k >= K) break;
      const int e = min(le[k], E - 1);   // (fewer than K finite scores: NaN logits)
      const float sk = a.logits[t * E + e], pk = a.probs[t * E + e];
      if (k == 0) sel_s0 = sk;
      g[k] = (!sigm && a.renorm) ? expf(sk - sel_s0) : pk;
      denom += g[k];
    }
    if (a.renorm) denom = sigm ? denom + 1e-20f : denom;
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      if (k >= K) break;
      float w = a.renorm ? g[k] / denom : g[k];
      a.topk_idx[t * K + k] = le[k];
      a.topk_w[t * K + k] = w * a.route_scale;
    }
  }
}

}  // namespace moe
