// Router on tensor cores with the routing in the epilogue: fp32 logits
// x . W_r^T, softmax / sigmoid scores, top-K with lower-index ties, gate
// weights of variant A or B, LSE and the near-tie count, in one kernel.
//
// Follows "08 MoE" (STA324 notes) §8.2 (s = x W_r, TopK on the logits,
// variant A = truncate, variant B = softmax over the selected logits) and
// §8.6 (sigmoid affinities with a selection-only bias, weights from the raw
// affinity); the "8-MoE" lecture notes (Switch Transformers: the router in
// full precision).
//
// The fp32 product x . W_r^T (x bf16) runs as bf16 MMAs on three-way bf16
// splits of W_r (hi, mid, lo: |w - hi - mid - lo| <= 2^-24 |w|).  The
// splits are stacked along N: one MMA per 16-wide k step, N = 3 EP, gives
// three fp32 accumulators in tensor memory (x.hi | x.mid | x.lo, each
// accumulating products of its own magnitude), which the epilogue sums per
// expert as (hi + mid) + lo: fp32-accurate logits without a partial-logit
// tensor in global memory.  Each stage carries one 128 x 64 tile of x and
// the three 64-column k blocks of the splits (one 3-D TMA box, which lands
// as the 3 EP rows of one K-major B operand).
//
// Roles (192 threads, one CTA per SM, persistent over 128-token tiles):
//   warp 0   TMA producer (x tile + split box per stage, STAGES-deep ring)
//   warp 1   MMA issuer (M=128, N=3 EP, 4 MMAs per stage), double-buffered
//            accumulators (2 x 3 EP tensor-memory columns)
//   warps 2-9 epilogue, in two phases per tile:
//            1. warps 2-5 (one per tensor-memory lane quarter) read their 32
//               tokens' accumulators, sum the splits per expert, add the
//               logit offset and write the logits into a shared tile
//               [128 tokens x E]; the accumulator is released at once, so
//               the next tile's main loop overlaps the routing;
//            2. all eight warps route: warp w takes tokens 16w..16w+15,
//               lane l the token 16w + (l & 15) and half (l >> 4) of the
//               experts; partner lanes combine their max, sum and top-K
//               lists by shuffles; each warp stores its 16 tokens' logits
//               and probs rows as one contiguous block.
// Every barrier wait is bounded (see tc::mbar_wait); on timeout the kernel
// records MOE_DEVERR_TIMEOUT, drains its copies and MMAs and returns.
#pragma once
#include "gemm_tc.cuh"
#include "router.cuh"

namespace moe {
namespace rtc {

constexpr int kEpiWarps = 8;     // routing warps (the first four also read tensor memory)
constexpr int kTmemWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

template <int EP>
struct Smem {
  static constexpr int kA = 128 * 64 * 2;         // x tile of one k block
  static constexpr int kB = 3 * EP * 128;         // hi | mid | lo k blocks of W_r
  static constexpr int kStage = kA + kB;
  static constexpr int STAGES = EP == 32 ? 6 : 4;
  static constexpr int kBars = (2 * STAGES + 5) * 8;
  static constexpr int kStgLd = EP + 1;           // staging row stride (floats)
  static constexpr int kParOff = STAGES * kStage + kBars + 16;   // offset, bias [64] each
  static constexpr int kStgOff = kParOff + 2 * 64 * 4;
  static constexpr int kBytes = 1024 + kStgOff + 128 * kStgLd * 4;   // one [128 x EP] tile
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

// Writes rows [row0, row0 + nrows) of a [T, E] fp32 tensor from the warp's
// staging tile (row r at stg + r * ld): the rows are contiguous in global
// memory, so the warp stores them as one block (16-byte stores when E is a
// multiple of 4).
__device__ __forceinline__ void block_store_rows(float* __restrict__ g, int64_t row0, int nrows,
                                                 int E, const float* stg, int ld, int lane) {
  float* dst = g + row0 * E;
  const int n = nrows * E;
  if ((E & 3) == 0) {
    for (int i = 4 * lane; i < n; i += 128) {
      const int r = i / E, c = i - r * E;
      const float* sp = stg + r * ld + c;
      *reinterpret_cast<float4*>(dst + i) = make_float4(sp[0], sp[1], sp[2], sp[3]);
    }
  } else {
    for (int i = lane; i < n; i += 32) {
      const int r = i / E;
      dst[i] = stg[r * ld + (i - r * E)];
    }
  }
}

// (v, e, s) into the list of N = K + 1 entries kept in selection order:
// larger score first, equal scores by lower expert index.
template <int N>
__device__ __forceinline__ void topk_insert(float (&lu)[N], int (&le)[N], float (&ls)[N], float v,
                                            int e, float s) {
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const bool gt = v > lu[j] || (v == lu[j] && e < le[j]);
    const float tv = lu[j], ts = ls[j];
    const int te = le[j];
    lu[j] = gt ? v : tv; le[j] = gt ? e : te; ls[j] = gt ? s : ts;
    v = gt ? tv : v; e = gt ? te : e; s = gt ? ts : s;
  }
}

template <int EP, int K>
__global__ void __launch_bounds__(kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
                 const RouteArgs a, const float* __restrict__ offset, int D) {
  using S = Smem<EP>;
  constexpr int STAGES = S::STAGES;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_s;
  __shared__ int epi_stop_s;   // written before, read after an epilogue barrier
  volatile int* abort_flag = &abort_flag_s;
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + STAGES * S::kStage;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bars + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bars + 8u * (2 * STAGES + 2 + b); };
  const uint32_t done_bar = bars + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES * S::kStage + S::kBars);
  float* off_s = reinterpret_cast<float*>(gbase + S::kParOff);
  float* bias_s = off_s + 64;
  constexpr int NA = 3 * EP;                                // one accumulator's columns
  constexpr uint32_t kCols = 2 * NA <= 256 ? 256u : 512u;  // two accumulators

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (a.T + 127) / 128;
  const int nk = D / 64;
  // Tiles start their k loop at different k blocks, so the CTAs running at
  // the same time do not all load the same W_r block from L2 at once; the
  // accumulation order is fixed by the tile index (deterministic).
  auto rot_of = [&](int t) { return (int)(((int64_t)t * 5) % nk); };
  if (threadIdx.x == 0) {
    abort_flag_s = 0;
    epi_stop_s = 0;
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(accf_bar(b), 1);
      tc::mbar_init(acce_bar(b), kTmemWarps);
    }
    tc::mbar_init(done_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     tc::smem_u32(tmem_slot)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();   // the set-up above touched only this CTA's shared and tensor memory

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int rot = rot_of(t);
        for (int i = 0; i < nk; ++i) {
          const int kb = i + rot < nk ? i + rot : i + rot - nk;
          if (!tc::mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + stage * S::kStage;
          const uint32_t fb = full_bar(stage);
          tc::mbar_expect_tx(fb, S::kStage);
          issued_parity[stage] = (int)phase;
          tc::tma_2d(sa, &mapX, fb, kb * 64, t * 128);
          tc::tma_3d(sa + S::kA, &mapW, fb, kb * 64, 0, 0);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        if (issued_parity[s] >= 0) tc::mbar_wait(full_bar(s), (uint32_t)issued_parity[s], abort_flag);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = tc::make_idesc(128, NA, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        if (!tc::mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t dt = tmem + acc * NA;
        for (int kb = 0; kb < nk; ++kb) {   // k blocks in the producer's (rotated) order
          if (!tc::mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = base + stage * S::kStage;
          const uint32_t sb = sa + S::kA;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = tc::sw128_desc(sa + ks * 32, 16, 1024);
            const uint64_t bd = tc::sw128_desc(sb + ks * 32, 16, 1024);
            tc::umma(dt, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
          }
          tc::umma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc::umma_commit(accf_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      tc::umma_commit(done_bar);
      tc::mbar_wait(done_bar, 0, abort_flag);
    }
  } else {
    // ---------------- epilogue ----------------
    constexpr int HE = EP / 2;                               // experts per lane
    const int E = a.E;
    const int ew = warp - 2;
    for (int e = ew * 32 + lane; e < 64; e += kEpiWarps * 32) {
      off_s[e] = (offset != nullptr && e < E) ? offset[e] : 0.f;
      bias_s[e] = (a.sel_bias != nullptr && e < E) ? a.sel_bias[e] : 0.f;
    }
    auto epi_sync = [] {   // the eight epilogue warps only
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
    };
    epi_sync();
    float* stg = reinterpret_cast<float*>(gbase + S::kStgOff);   // [128][kStgLd]
    const float NEG = -INFINITY;
    const bool sigm = a.score_fn != MOE_SOFTMAX;
    const int half = lane >> 4;
    const int rloc = ew * 16 + (lane & 15);                  // this lane's token in the tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
      // phase 1: splits -> logits (+ offset) in the shared tile
      bool ok = true;
      if (ew < kTmemWarps) {
        const int q = warp & 3;                              // tensor-memory lane quarter
        ok = (lane == 0) ? tc::mbar_wait(accf_bar(acc), acc_phase, abort_flag) : true;
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) {
          tc::tc_fence_after();
          uint32_t r0[32], r1[32], r2[32];
          const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + acc * NA;
          float* srow = stg + (q * 32 + lane) * S::kStgLd;
#pragma unroll
          for (int c = 0; c < EP; c += 32) {
            tc::tmem_ld32(tb + c, r0);
            tc::tmem_ld32(tb + EP + c, r1);
            tc::tmem_ld32(tb + 2 * EP + c, r2);
            tc::tmem_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              srow[c + i] = ((__uint_as_float(r0[i]) + __uint_as_float(r1[i])) +
                             __uint_as_float(r2[i])) + off_s[c + i];
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(acce_bar(acc));   // accumulator free for tile t + 2
        } else if (lane == 0) {
          epi_stop_s = 1;   // a wait gave up: every epilogue warp leaves after the barrier
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      epi_sync();
      if (*reinterpret_cast<volatile int*>(&epi_stop_s)) break;   // same decision in all eight warps
      // phase 2: route 16 tokens per warp, two lanes per token
      const int64_t row0 = (int64_t)t * 128 + ew * 16;
      if (row0 < a.T) {
        const int nrows = (int)((a.T - row0) < 16 ? (a.T - row0) : 16);
        const int64_t tok = (int64_t)t * 128 + rloc;
        const bool valid = tok < a.T;
        float* srow = stg + rloc * S::kStgLd;
        block_store_rows(a.logits, row0, nrows, E, stg + ew * 16 * S::kStgLd, S::kStgLd, lane);
        // this lane's experts e = half * HE + j, read from the shared tile in
        // rolled loops (the code stays small: it runs once per tile)
        const int e0 = half * HE;
        const int e1 = min(E, e0 + HE);
        float m = NEG;
#pragma unroll 4
        for (int e = e0; e < e1; ++e) m = fmaxf(m, srow[e]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        // top-(K+1) of this lane's experts (selection score u = s, or
        // sigmoid + bias), before the row is overwritten with the scores
        float lu[K + 1], ls[K + 1];
        int le[K + 1];
#pragma unroll
        for (int k = 0; k <= K; ++k) { lu[k] = NEG; le[k] = 0x7fffffff; ls[k] = 0.f; }
        float z = 0.f;
#pragma unroll 2
        for (int e = e0; e < e1; ++e) {
          const float sv = srow[e];
          z += __expf(sv - m);
          const float u = sigm ? 1.0f / (1.0f + __expf(-sv)) + bias_s[e] : sv;
          if (u > lu[K]) topk_insert<K + 1>(lu, le, ls, u, e, sv);
        }
        z += __shfl_xor_sync(0xffffffffu, z, 16);
        const float inv_z = 1.0f / z;
        const float lse = m + logf(z);
        __syncwarp();                                         // logits rows stored
        // scores (softmax probs or sigmoid affinities) into the same rows
#pragma unroll 4
        for (int e = e0; e < e1; ++e) {
          const float sv = srow[e];
          srow[e] = sigm ? 1.0f / (1.0f + __expf(-sv)) : __expf(sv - m) * inv_z;
        }
        __syncwarp();
        block_store_rows(a.probs, row0, nrows, E, stg + ew * 16 * S::kStgLd, S::kStgLd, lane);
        // merge with the partner lane's list
        float pu[K + 1], ps[K + 1];
        int pe[K + 1];
#pragma unroll
        for (int k = 0; k <= K; ++k) {
          pu[k] = __shfl_xor_sync(0xffffffffu, lu[k], 16);
          pe[k] = __shfl_xor_sync(0xffffffffu, le[k], 16);
          ps[k] = __shfl_xor_sync(0xffffffffu, ls[k], 16);
        }
#pragma unroll
        for (int k = 0; k <= K; ++k)
          if (pu[k] != NEG) topk_insert<K + 1>(lu, le, ls, pu[k], pe[k], ps[k]);
        float margin = INFINITY;
#pragma unroll
        for (int k = 1; k <= K; ++k)
          if (lu[k] != NEG) margin = fminf(margin, lu[k - 1] - lu[k]);
        const bool writer = valid && half == 0;
        const unsigned tie = __ballot_sync(0xffffffffu, writer && margin < kNearTie);
        if (lane == 0 && tie != 0u) atomicAdd(a.near_ties, __popc(tie));
        // gate weights
        float g[K];
        float denom = 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k) {
          if (!sigm) g[k] = a.renorm ? __expf(ls[k] - ls[0]) : __expf(ls[k] - m) * inv_z;
          else g[k] = 1.0f / (1.0f + __expf(-ls[k]));
          denom += g[k];
        }
        if (a.renorm && sigm) denom += 1e-20f;
        const float inv_d = 1.0f / denom;
        if (writer) {
          a.lse[tok] = lse;
#pragma unroll
          for (int k = 0; k < K; ++k) {
            a.topk_idx[tok * K + k] = le[k];
            a.topk_w[tok * K + k] = (a.renorm ? g[k] * inv_d : g[k]) * a.route_scale;
          }
        }
      }
      epi_sync();   // the shared tile is rewritten by the next tile's phase 1
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols)
                 : "memory");
  }
}

}  // namespace rtc
}  // namespace moe
