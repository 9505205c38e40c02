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
// splits are stacked along N ([hi; mid; lo], 3 EP rows, EP = E rounded up
// to 8, 16, 32 or 64): one MMA per 16-wide k step gives three fp32
// accumulators in tensor memory (x.hi | x.mid | x.lo, each accumulating
// products of its own magnitude), which the epilogue sums per expert as
// (hi + mid) + lo: fp32-accurate logits without a partial-logit tensor in
// global memory.
//
// Tiles: each CTA takes bm tokens per tile (bm <= 128, a multiple of 8,
// chosen by the host so that the tiles spread evenly over the SMs); the MMA
// is always M = 128 (M = 256 for a pair) and the accumulator rows past bm
// are not read.  For E > 16 two CTAs of a cluster share each MMA
// (cta_group::2, M = 256): each loads its own bm token rows and half of the
// stacked split rows, so a CTA streams half of W_r per tile.  Each stage
// carries two k blocks: two bm x 64 tiles of x and two 64-column blocks of
// the split rows (half as many barrier round trips per byte as one k block
// per stage: measured faster, most at the power-capped clocks of a full
// step).
//
// Roles (320 threads, one CTA per SM, persistent over tiles):
//   warp 0   TMA producer (x tile + split rows per stage, STAGES-deep ring)
//   warp 1   MMA issuer (the pair leader only for a pair; N = 3 EP rounded
//            up to 16, 4 MMAs per stage), double-buffered accumulators
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
#include <type_traits>

#include "gemm_tc.cuh"
#include "router.cuh"

namespace moe {
namespace rtc {

constexpr int kEpiWarps = 8;     // routing warps (the first four also read tensor memory)
constexpr int kTmemWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kSmemMax = 232448;   // dynamic shared memory per CTA

// EP: split width; PAIR: two CTAs per MMA (each holds NB = NA / 2 rows of
// the stacked splits).
template <int EP, bool PAIR>
struct Smem {
  static constexpr int NA = (3 * EP + 15) / 16 * 16;   // MMA N (24 runs as 32)
  static constexpr int NAS = (NA + 31) / 32 * 32;      // accumulator stride (columns)
  static constexpr int NB = PAIR ? NA / 2 : NA;        // B rows in this CTA
  static constexpr int kA = 128 * 64 * 2;              // x tile of one k block (bm <= 128 rows)
  // stage: [x kb | x kb+1 | splits kb | splits kb+1]
  // split rows one stage receives: a pair's box is NB rows (rows past 3 EP
  // are zero-filled); a single CTA's box is the 3 EP rows (the N = 32 MMA
  // of EP = 8 also reads 8 unwritten rows, whose columns are never read)
  static constexpr int kBoxB = PAIR ? NB * 128 : 3 * EP * 128;
  static constexpr int kB = (NB * 128 + 1023) / 1024 * 1024;
  static constexpr int kStage = 2 * (kA + kB);   // two k blocks per stage
  static constexpr int kStgLd = EP + 1;                // staging row stride (floats)
  static constexpr int kStg = 128 * kStgLd * 4;        // one [128 x EP] staging tile
  static constexpr int kFixed = 1024 + 2048 + kStg;    // alignment, barriers, params, staging
  static constexpr int kFit = (kSmemMax - kFixed) / kStage;
  static constexpr int STAGES = kFit < 8 ? kFit : 8;
  static constexpr int kBars = (2 * STAGES + 5) * 8;
  static constexpr int kParOff = STAGES * kStage + kBars + 16;   // offset, bias [64] each
  static constexpr int kStgOff = kParOff + 2 * 64 * 4;
  static constexpr int kBytes = 1024 + kStgOff + kStg;
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(kBytes + 64 <= kSmemMax, "shared memory per CTA (with the static words)");
  static_assert(!PAIR || NB % 8 == 0, "whole 8-row swizzle atoms per CTA");
};

// Writes rows [row0, row0 + nrows) of a [T, E] fp32 tensor from the warp's
// staging tile (row r at stg + r * ld): the rows are contiguous in global
// memory, so the warp stores them as one block (16-byte stores when E is a
// multiple of 4; E = EP divides by a constant).
template <int EP>
__device__ __forceinline__ void block_store_rows(float* __restrict__ g, int64_t row0, int nrows,
                                                 int E, const float* stg, int ld, int lane) {
  float* dst = g + row0 * E;
  const int n = nrows * E;
  if (E == EP) {
    for (int i = 4 * lane; i < n; i += 128) {
      const int r = i / EP, c = i % EP;
      const float* sp = stg + r * ld + c;
      *reinterpret_cast<float4*>(dst + i) = make_float4(sp[0], sp[1], sp[2], sp[3]);
    }
  } else if ((E & 3) == 0) {
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

template <int EP, int K, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
                 const RouteArgs a, const float* __restrict__ offset, int D, int bm) {
  using S = Smem<EP, PAIR>;
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
  constexpr int NA = S::NA;                                 // MMA width
  constexpr int NAS = S::NAS;                               // accumulator stride
  constexpr uint32_t kCols = 2 * NAS <= 64 ? 64u : 2 * NAS <= 128 ? 128u
                           : 2 * NAS <= 256 ? 256u : 512u;  // two accumulators

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = PAIR ? (int)tc::cluster_rank() : 0;     // 0 = pair leader
  const bool leader = rank == 0;
  const int unit = PAIR ? blockIdx.x >> 1 : blockIdx.x;    // this CTA's tile stream
  const int n_units = PAIR ? gridDim.x >> 1 : gridDim.x;
  const int U = PAIR ? 2 * bm : bm;                         // tokens per tile (both CTAs)
  const int n_tiles = (a.T + U - 1) / U;
  const int nk = D / 64;
  // Tiles start their k loop at different k blocks, so the CTAs running at
  // the same time do not all load the same W_r block from L2 at once; the
  // accumulation order is fixed by the tile index (deterministic).
  const int nk2 = nk / 2;                                  // stages per tile
  auto rot_of = [&](int t) { return (int)(((int64_t)t * 5) % nk2); };
  if (threadIdx.x == 0) {
    abort_flag_s = 0;
    epi_stop_s = 0;
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(accf_bar(b), 1);
      tc::mbar_init(acce_bar(b), kTmemWarps * (PAIR ? 2 : 1));   // both CTAs' readers
    }
    tc::mbar_init(done_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    __syncwarp();
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       tc::smem_u32(tmem_slot)),
                   "r"(kCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       tc::smem_u32(tmem_slot)),
                   "r"(kCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) tc::cluster_sync();   // both CTAs' barriers exist before any remote use
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_begin();   // the set-up above touched only this CTA's shared and tensor memory

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs of a pair) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
      const uint32_t tx = 2u * (uint32_t)(bm * 128 + S::kBoxB) * (PAIR ? 2u : 1u);
      bool ok = true;
      for (int t = unit; t < n_tiles && ok; t += n_units) {
        const int rot = rot_of(t);
        const int row = t * U + rank * bm;                   // this CTA's first token
        for (int i = 0; i < nk2; ++i) {
          const int kb = 2 * (i + rot < nk2 ? i + rot : i + rot - nk2);
          if (!tc::mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + stage * S::kStage;
          const uint32_t fb = full_bar(stage);
          if (!PAIR || leader) tc::mbar_expect_tx(fb, tx);
          issued_parity[stage] = (int)phase;
          if constexpr (PAIR) {
            const uint32_t lfb = tc::mapa(fb, 0);           // the leader's full barrier
            tc::tma_2d_pair_nohint(sa, &mapX, lfb, kb * 64, row);
            tc::tma_2d_pair_nohint(sa + S::kA, &mapX, lfb, kb * 64 + 64, row);
            tc::tma_2d_pair_nohint(sa + 2 * S::kA, &mapW, lfb, kb * 64, rank * S::NB);
            tc::tma_2d_pair_nohint(sa + 2 * S::kA + S::kB, &mapW, lfb, kb * 64 + 64, rank * S::NB);
          } else {
            tc::tma_2d(sa, &mapX, fb, kb * 64, row);
            tc::tma_2d(sa + S::kA, &mapX, fb, kb * 64 + 64, row);
            tc::tma_2d(sa + 2 * S::kA, &mapW, fb, kb * 64, 0);
            tc::tma_2d(sa + 2 * S::kA + S::kB, &mapW, fb, kb * 64 + 64, 0);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // drain: the copies have landed before teardown (a pair's copies all
      // complete on the leader's barriers)
      if (!PAIR || leader)
        for (int s = 0; s < STAGES; ++s)
          if (issued_parity[s] >= 0)
            tc::mbar_wait(full_bar(s), (uint32_t)issued_parity[s], abort_flag);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = tc::make_idesc(PAIR ? 256 : 128, NA, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = unit; t < n_tiles && ok; t += n_units) {
        if (!tc::mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t dt = tmem + acc * NAS;
        for (int kb = 0; kb < nk2; ++kb) {   // k block pairs in the producer's (rotated) order
          if (!tc::mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = base + stage * S::kStage;
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const uint32_t sas = sa + sub * S::kA;
            const uint32_t sbs = sa + 2 * S::kA + sub * S::kB;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = tc::sw128_desc(sas + ks * 32, 16, 1024);
              const uint64_t bd = tc::sw128_desc(sbs + ks * 32, 16, 1024);
              const uint32_t accum = (kb | sub | ks) != 0 ? 1u : 0u;
              if constexpr (PAIR) tc::umma_pair(dt, ad, bd, idesc, accum);
              else tc::umma(dt, ad, bd, idesc, accum);
            }
          }
          if constexpr (PAIR) tc::umma_commit_pair_both(empty_bar(stage));
          else tc::umma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) tc::umma_commit_pair_both(accf_bar(acc));
        else tc::umma_commit(accf_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if constexpr (PAIR) tc::umma_commit_pair_local(done_bar);
      else tc::umma_commit(done_bar);
      tc::mbar_wait(done_bar, 0, abort_flag);
    }
  } else {
    // ---------------- epilogue ----------------
    constexpr int HE = EP / 2;                               // experts per lane
    constexpr int CH = HE < 8 ? HE : 8;                      // unrolled chunk
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
    for (int t = unit; t < n_tiles; t += n_units) {
      // phase 1: splits -> logits (+ offset) in the shared tile
      bool ok = true;
      if (ew < kTmemWarps) {
        const int q = warp & 3;                              // tensor-memory lane quarter
        ok = (lane == 0) ? tc::mbar_wait(accf_bar(acc), acc_phase, abort_flag) : true;
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) {
          tc::tc_fence_after();
          const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + acc * NAS;
          float* srow = stg + (q * 32 + lane) * S::kStgLd;
          if constexpr (EP >= 32) {
            uint32_t r0[32], r1[32], r2[32];
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
          } else {
            // all three splits of the (8 or 16) experts in one or two loads
            constexpr int NC = NAS / 32;
            uint32_t r[NC][32];
#pragma unroll
            for (int c = 0; c < NC; ++c) tc::tmem_ld32(tb + 32 * c, r[c]);
            tc::tmem_wait();
#pragma unroll
            for (int i = 0; i < EP; ++i)
              srow[i] = ((__uint_as_float(r[i / 32][i % 32]) +
                          __uint_as_float(r[(EP + i) / 32][(EP + i) % 32])) +
                         __uint_as_float(r[(2 * EP + i) / 32][(2 * EP + i) % 32])) + off_s[i];
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) {   // accumulator free for tile t + 2 (the pair leader's barrier)
            if (!PAIR || leader) tc::mbar_arrive(acce_bar(acc));
            else tc::mbar_arrive_remote(tc::mapa(acce_bar(acc), 0));
          }
        } else if (lane == 0) {
          epi_stop_s = 1;   // a wait gave up: every epilogue warp leaves after the barrier
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      epi_sync();
      if (*reinterpret_cast<volatile int*>(&epi_stop_s)) break;   // same decision in all eight warps
      // phase 2: route 16 tokens per warp, two lanes per token
      const int64_t tok0 = (int64_t)t * U + rank * bm;       // this CTA's first token
      const int r0 = ew * 16;                                // this warp's first row
      if (r0 < bm && tok0 + r0 < a.T) {
        const int nrows = (int)min((int64_t)min(16, bm - r0), a.T - (tok0 + r0));
        const int64_t tok = tok0 + rloc;
        const bool valid = rloc < bm && tok < a.T;
        float* srow = stg + rloc * S::kStgLd;
        block_store_rows<EP>(a.logits, tok0 + r0, nrows, E, stg + r0 * S::kStgLd, S::kStgLd, lane);
        // this lane's experts e = e0 + j (j < HE, e < E), read from the
        // shared row in unrolled chunks of CH (straight-line code, no
        // data-dependent branches)
        const int e0 = half * HE;
        float m = NEG;
#pragma unroll 1
        for (int jc = 0; jc < HE; jc += CH) {
#pragma unroll
          for (int jj = 0; jj < CH; ++jj) {
            const int e = e0 + jc + jj;
            if (e < E) m = fmaxf(m, srow[e]);
          }
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        // softmax denominator, and the top-(K+1) of this lane's experts by
        // selection score (u = s, or sigmoid + bias), kept in selection
        // order (larger first, equal scores by lower expert index)
        float lu[K + 1];
        int le[K + 1];
#pragma unroll
        for (int k = 0; k <= K; ++k) { lu[k] = NEG; le[k] = 0x7fffffff; }
        float z = 0.f;
        // (the score function is uniform: one loop per form)
        auto select = [&](auto sig) {
          constexpr bool SIG = decltype(sig)::value;
#pragma unroll 1
          for (int jc = 0; jc < HE; jc += CH) {
#pragma unroll
            for (int jj = 0; jj < CH; ++jj) {
              const int e = e0 + jc + jj;
              const bool in = e < E;
              const float sv = in ? srow[e] : NEG;
              z += in ? __expf(sv - m) : 0.f;
              float u = SIG ? 1.0f / (1.0f + __expf(-sv)) + bias_s[e] : sv;
              u = (in && u == u) ? u : NEG;     // padding experts and NaN never selected
              topk_push<K + 1>(lu, le, u, e);   // e ascending: an equal score stays behind
            }
          }
        };
        if (sigm) select(std::true_type{});
        else select(std::false_type{});
        z += __shfl_xor_sync(0xffffffffu, z, 16);
        const float inv_z = 1.0f / z;
        const float lse = m + logf(z);
        // merge the partner lane's list: its experts all lie above this
        // lane's for half 0 (the lane that writes), so an equal score from
        // the partner stays behind
        float pu[K + 1];
        int pe[K + 1];
#pragma unroll
        for (int k = 0; k <= K; ++k) {   // both lists exchanged before either changes
          pu[k] = __shfl_xor_sync(0xffffffffu, lu[k], 16);
          pe[k] = __shfl_xor_sync(0xffffffffu, le[k], 16);
        }
#pragma unroll
        for (int k = 0; k <= K; ++k) topk_push<K + 1>(lu, le, pu[k], pe[k]);
        // logits of the selected experts (the row still holds logits)
        float ls[K];
#pragma unroll
        for (int k = 0; k < K; ++k) ls[k] = srow[min(le[k], E - 1)];
        __syncwarp();                                   // logits rows stored and read
        // scores (softmax probs or sigmoid affinities) into the same rows
        auto scores = [&](auto sig) {
          constexpr bool SIG = decltype(sig)::value;
#pragma unroll 1
          for (int jc = 0; jc < HE; jc += CH) {
#pragma unroll
            for (int jj = 0; jj < CH; ++jj) {
              const int e = e0 + jc + jj;
              if (e < E) {
                const float sv = srow[e];
                srow[e] = SIG ? 1.0f / (1.0f + __expf(-sv)) : __expf(sv - m) * inv_z;
              }
            }
          }
        };
        if (sigm) scores(std::true_type{});
        else scores(std::false_type{});
        __syncwarp();
        block_store_rows<EP>(a.probs, tok0 + r0, nrows, E, stg + r0 * S::kStgLd, S::kStgLd, lane);
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
  if constexpr (PAIR) tc::cluster_sync();   // the leader's MMAs into both CTAs are done
  tc::tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols)
                   : "memory");
  }
}

}  // namespace rtc
}  // namespace moe
