// Tensor-core (tcgen05 / TMEM / TMA) grouped GEMMs for the expert SwiGLU
// projections, forward and backward, bf16 operands, fp32 accumulation.
//
// The pages ask for grouped/batched GEMMs over experts instead of a Python
// loop of small per-expert matmuls (STA324 notes "08 MoE" §8.8) on tokens
// grouped contiguously per expert ("8-MoE" lecture notes, MoE 高效推理);
// the kernel design itself is ours, for sm_100a:
//
//   * persistent grid (one CTA per SM), static round-robin tile schedule;
//     the number of 128-row tiles is read on the device (no host sync) and
//     every tile's expert comes from the dispatch's tile -> expert map, so
//     experts without rows cost nothing;
//   * warp 0: TMA producer (128B-swizzled boxes into a STAGES-deep ring);
//     warp 1: one thread issues tcgen05.mma (M=128, N=BN, K=16) into a ring
//     of fp32 accumulators in tensor memory (two, or four when BN = 128);
//     warps 2-9: epilogue
//     (two warps per tensor-memory lane quarter; tcgen05.ld, fused SwiGLU /
//     SwiGLU-backward, bf16 stores), overlapped with the next tile's main
//     loop;
//   * ROWS mode: C[r, n] = sum_k A[r, k] B_e[n, k] (forward, data gradients);
//     WGRAD mode: C_g[m, n] = sum_{r in rows(g)} A[r, m] B[r, n] (weight
//     gradients; the reduction runs over the group's own rows and the zero
//     padding rows beyond them contribute nothing);
//   * GATHER variants copy the row operand (gate/up A rows, gate/up wgrad B
//     rows) straight from the token rows of x with cp.async in the
//     producer warp, instead of TMA boxes of a permuted copy;
//   * dense variants (no tile map, one group, fp32 epilogues) serve the
//     router's fp32 products, which run as bf16 MMAs on three-way bf16
//     splits of the fp32 operand (x . W_r^T, ds^T . x, ds . W_r);
//   * every mbarrier wait is bounded in time; on timeout the kernel records
//     MOE_DEVERR_TIMEOUT, drains its own copies and MMAs, frees tensor
//     memory and returns.
#pragma once
#include <cuda.h>
#include "common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                    // one 128-byte swizzle row of bf16
constexpr int kEpiWarps = 8;                  // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

enum { MODE_ROWS = 0, MODE_WGRAD = 1 };
enum {
  EPI_STORE = 0,       // bf16 C
  EPI_SWIGLU = 1,      // a13 = C (gate | up) and h = silu(gate) * up
  EPI_SWIGLU_BWD = 2,  // da13 from dh = C and the saved a13
  EPI_WGRAD = 3,       // bf16 weight gradient per group
  EPI_F32 = 4,         // fp32 C, rows < dense_m (dense ROWS)
  EPI_WGRAD_F32 = 5,   // fp32 C, rows < m_limit (dense WGRAD)
  // one slot per token (K = 1, no shared expert): the row of token t is
  // row_slot^-1(t), so combine and unpermute-sum are row scatters
  EPI_COMBINE1 = 6,    // bf16 C (o) and y[token(r)] = g_token * C
  EPI_DX1 = 7          // dx[token(r)] = C + ds_token . W_r (no row output)
};

struct Params {
  int E, F, Kd;
  int nN;                      // ROWS: output column tiles
  int group_m;                 // ROWS: row tiles per rasterisation group
  const int32_t* tile_expert;  // ROWS
  const int32_t* stats;        // ROWS: stats[3] = 128-row tiles in use
  const int32_t* offsets;      // WGRAD: first row of each group
  const int32_t* kept;         // WGRAD: rows of each routed group
  int T;                       // WGRAD: rows of the shared group
  int n_groups;                // WGRAD
  int nMo, nNo, No;            // WGRAD tiles per group, output columns
  int64_t strideCE;            // WGRAD: elements per group output
  __nv_bfloat16* out;  int64_t ld_out;
  __nv_bfloat16* out2; int64_t ld_out2;    // SwiGLU: h
  const __nv_bfloat16* aux; int64_t ld_aux;  // SwiGLU bwd: a13
  __nv_bfloat16* out_shared;               // WGRAD: shared group output
  // dense variants
  int dense_m;                 // ROWS: > 0 = one group of dense_m rows, no tile map
  int dense_rows;              // WGRAD: > 0 = dense_rows rows, no groups of experts:
  int dense_split;             //   group g takes rows [g, g + 1) * dense_split (a K
                               //   split, multiple of 64; 0 = one group of all rows)
                               //   and writes its partial at out_f32 + g * strideCE
  int m_limit;                 // WGRAD_F32: output rows
  float* out_f32; int64_t ld_f32;          // F32 epilogues
  // gathered rows (the GATHER kernels copy token rows of x instead of
  // reading a permuted copy): row r holds token row_slot[r] / gK, or token
  // r - offsets[E] inside the shared group, or zeros (padding)
  const __nv_bfloat16* gx;     // x [T, Kd] (ROWS) or [T, No] (WGRAD)
  const int32_t* row_slot;
  int gK;                      // slots per token
  int shared_T;                // rows of the shared group (0: none)
  // token-order epilogues (COMBINE1, DX1): token of row r = row_slot[r];
  // tokens whose slot has no row (slot_row < 0) are written at kernel start
  const int32_t* slot_row;
  const float* tw;             // COMBINE1: gate weight per token
  __nv_bfloat16* tout;         // y or dx [T, ld_out]
  const float* ds;             // DX1: router logit gradient [T, Er]
  const float* w_r;            // DX1: router weight [Er, ld_out]
  int Er;                      // DX1: router experts (<= 8)
};

// ----------------------------------------------------------------------------
// PTX wrappers (written from the PTX ISA for sm_100a)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// The same with cluster-scope acquire: the phase was completed by arrivals
// (release.cluster) from the other CTA of a pair after it wrote shared
// memory that this CTA's tensor-core instructions read.
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for phase `parity` of `bar`.  False once the kernel aborted.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       bool cluster_acquire = false) {
  auto probe = [&] {
    return cluster_acquire ? mbar_try_cluster(bar, parity) : mbar_try(bar, parity);
  };
  if (probe()) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (probe()) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        set_dev_error(MOE_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                       int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                       int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
// ---- CTA-pair (cta_group::2) forms: two SMs of one cluster share each MMA
// (each holds half of A's rows and half of B's columns; each gets its own
// 128-row slice of the accumulator) -------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory completing on the pair leader's
// barrier (`bar` is a shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_2d_pair_nohint(uint32_t dst, const CUtensorMap* map,
                                                   uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                          uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once the
// MMAs issued so far are complete.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"(mask)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// Arrive on a barrier in another CTA of the cluster (cluster address).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor: kind::f16, bf16 x bf16 -> f32, M x N.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                     uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 32 TMEM lanes x 32 consecutive fp32 columns: thread i of the warp gets lane
// (base lane + i), columns [col, col+32).  tmem_wait() must follow before
// the registers are read.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void u2f32(const uint32_t (&r)[32], float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Epilogue math on bf16-rounded outputs: the hardware approximate divide
// (__fdividef) and exponential (__expf) instead of IEEE division, which
// would compile to a branchy subroutine.
__device__ __forceinline__ float fast_sigmoid(float a) {
  return __fdividef(1.0f, 1.0f + __expf(-a));
}
__device__ __forceinline__ void bf16x8_to_f(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

// L2 cache policies: epilogue outputs are written once and read by a later
// kernel (evict first, so they do not push out operand tiles that are still
// being reused); row tiles of the ROWS GEMMs are reused across the whole
// column sweep of their rasterisation group (evict last).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(pol)
      : "memory");
}

// ---- row gather: 16-byte cp.async copies ------------------------------------
// A gathered operand row (128 bytes of one k block) is copied by 8 lanes,
// 16 bytes each, into the 128B-swizzled layout a TMA box load would have
// produced: chunk c of tile row r lands at r * 128 + ((c ^ (r & 7)) << 4)
// from a 1024-byte aligned tile.  src_bytes = 0 writes zeros (padding rows)
// without reading.  Each copying lane arrives on the stage's full barrier
// when its copies complete (no wait in the producer); the copies are
// generic-proxy writes, so the MMA thread fences them into the async proxy
// after its barrier wait and before the tensor cores read the stage.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` (counted in its expected arrivals) once every cp.async
// this thread issued so far has completed; the thread does not wait.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- TMA stores (shared -> global, bulk async-groups of the issuing thread)
// Box `src` (shared, laid out as the map's swizzle wants) to the tensor of
// `map` at element coordinates (x, y); x * 2 bytes is a multiple of 16 and
// both coordinates are non-negative (rows past the tensor are clipped).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until at most one committed group still reads its shared source.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Waits until no committed group still reads its shared source.
__device__ __forceinline__ void bulk_wait_read_0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until every committed group has completed its global writes.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 32 floats -> 32 bf16 at p (64 bytes, 16-byte aligned), with an L2 policy.
__device__ __forceinline__ void store32_bf16(__nv_bfloat16* p, const float (&v)[32],
                                             uint64_t pol) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h2[i] = __floats2bfloat162_rn(v[8 * q + 2 * i], v[8 * q + 2 * i + 1]);
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p + 8 * q),
                 "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol)
                 : "memory");
  }
}
// ---- warp-staged epilogue I/O ------------------------------------------------
// An epilogue lane owns one accumulator row, so writing its 32 columns
// directly would make every warp-wide 16-byte access touch 32 different
// rows.  Instead each warp passes a 32-row x 32-column bf16 block through a
// private shared-memory tile (row stride 80 bytes: the 16-byte accesses of
// both the row-wise and the segment-wise pass fall in distinct banks), and
// global memory sees 64-byte row segments, 8 rows per instruction.
constexpr int kStgRow = 80;
constexpr int kStgBytes = 32 * kStgRow;

__device__ __forceinline__ void sts128(uint32_t a, const uint4& u) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(u.x), "r"(u.y), "r"(u.z),
               "r"(u.w)
               : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 u;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
               : "r"(a)
               : "memory");
  return u;
}
__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
  uint4 u;
  __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h2[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  return u;
}

// Stores this lane's 32 values (its row of the block) as bf16; w0 addresses
// the block's first row and column, ld is the row stride in elements.
__device__ __forceinline__ void staged_store32(uint32_t stg, const float (&v)[32],
                                               __nv_bfloat16* w0, int64_t ld, uint64_t pol,
                                               int nrows = 32) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) sts128(stg + lane * kStgRow + j * 16, pack8_bf16(v + 8 * j));
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2), pc = lane & 3;
    const uint4 u = lds128(stg + r * kStgRow + pc * 16);
    if (r < nrows)
      asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(
                       w0 + r * ld + pc * 8),
                   "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol)
                   : "memory");
  }
  __syncwarp();
}

// staged_store32 of values already packed to bf16 (pk[4 j + i] holds the
// pairs of columns 8 j + 2 i, 8 j + 2 i + 1).
__device__ __forceinline__ void staged_store32_pk(uint32_t stg, const uint4 (&pk)[4],
                                                  __nv_bfloat16* w0, int64_t ld, uint64_t pol) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) sts128(stg + lane * kStgRow + j * 16, pk[j]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2), pc = lane & 3;
    const uint4 u = lds128(stg + r * kStgRow + pc * 16);
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(
                     w0 + r * ld + pc * 8),
                 "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol)
                 : "memory");
  }
  __syncwarp();
}

// Staging of one TMA-store box: 32 rows x 32 bf16 columns (64-byte rows)
// in the 64-byte swizzle (16-byte chunk j of row r sits at chunk
// j ^ ((r >> 1) & 3)), so the 16-byte stores of any 8 consecutive lanes
// fall in distinct banks.  Lane r writes row r; `buf` is 512-byte aligned.
constexpr int kTmaBox = 32 * 64;
__device__ __forceinline__ void stage_box_sw64(uint32_t buf, const uint4 (&u)[4]) {
  const int r = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) sts128(buf + r * 64 + ((j ^ ((r >> 1) & 3)) << 4), u[j]);
}

// Staging of one fp32 TMA-store box: 32 rows x 32 floats (128-byte rows) in
// the 128-byte swizzle (16-byte chunk j of row r at chunk j ^ (r % 8)), so
// the 16-byte stores of any 8 consecutive lanes fall in distinct banks.
// Lane r writes row r; `buf` is 1024-byte aligned.
__device__ __forceinline__ void stage_box_f32_sw128(uint32_t buf, const float (&v)[32]) {
  const int r = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint4 u;
    u.x = __float_as_uint(v[4 * j]);
    u.y = __float_as_uint(v[4 * j + 1]);
    u.z = __float_as_uint(v[4 * j + 2]);
    u.w = __float_as_uint(v[4 * j + 3]);
    sts128(buf + r * 128 + ((j ^ (r & 7)) << 4), u);
  }
}

// staged_store32 to scattered rows: block row i goes to w0 + tok_i * ld,
// where tok_i is lane i's `tok` (rows with tok < 0 are skipped).
__device__ __forceinline__ void staged_store32_tok(uint32_t stg, const float (&v)[32],
                                                   __nv_bfloat16* w0, int64_t ld, int tok,
                                                   uint64_t pol) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) sts128(stg + lane * kStgRow + j * 16, pack8_bf16(v + 8 * j));
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2), pc = lane & 3;
    const int tr = __shfl_sync(0xffffffffu, tok, r);
    const uint4 u = lds128(stg + r * kStgRow + pc * 16);
    if (tr >= 0)
      asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(
                       w0 + (int64_t)tr * ld + pc * 8),
                   "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol)
                   : "memory");
  }
  __syncwarp();
}

// 32 fp32 values of one row (16-byte stores).
__device__ __forceinline__ void store32_f32(float* p, const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    *reinterpret_cast<float4*>(p + 4 * i) = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2],
                                                        v[4 * i + 3]);
}

// Coalesced load of a 32 x 32 bf16 block (w0: first row and column): piece
// i of this lane is row 8 i + lane / 4, columns 8 (lane % 4) .. + 7.
__device__ __forceinline__ void block_load32(const __nv_bfloat16* w0, int64_t ld, uint4 (&u)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    u[i] = *reinterpret_cast<const uint4*>(w0 + (i * 8 + (lane >> 2)) * ld + (lane & 3) * 8);
}
// The pieces of block_load32 -> this lane's row (32 floats).
__device__ __forceinline__ void staged_rows32(uint32_t stg, const uint4 (&u)[4], float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i) sts128(stg + (i * 8 + (lane >> 2)) * kStgRow + (lane & 3) * 16, u[i]);
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) bf16x8_to_f(lds128(stg + lane * kStgRow + j * 16), v + 8 * j);
  __syncwarp();
}

__device__ __forceinline__ void load32_bf16(const __nv_bfloat16* p, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) load8(p + 8 * q, v + 8 * q);
}

// ----------------------------------------------------------------------------
// Tile decode (identical in all roles)
// ----------------------------------------------------------------------------
struct Tile {
  int e;        // expert / group (E = shared)
  int m0;       // ROWS: first row; WGRAD: first output row
  int n0;       // first output column (SwiGLU: first F column j0)
  int row0;     // WGRAD: first input row of the group
  int nk;       // K blocks (0: empty group)
};

// M rows per tile: 128, or 256 for a CTA pair (this CTA holds 128 of them).
// n_mt: row tiles in use (ROWS; read once per kernel from stats).
template <int MODE, int EPI, int BN, bool PAIR>
__device__ __forceinline__ Tile decode(int t, const Params& p, int rank, int n_mt) {
  constexpr int MU = PAIR ? 2 * BM : BM;
  Tile d;
  if (MODE == MODE_ROWS) {
    // Grouped rasterisation: tiles run in groups of p.group_m row tiles, the
    // column tile outermost inside a group, so the CTAs that run at the same
    // time share their row tiles (kept in L2) and a few weight column
    // slices, instead of streaming an expert's weights once per row tile.
    // With a CTA pair a row tile is 256 rows: two 128-row tiles of one
    // expert (expert segments are then 256-row aligned).
    const int group = t / (p.group_m * p.nN);
    const int first = group * p.group_m;
    const int gm = min(p.group_m, n_mt - first);
    const int local = t - group * p.group_m * p.nN;
    const int mt = first + local % gm, nt = local / gm;
    d.e = p.dense_m > 0 ? 0 : p.tile_expert[mt * (MU / BM)];
    d.m0 = mt * MU + rank * BM;
    d.n0 = nt * (EPI == EPI_SWIGLU ? BN / 2 : BN);
    d.row0 = 0;
    d.nk = p.Kd / BK;
  } else {
    const int per = p.nMo * p.nNo;
    const int g = t / per, rem = t % per;
    d.e = g;
    d.m0 = (rem / p.nNo) * MU + rank * BM;
    d.n0 = (rem % p.nNo) * BN;
    const int split = p.dense_split > 0 ? p.dense_split : p.dense_rows;
    d.row0 = p.dense_rows > 0 ? g * split : p.offsets[g];
    const int rows = p.dense_rows > 0 ? min(split, p.dense_rows - d.row0)
                     : g < p.E           ? p.kept[g]
                                         : p.T;
    d.nk = (rows + BK - 1) / BK;
  }
  return d;
}

// Shared memory per CTA: BNC = columns of B this CTA holds (BN, or BN/2
// for a CTA pair).
template <int BN, int STAGES, bool PAIR, int KB = 1>
struct Smem {
  static constexpr int BNC = PAIR ? BN / 2 : BN;
  // accumulators in tensor memory (512 columns): four of BN = 128 columns,
  // two of 192 or 256, so short tiles (few k blocks) run ahead of the
  // epilogue; one of BN = 512 (CTA pairs), which halves the operand bytes
  // per MMA and leaves the epilogue unoverlapped
  static constexpr int NACC = BN <= 128 ? 4 : BN <= 256 ? 2 : 1;
  static constexpr int kA = BM * BK * 2;        // 16 KB
  static constexpr int kB = BNC * BK * 2;
  static constexpr int kStage = KB * (kA + kB);   // KB k blocks: [A0 A1 .. | B0 B1 ..]
  // full, empty, copies-done per stage; full, empty per accumulator; done
  // (+kEpiWarps: the SwiGLU-backward epilogue warps' own load barriers)
  static constexpr int kBars = (3 * STAGES + 2 * NACC + 1 + kEpiWarps) * 8;
  // token table of the gathering producer (128 rows)
  static constexpr int kTokOff = STAGES * kStage + kBars + 16;
  // epilogue staging per epilogue warp: two 2 KB boxes for the epilogues
  // that store through TMA (or one 4 KB fp32 box), a 2.5 KB tile for the
  // others (the 192-wide tiles, whose five stages leave no room for the
  // boxes); 1024-byte aligned (the fp32 box's 128-byte swizzle)
  static constexpr int kStgW = BN == 192 ? kStgBytes : 2 * kTmaBox;
  static constexpr int kEpiOff = (kTokOff + 512 + 1023) / 1024 * 1024;
  static constexpr int kBytes = 1024 + kEpiOff + kEpiWarps * kStgW;
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

// k blocks per pipeline stage: two for pair tiles and 128-wide tiles
// (stages of 48-96 KB per CTA instead of 24-48 KB, about the same bytes in
// flight with half the barrier round trips; measured 3-15% faster on the
// OLMoE-, Mixtral- and DeepSeek-shaped GEMMs and 23% on the router weight
// gradient, results bit-identical), else one (the 192/256-wide single-CTA
// tiles, where two 80-96 KB stages measured slower than 4-5 of one k
// block, and the gathering producer).  The kernel and its launch both take
// the shared-memory layout from here.
template <int BN, int STAGES, int MODE, bool PAIR, bool GATHER>
constexpr int stage_kb() {
  return (!GATHER && ((PAIR && BN == 512 && STAGES == 2) || (PAIR && BN == 256 && STAGES == 3) ||
                      (PAIR && BN == 128 && STAGES == 4) || (!PAIR && BN == 128 && STAGES == 3)))
             ? 2 : 1;
}
template <int BN, int STAGES, int MODE, bool PAIR, bool GATHER>
using KernelSmem = Smem<BN, STAGES, PAIR, stage_kb<BN, STAGES, MODE, PAIR, GATHER>()>;

// GATHER: the row operand comes from the token rows of x (Params.row_slot)
// by 16-byte cp.async copies issued by the whole producer warp: the A rows
// of a ROWS tile (gate/up + SwiGLU), or the B rows of a WGRAD k block
// (gate/up weight gradient); the other operand still arrives by TMA box.
// mapO / mapO2: the outputs of the SwiGLU (a13, h), plain-store (out) and
// weight-gradient (the routed experts' out as [E * rows, No], the shared
// expert's out_shared) epilogues as 2-D bf16 tensors with 32 x 32 boxes in
// the 64-byte swizzle (kTmaOut: every tile width but 192); unused by the
// other instantiations.
template <int BN, int STAGES, int MODE, bool A_MN, bool B_MN, int EPI, bool PAIR,
          bool GATHER = false>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
            const __grid_constant__ CUtensorMap mapBs, const __grid_constant__ CUtensorMap mapO,
            const __grid_constant__ CUtensorMap mapO2, const Params p, int total_hint) {
  constexpr bool kTmaOut = BN != 192 && (EPI == EPI_SWIGLU || EPI == EPI_STORE || EPI == EPI_WGRAD);
  // SwiGLU backward: the saved a13 blocks come in by TMA (mapO) into the
  // warp's two staging boxes, dA13 is computed in place and stored by TMA
  // (mapO2)
  constexpr bool kTmaBwd = BN != 192 && EPI == EPI_SWIGLU_BWD;
  // fp32 outputs (the router products): one 32 x 32 fp32 box per warp in
  // the 128-byte swizzle, stored by TMA (mapO)
  constexpr bool kTmaF32 = BN != 192 && EPI == EPI_F32;
  constexpr int KB = stage_kb<BN, STAGES, MODE, PAIR, GATHER>();
  using S = KernelSmem<BN, STAGES, MODE, PAIR, GATHER>;
  constexpr int BNC = S::BNC;
  constexpr int NACC = S::NACC;
  // N of one MMA (at most 256) and MMAs per k step; the B rows of MMA block
  // m sit at sb + m * BLK * 128 in each CTA (BLK rows per CTA and block)
  constexpr int NBM = BN > 256 ? BN / 256 : 1;
  constexpr int NMM = BN / NBM;
  constexpr int BLK = PAIR ? NMM / 2 : NMM;
  static_assert(BN <= 256 || (PAIR && !GATHER), "BN = 512 only on CTA pairs, box-loaded operands");
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_s;
  volatile int* abort_flag = &abort_flag_s;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + STAGES * S::kStage;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bars + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bars + 8u * (2 * STAGES + NACC + b); };
  const uint32_t done_bar = bars + 8u * (2 * STAGES + 2 * NACC);
  // gathered rows in a pair's second CTA: its lanes' cp.async copies arrive
  // here; warp 1 forwards each completed stage to the leader's full barrier
  auto cpd_bar = [&](int s) { return bars + 8u * (2 * STAGES + 2 * NACC + 1 + s); };
  // epilogue warp w's barrier for its TMA loads of saved a13 blocks
  auto epi_bar = [&](int w) { return bars + 8u * (3 * STAGES + 2 * NACC + 1 + w); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES * S::kStage + S::kBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = PAIR ? (int)cluster_rank() : 0;        // 0 = pair leader
  const bool leader = rank == 0;
  const int unit = PAIR ? blockIdx.x >> 1 : blockIdx.x;   // this CTA's tile stream
  const int n_units = PAIR ? gridDim.x >> 1 : gridDim.x;
  // tensor memory: NACC BN-column fp32 accumulators; tcgen05.alloc takes a
  // power of two between 32 and 512 columns
  constexpr uint32_t kCols = (NACC * BN <= 128) ? 128u : (NACC * BN <= 256) ? 256u : 512u;
  static_assert(NACC * BN <= 512 && (kCols & (kCols - 1)) == 0, "tensor-memory columns");
  static_assert(!PAIR || (BNC % 64 == 0), "pair tiles hold whole 64-column B boxes");

  if (threadIdx.x == 0) {
    abort_flag_s = 0;
    // full barrier: the arming arrive (TMA bytes); with gathered rows also
    // one arrive per producer lane when its copies of the stage complete,
    // and in a pair the other CTA's forwarded arrive
    const uint32_t n_full = GATHER ? (PAIR ? 34u : 33u) : 1u;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), n_full);
      mbar_init(empty_bar(s), 1);
      mbar_init(cpd_bar(s), 32);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), kEpiWarps * (PAIR ? 2 : 1));   // both CTAs' epilogues
    }
    mbar_init(done_bar, 1);
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(epi_bar(w), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    __syncwarp();
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the set-up above touched only this CTA's shared and tensor memory
  pdl_begin();

  // Each role decodes tile t + n_units while it works on tile t, so the
  // global loads a decode needs (tile -> expert map, group offsets) never
  // stall a tile boundary.
  constexpr int kMU = PAIR ? 2 * BM : BM;
  const int n_mt = (MODE != MODE_ROWS) ? 0
                   : p.dense_m > 0    ? (p.dense_m + kMU - 1) / kMU
                                      : p.stats[3] / (PAIR ? 2 : 1);
  const int total = (MODE == MODE_ROWS) ? n_mt * p.nN : total_hint;
  auto decode_at = [&](int t) {
    return t < total ? decode<MODE, EPI, BN, PAIR>(t, p, rank, n_mt) : Tile{0, 0, 0, 0, 0};
  };

  if (warp == 0) {
    if constexpr (GATHER) {
      // ---------- producer with gathered rows (whole warp) ----------
      // The row operand (A of a ROWS tile, B of a WGRAD k block) is copied
      // from the token rows of x with 16-byte cp.async: one warp
      // instruction moves 4 rows x 128 bytes (lane = 8 * row + chunk).  The
      // tile's (ROWS) or k block's (WGRAD) tokens go through a small
      // shared table; row slots are loaded one tile / k block ahead.  Lane 0
      // waits for free stages, arms the barrier for the TMA box loads of
      // the other operand and issues them.
      static_assert((MODE == MODE_ROWS && EPI == EPI_SWIGLU && !A_MN) ||
                        (MODE == MODE_WGRAD && B_MN),
                    "gathered operands: gate/up A rows or gate/up wgrad B rows");
      constexpr int kRowsG = MODE == MODE_ROWS ? BM : BK;   // gathered rows per stage
      int32_t* tok_s = reinterpret_cast<int32_t*>(gbase + S::kTokOff);
      const uint32_t tok_a = smem_u32(tok_s);
      const int shared0 = p.offsets[p.E];
      const int cch = lane & 7, rsub = lane >> 3;
      // first row of the gathered rows this lane's slot loads cover
      auto lane_row = [&](const Tile& d, int kb) {
        return MODE == MODE_ROWS ? d.m0 + 4 * lane : d.row0 + kb * BK + 2 * lane;
      };
      constexpr int kSl = kRowsG / 32;   // slots per lane: 4 (ROWS) or 2 (WGRAD)
      auto load_slots = [&](const Tile& d, int kb, bool valid, int (&v)[kSl]) {
        const int32_t* q = p.row_slot + lane_row(d, kb);
#pragma unroll
        for (int i = 0; i < kSl; ++i) v[i] = valid ? q[i] : -1;
      };
      auto token = [&](int r, int sl) {
        if (sl >= 0) return sl / p.gK;
        const int u = r - shared0;
        return (u >= 0 && u < p.shared_T) ? u : -1;   // -1: zeros
      };
      int sl[kSl];
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
      // the gathered rows of one stage -> this lane's tokens (row rsub + 4 i)
      int tk[kRowsG / 4];
      auto publish = [&](const Tile& d, int kb) {
        const int r = lane_row(d, kb);
        __syncwarp();   // every lane has read the previous table
#pragma unroll
        for (int i = 0; i < kSl; ++i)
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(tok_a + 4u * (kSl * lane + i)),
                       "r"(token(r + i, sl[i]))
                       : "memory");
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kRowsG / 4; ++i) {
          int v;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(tok_a + 4u * (rsub + 4 * i)) : "memory");
          tk[i] = v;
        }
      };
      bool ok = true;
      Tile nxt = decode_at(unit);
      load_slots(nxt, 0, unit < total && nxt.nk > 0, sl);
      for (int t = unit; t < total && ok; t += n_units) {
        const Tile d = nxt;
        nxt = decode_at(t + n_units);
        const bool nxt_ok = t + n_units < total && nxt.nk > 0;
        if (d.nk == 0) { load_slots(nxt, 0, nxt_ok, sl); continue; }
        const CUtensorMap* mb = (MODE == MODE_ROWS && d.e >= p.E) ? &mapBs : &mapB;
        const int eb = (MODE == MODE_ROWS && d.e >= p.E) ? 0 : d.e;
        if (MODE == MODE_ROWS) {
          publish(d, 0);
          load_slots(nxt, 0, nxt_ok, sl);
        }
        for (int kb = 0; kb < d.nk; ++kb) {
          if (MODE == MODE_WGRAD) {
            publish(d, kb);
            if (kb + 1 < d.nk) load_slots(d, kb + 1, true, sl);
            else load_slots(nxt, 0, nxt_ok, sl);
          }
          int w = 1;
          if (lane == 0) w = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag) ? 1 : 0;
          if (__shfl_sync(0xffffffffu, w, 0) == 0) { ok = false; break; }
          const uint32_t sa = base + stage * S::kStage;
          const uint32_t sb = sa + S::kA;
          const uint32_t fb = full_bar(stage);
          if (lane == 0) {
            const uint32_t tb = PAIR ? mapa(fb, 0) : fb;   // barrier the TMA copies complete on
            const uint32_t box_bytes = MODE == MODE_ROWS ? S::kB : S::kA;
            if (!PAIR || leader) mbar_expect_tx(fb, box_bytes * (PAIR ? 2 : 1));
            issued_parity[stage] = (int)phase;
            if constexpr (MODE == MODE_ROWS) {
              if constexpr (PAIR) {
                tma_3d_pair(sb, mb, tb, kb * BK, (rank ? p.F : 0) + d.n0, eb);
              } else {
                tma_3d(sb, mb, tb, kb * BK, d.n0, eb);
                tma_3d(sb + (BN / 2) * 128, mb, tb, kb * BK, p.F + d.n0, eb);
              }
            } else {
              const int r = d.row0 + kb * BK;
              if constexpr (PAIR) {
                tma_2d_pair_nohint(sa, &mapA, tb, d.m0, r);
                tma_2d_pair_nohint(sa + 8192, &mapA, tb, d.m0 + 64, r);
              } else {
                tma_2d(sa, &mapA, tb, d.m0, r);
                tma_2d(sa + 8192, &mapA, tb, d.m0 + 64, r);
              }
            }
          }
          if constexpr (MODE == MODE_ROWS) {
            // A: 128 rows x 64 columns of x; row rsub + 4 i, chunk cch
            const __nv_bfloat16* src0 = p.gx + kb * BK + cch * 8;
#pragma unroll
            for (int i = 0; i < BM / 4; ++i) {
              const int r = rsub + 4 * i;
              const int tkn = tk[i];
              cp_async16(sa + r * 128 + ((cch ^ (r & 7)) << 4),
                         src0 + (int64_t)(tkn < 0 ? 0 : tkn) * p.Kd, tkn < 0 ? 0u : 16u);
            }
          } else {
            // B: 64 rows (k) x BNC columns of x, in 64-column boxes
            const int col0 = d.n0 + (PAIR ? rank * BNC : 0) + cch * 8;
#pragma unroll
            for (int c = 0; c < BNC / 64; ++c) {
              const __nv_bfloat16* src0 = p.gx + col0 + c * 64;
#pragma unroll
              for (int i = 0; i < BK / 4; ++i) {
                const int r = rsub + 4 * i;
                const int tkn = tk[i];
                cp_async16(sb + c * 8192 + r * 128 + ((cch ^ (r & 7)) << 4),
                           src0 + (int64_t)(tkn < 0 ? 0 : tkn) * p.No, tkn < 0 ? 0u : 16u);
              }
            }
          }
          cp_async_arrive(PAIR && !leader ? cpd_bar(stage) : fb);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      cp_async_wait_all();   // no copy of this CTA in flight at teardown
      if (lane == 0 && (!PAIR || leader))
        for (int s = 0; s < STAGES; ++s)
          if (issued_parity[s] >= 0) mbar_wait(full_bar(s), (uint32_t)issued_parity[s], abort_flag);
    } else if (lane == 0) {
      // ---------------- TMA producer (both CTAs of a pair) ----------------
      const uint64_t pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
      bool ok = true;
      Tile nxt = decode_at(unit);
      for (int t = unit; t < total && ok; t += n_units) {
        const Tile d = nxt;
        nxt = decode_at(t + n_units);
        const CUtensorMap* mb = (MODE == MODE_ROWS && d.e >= p.E) ? &mapBs : &mapB;
        const int eb = (MODE == MODE_ROWS && d.e >= p.E) ? 0 : d.e;
        for (int kb = 0; kb < d.nk; kb += KB) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const int nb = d.nk - kb < KB ? d.nk - kb : KB;
          const uint32_t sa = base + stage * S::kStage;
          const uint32_t sb = sa + KB * S::kA;
          const uint32_t fb = full_bar(stage);
          if (!PAIR || leader) mbar_expect_tx(fb, (S::kA + S::kB) * nb * (PAIR ? 2 : 1));
          issued_parity[stage] = (int)phase;
          if constexpr (PAIR) {
            const uint32_t lfb = mapa(fb, 0);           // the leader's full barrier
            if (MODE == MODE_ROWS) {
              for (int j = 0; j < nb; ++j) {
              const int kbj = kb + j;
              const uint32_t saj = sa + j * S::kA, sbj = sb + j * S::kB;
              tma_2d_pair(saj, &mapA, lfb, kbj * BK, d.m0, pol_a);
#pragma unroll
              for (int m = 0; m < NBM; ++m) {
                const uint32_t sbm = sbj + m * BLK * 128;
                if (EPI == EPI_SWIGLU) {
                  // this CTA holds the gate (rank 0) or the up (rank 1) rows
                  // of MMA block m: j = n0 + m BLK ...
                  tma_3d_pair(sbm, mb, lfb, kbj * BK, (rank ? p.F : 0) + d.n0 + m * BLK, eb);
                } else if (!B_MN) {
                  tma_3d_pair(sbm, mb, lfb, kbj * BK, d.n0 + m * NMM + rank * BLK, eb);
                } else {
#pragma unroll
                  for (int c = 0; c < BLK / 64; ++c)
                    tma_3d_pair(sbm + c * 8192, mb, lfb, d.n0 + m * NMM + rank * BLK + c * 64,
                                kbj * BK, eb);
                }
              }
              }
            } else {
              for (int j = 0; j < nb; ++j) {
                const int r = d.row0 + (kb + j) * BK;
                const uint32_t saj = sa + j * S::kA, sbj = sb + j * S::kB;
                tma_2d_pair_nohint(saj, &mapA, lfb, d.m0, r);
                tma_2d_pair_nohint(saj + 8192, &mapA, lfb, d.m0 + 64, r);
#pragma unroll
                for (int m = 0; m < NBM; ++m)
#pragma unroll
                  for (int c = 0; c < BLK / 64; ++c)
                    tma_2d_pair_nohint(sbj + m * BLK * 128 + c * 8192, &mapB, lfb,
                                       d.n0 + m * NMM + rank * BLK + c * 64, r);
              }
            }
          } else {
            for (int j = 0; j < nb; ++j) {
              const int kbj = kb + j;
              const uint32_t saj = sa + j * S::kA, sbj = sb + j * S::kB;
              if (MODE == MODE_ROWS) {
                tma_2d_hint(saj, &mapA, fb, kbj * BK, d.m0, pol_a);
                if (EPI == EPI_SWIGLU) {
                  tma_3d(sbj, mb, fb, kbj * BK, d.n0, eb);
                  tma_3d(sbj + (BN / 2) * 128, mb, fb, kbj * BK, p.F + d.n0, eb);
                } else if (!B_MN) {
                  tma_3d(sbj, mb, fb, kbj * BK, d.n0, eb);
                } else {
#pragma unroll
                  for (int c = 0; c < BN / 64; ++c)
                    tma_3d(sbj + c * 8192, mb, fb, d.n0 + c * 64, kbj * BK, eb);
                }
              } else {
                const int r = d.row0 + kbj * BK;
                tma_2d(saj, &mapA, fb, d.m0, r);
                tma_2d(saj + 8192, &mapA, fb, d.m0 + 64, r);
#pragma unroll
                for (int c = 0; c < BN / 64; ++c)
                  tma_2d(sbj + c * 8192, &mapB, fb, d.n0 + c * 64, r);
              }
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // drain: the copies this CTA's barriers track have landed before
      // teardown (a pair's copies all complete on the leader's barriers)
      if (!PAIR || leader)
        for (int s = 0; s < STAGES; ++s)
          if (issued_parity[s] >= 0) mbar_wait(full_bar(s), (uint32_t)issued_parity[s], abort_flag);
    }
  } else if (warp == 1) {
    if constexpr (PAIR && GATHER) {
      // ---- second CTA of a pair: forward completed gathered stages ----
      if (lane == 0 && !leader) {
        int stage = 0;
        uint32_t phase = 0;
        Tile nxt = decode_at(unit);
        bool ok = true;
        for (int t = unit; t < total && ok; t += n_units) {
          const Tile d = nxt;
          nxt = decode_at(t + n_units);
          for (int kb = 0; kb < d.nk; ++kb) {
            if (!mbar_wait(cpd_bar(stage), phase, abort_flag)) { ok = false; break; }
            fence_proxy_async();
            mbar_arrive_remote(mapa(full_bar(stage), 0));
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
        }
      }
    }
    // ---------------- MMA issuer (the pair leader only) ----------------
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = make_idesc(PAIR ? 2 * BM : BM, NMM, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      Tile nxt = decode_at(unit);
      for (int t = unit; t < total && ok; t += n_units) {
        const Tile d = nxt;
        nxt = decode_at(t + n_units);
        if (d.nk == 0) continue;
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t dt = tmem + acc * BN;
        for (int kb = 0; kb < d.nk; kb += KB) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, PAIR && GATHER)) { ok = false; break; }
          if constexpr (GATHER) fence_proxy_async();   // cp.async rows -> async proxy
          tc_fence_after();
          const int nb = d.nk - kb < KB ? d.nk - kb : KB;
          for (int j = 0; j < nb; ++j) {
          const uint32_t sa = base + stage * S::kStage + j * S::kA;
          const uint32_t sb = base + stage * S::kStage + KB * S::kA + j * S::kB;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t ad = A_MN ? sw128_desc(sa + ks * 2048, 8192, 1024)
                                     : sw128_desc(sa + ks * 32, 16, 1024);
#pragma unroll
            for (int m = 0; m < NBM; ++m) {
              const uint32_t sbm = sb + m * BLK * 128;
              const uint64_t bd = B_MN ? sw128_desc(sbm + ks * 2048, 8192, 1024)
                                       : sw128_desc(sbm + ks * 32, 16, 1024);
              if constexpr (PAIR) umma_pair(dt + m * NMM, ad, bd, idesc, (kb | j | ks) != 0 ? 1u : 0u);
              else umma(dt + m * NMM, ad, bd, idesc, (kb | j | ks) != 0 ? 1u : 0u);
            }
          }
          }   // j
          if constexpr (PAIR) umma_commit_pair_both(empty_bar(stage));
          else umma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) umma_commit_pair_both(accf_bar(acc));
        else umma_commit(accf_bar(acc));
        if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread complete before teardown
      if constexpr (PAIR) umma_commit_pair_local(done_bar);
      else umma_commit(done_bar);
      mbar_wait(done_bar, 0, abort_flag);
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    // Two warps per TMEM lane quarter q = warp % 4 (the lanes a warp may
    // read); warp half hh takes the first or second half of the columns.
    const int q = warp & 3;
    const int hh = (warp - 2) >> 2;
    const int rloc = q * 32 + lane;
    constexpr int HC = BN / 2;           // columns per warp (plain epilogues)
    constexpr int HJ = BN / 4;           // gate (= up) columns per warp (SwiGLU)
    const uint64_t pol_out = policy_evict_first();
    const uint32_t stg = base + S::kEpiOff + (warp - 2) * S::kStgW;   // staging tile
    // Output blocks (32 rows x 32 columns, bf16) go out as TMA stores from
    // two staging boxes (lane 0 issues and tracks them): they move the bytes
    // faster than the warp's own global stores, which shortens the 512-wide
    // tiles' unoverlapped epilogue and frees the others' epilogue warps
    // sooner.  u: this lane's row of the block, packed.
    int box = 0;
    auto tma_out_pk = [&](const uint4 (&u)[4], const CUtensorMap* map, int x, int64_t y) {
      const uint32_t buf = stg + box * kTmaBox;
      box ^= 1;
      if (lane == 0) bulk_wait_read_1();   // the store that last read `buf` is done with it
      __syncwarp();
      stage_box_sw64(buf, u);
      fence_proxy_async();                 // visible to the async proxy
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(map, buf, x, (int)y);
        bulk_commit();
      }
    };
    auto tma_out = [&](const float (&v)[32], const CUtensorMap* map, int x, int64_t y) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) u[j] = pack8_bf16(v + 8 * j);
      tma_out_pk(u, map, x, y);
    };
    // a plain-store / weight-gradient block at column x of this warp's rows
    // (weight gradient: expert d.e's rows of the stacked routed experts, or
    // the shared expert's tensor)
    auto tma_out_tile = [&](const Tile& d, const uint4 (&u)[4], int x, int64_t row0) {
      if constexpr (EPI == EPI_WGRAD) {
        if (d.e < p.E) tma_out_pk(u, &mapO, x, d.e * (p.strideCE / p.No) + row0);
        else tma_out_pk(u, &mapO2, x, row0);
      } else {
        tma_out_pk(u, &mapO, x, row0);
      }
    };
    if constexpr (EPI == EPI_COMBINE1 || EPI == EPI_DX1) {
      // tokens whose slot holds no row (sentinel, dropped): y_t = 0, or
      // dx_t = ds_t . W_r (the router part alone), while the first tile's
      // main loop runs.  Each lane checks one token (one load per lane for
      // a whole grid's worth of tokens); the warp writes the masked ones.
      const int stride = gridDim.x * kEpiWarps * 32;
      for (int t0 = (blockIdx.x * kEpiWarps + (warp - 2)) * 32; t0 < p.T; t0 += stride) {
        const bool masked = t0 + lane < p.T && p.slot_row[t0 + lane] < 0;
        unsigned todo = __ballot_sync(0xffffffffu, masked);
        while (todo != 0u) {
          const int t = t0 + __ffs(todo) - 1;
          todo &= todo - 1u;
          __nv_bfloat16* dst = p.tout + (int64_t)t * p.ld_out;
          float dse[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) dse[e] = (EPI == EPI_DX1 && e < p.Er) ? p.ds[(int64_t)t * p.Er + e] : 0.f;
          for (int c = lane * 8; c < p.ld_out; c += 256) {
            float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if constexpr (EPI == EPI_DX1) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                if (e < p.Er) {
                  float w[8];
                  load8(p.w_r + (int64_t)e * p.ld_out + c, w);
#pragma unroll
                  for (int i = 0; i < 8; ++i) a[i] = fmaf(dse[e], w[i], a[i]);
                }
              }
            }
            store8(dst + c, a);
          }
        }
      }
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t bwd_phase = 0;   // parity of this warp's a13 load barrier
    Tile nxt = decode_at(unit);
    for (int t = unit; t < total; t += n_units) {
      const Tile d = nxt;
      nxt = decode_at(t + n_units);
      if (EPI == EPI_WGRAD && d.nk == 0) {
        __nv_bfloat16* og = d.e < p.E ? p.out + (int64_t)d.e * p.strideCE : p.out_shared;
        __nv_bfloat16* dst = og + (int64_t)(d.m0 + rloc) * p.No + d.n0 + hh * HC;
        for (int c = 0; c < HC; c += 8) zero8(dst + c);
        continue;
      }
      const int64_t row0 = d.m0 + q * 32;   // this warp's first row
      // SwiGLU backward: this warp's first a and b blocks of the saved a13
      // are requested before the accumulator wait so their latency overlaps
      // the main loop (192-wide tiles: coalesced loads, each later block
      // fetched kPf blocks ahead; others: TMA into the staging boxes, each
      // later chunk's blocks once the previous chunk's dA13 stores have read
      // the boxes).
      constexpr int kNch = HC / 32;
      constexpr int kPf = kNch < 2 ? kNch : 2;
      uint4 pa[EPI == EPI_SWIGLU_BWD ? kPf : 1][4], pb[EPI == EPI_SWIGLU_BWD ? kPf : 1][4];
      const __nv_bfloat16* a13s = p.aux + row0 * p.ld_aux + d.n0 + hh * HC;
      const uint32_t eb = epi_bar(warp - 2);
      auto bwd_load = [&](int c) {
        if (lane == 0) {
          bulk_wait_read_0();
          mbar_expect_tx(eb, 2 * kTmaBox);
          tma_2d(stg, &mapO, eb, d.n0 + hh * HC + c, (int)row0);
          tma_2d(stg + kTmaBox, &mapO, eb, p.F + d.n0 + hh * HC + c, (int)row0);
        }
      };
      if constexpr (kTmaBwd) {
        bwd_load(0);
      } else if constexpr (EPI == EPI_SWIGLU_BWD) {
#pragma unroll
        for (int c = 0; c < kPf; ++c) {
          block_load32(a13s + 32 * c, p.ld_aux, pa[c]);
          block_load32(a13s + p.F + 32 * c, p.ld_aux, pb[c]);
        }
      }
      // token-order epilogues: this lane's row -> token, gate weight or ds
      int my_tok = -1;
      float my_g = 0.f, dse[EPI == EPI_DX1 ? 8 : 1];
      if constexpr (EPI == EPI_COMBINE1 || EPI == EPI_DX1) {
        my_tok = p.row_slot[row0 + lane];
        if constexpr (EPI == EPI_COMBINE1) {
          if (my_tok >= 0) my_g = p.tw[my_tok];
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dse[e] = (my_tok >= 0 && e < p.Er) ? p.ds[(int64_t)my_tok * p.Er + e] : 0.f;
        }
      }
      bool ok = (lane == 0) ? mbar_wait(accf_bar(acc), acc_phase, abort_flag) : true;
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + acc * BN;
      if constexpr ((EPI == EPI_STORE || EPI == EPI_WGRAD) && HC <= (kTmaOut ? 256 : 128)) {
        // the whole accumulator slice is read (packed to bf16 in registers:
        // up to 128 of them for the 512-wide tiles) and released before the
        // stores, so the next tile's MMAs need not wait for this tile's
        // global stores
        __nv_bfloat16* w0;
        int64_t ld;
        if (EPI == EPI_STORE) {
          w0 = p.out + row0 * p.ld_out + d.n0 + hh * HC;
          ld = p.ld_out;
        } else {
          __nv_bfloat16* og = d.e < p.E ? p.out + (int64_t)d.e * p.strideCE : p.out_shared;
          w0 = og + row0 * p.No + d.n0 + hh * HC;
          ld = p.No;
        }
        uint4 pk[HC / 32][4];
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld32(tbase + hh * HC + c, r);
          tmem_wait();
          u2f32(r, v);
#pragma unroll
          for (int j = 0; j < 4; ++j) pk[c / 32][j] = pack8_bf16(v + 8 * j);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (!PAIR || leader) mbar_arrive(acce_bar(acc));
          else mbar_arrive_remote(mapa(acce_bar(acc), 0));   // the leader's barrier
        }
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          if constexpr (kTmaOut) tma_out_tile(d, pk[c / 32], d.n0 + hh * HC + c, row0);
          else staged_store32_pk(stg, pk[c / 32], w0 + c, ld, pol_out);
        }
        if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
        continue;
      } else if constexpr (EPI == EPI_STORE || EPI == EPI_WGRAD) {
        __nv_bfloat16* w0;
        int64_t ld;
        if (EPI == EPI_STORE) {
          w0 = p.out + row0 * p.ld_out + d.n0 + hh * HC;
          ld = p.ld_out;
        } else {
          __nv_bfloat16* og = d.e < p.E ? p.out + (int64_t)d.e * p.strideCE : p.out_shared;
          w0 = og + row0 * p.No + d.n0 + hh * HC;
          ld = p.No;
        }
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld32(tbase + hh * HC + c, r);
          tmem_wait();
          u2f32(r, v);
          if constexpr (kTmaOut) {
            uint4 u[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) u[j] = pack8_bf16(v + 8 * j);
            tma_out_tile(d, u, d.n0 + hh * HC + c, row0);
          } else {
            staged_store32(stg, v, w0 + c, ld, pol_out);
          }
        }
      } else if constexpr (EPI == EPI_COMBINE1 || EPI == EPI_DX1) {
        const int col0 = d.n0 + hh * HC;
        __nv_bfloat16* w0 = p.out + row0 * p.ld_out + col0;
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld32(tbase + hh * HC + c, r);
          tmem_wait();
          u2f32(r, v);
          if constexpr (EPI == EPI_COMBINE1) {
            staged_store32(stg, v, w0 + c, p.ld_out, pol_out);   // o, row order
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= my_g;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if (e < p.Er) {
                const float* wr = p.w_r + (int64_t)e * p.ld_out + col0 + c;
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                  const float4 w = *reinterpret_cast<const float4*>(wr + 4 * q4);
                  v[4 * q4] = fmaf(dse[e], w.x, v[4 * q4]);
                  v[4 * q4 + 1] = fmaf(dse[e], w.y, v[4 * q4 + 1]);
                  v[4 * q4 + 2] = fmaf(dse[e], w.z, v[4 * q4 + 2]);
                  v[4 * q4 + 3] = fmaf(dse[e], w.w, v[4 * q4 + 3]);
                }
              }
            }
          }
          staged_store32_tok(stg, v, p.tout + col0 + c, p.ld_out, my_tok, pol_out);
        }
      } else if constexpr (EPI == EPI_SWIGLU) {
        // accumulator columns of MMA block m: gate j in [m JB, (m+1) JB) at
        // [2 m JB, 2 m JB + JB), up for the same j at the next JB columns
        constexpr int JB = BN / 2 < 128 ? BN / 2 : 128;
        __nv_bfloat16* a13 = p.out + row0 * p.ld_out + d.n0 + hh * HJ;
        __nv_bfloat16* hr = p.out2 + row0 * p.ld_out2 + d.n0 + hh * HJ;
#pragma unroll
        for (int c = 0; c < HJ; c += 32) {
          uint32_t rg[32], ru[32];
          float ga[32], ub[32];
          const int jl = hh * HJ + c;
          const int gc = (jl / JB) * 2 * JB + jl % JB;
          tmem_ld32(tbase + gc, rg);
          tmem_ld32(tbase + gc + JB, ru);
          tmem_wait();
          u2f32(rg, ga);
          u2f32(ru, ub);
          const int xc = d.n0 + hh * HJ + c;   // column of gate j (up: + F) and of h
          if constexpr (kTmaOut) {
            // gate and up blocks: both boxes, one fence, one bulk group
            uint4 ug[4], uu[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              ug[j] = pack8_bf16(ga + 8 * j);
              uu[j] = pack8_bf16(ub + 8 * j);
            }
            if (lane == 0) bulk_wait_read_0();   // the last h store has read box 0
            __syncwarp();
            stage_box_sw64(stg, ug);
            stage_box_sw64(stg + kTmaBox, uu);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&mapO, stg, xc, (int)row0);
              tma_store_2d(&mapO, stg + kTmaBox, p.F + xc, (int)row0);
              bulk_commit();
            }
          } else {
            staged_store32(stg, ga, a13 + c, p.ld_out, pol_out);
            staged_store32(stg, ub, a13 + p.F + c, p.ld_out, pol_out);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) ga[i] = ga[i] * fast_sigmoid(ga[i]) * ub[i];
          if constexpr (kTmaOut) {
            // h block: box 0 once the gate / up stores have read it
            uint4 uh[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) uh[j] = pack8_bf16(ga + 8 * j);
            if (lane == 0) bulk_wait_read_0();
            __syncwarp();
            stage_box_sw64(stg, uh);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&mapO2, stg, xc, (int)row0);
              bulk_commit();
            }
          } else {
            staged_store32(stg, ga, hr + c, p.ld_out2, pol_out);
          }
        }
      } else if constexpr (EPI == EPI_F32 || EPI == EPI_WGRAD_F32) {
        const int64_t row = row0 + lane;
        const bool rv = row < (EPI == EPI_F32 ? (int64_t)p.dense_m : (int64_t)p.m_limit);
        float* dst = p.out_f32 + row * p.ld_f32 + d.n0 + hh * HC +
                     (EPI == EPI_WGRAD_F32 ? (int64_t)d.e * p.strideCE : 0);   // K-split partial
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld32(tbase + hh * HC + c, r);
          tmem_wait();
          u2f32(r, v);
          if constexpr (kTmaF32) {   // rows past dense_m: clipped by the tensor map
            if (lane == 0) bulk_wait_read_0();   // the last store has read the box
            __syncwarp();
            stage_box_f32_sw128(stg, v);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&mapO, stg, d.n0 + hh * HC + c, (int)row0);
              bulk_commit();
            }
          } else {
            if (rv) store32_f32(dst + c, v);
          }
        }
      } else if constexpr (kTmaBwd) {
#pragma unroll 1
        for (int c = 0; c < HC; c += 32) {
          uint32_t r[32];
          float dh[32], av[32], bv[32];
          tmem_ld32(tbase + hh * HC + c, r);
          mbar_wait(eb, bwd_phase, abort_flag);   // this chunk's a13 blocks landed
          bwd_phase ^= 1u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t o = lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
            bf16x8_to_f(lds128(stg + o), av + 8 * j);
            bf16x8_to_f(lds128(stg + kTmaBox + o), bv + 8 * j);
          }
          tmem_wait();
          u2f32(r, dh);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sg = fast_sigmoid(av[i]);
            const float da = dh[i] * bv[i] * sg * (1.f + av[i] * (1.f - sg));
            bv[i] = dh[i] * av[i] * sg;
            av[i] = da;
          }
          uint4 ua[4], ub[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ua[j] = pack8_bf16(av + 8 * j);
            ub[j] = pack8_bf16(bv + 8 * j);
          }
          stage_box_sw64(stg, ua);              // dA13 in place of the a13 blocks
          stage_box_sw64(stg + kTmaBox, ub);
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            const int xg = d.n0 + hh * HC + c;
            tma_store_2d(&mapO2, stg, xg, (int)row0);
            tma_store_2d(&mapO2, stg + kTmaBox, p.F + xg, (int)row0);
            bulk_commit();
          }
          if (c + 32 < HC) bwd_load(c + 32);
        }
      } else {  // EPI_SWIGLU_BWD
        __nv_bfloat16* da13 = p.out + row0 * p.ld_out + d.n0 + hh * HC;
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t r[32];
          float dh[32], av[32], bv[32];
          const int ci = c / 32, slot = ci % kPf;
          tmem_ld32(tbase + hh * HC + c, r);
          staged_rows32(stg, pa[slot], av);
          staged_rows32(stg, pb[slot], bv);
          if (ci + kPf < kNch) {
            block_load32(a13s + 32 * (ci + kPf), p.ld_aux, pa[slot]);
            block_load32(a13s + p.F + 32 * (ci + kPf), p.ld_aux, pb[slot]);
          }
          tmem_wait();
          u2f32(r, dh);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sg = fast_sigmoid(av[i]);
            const float da = dh[i] * bv[i] * sg * (1.f + av[i] * (1.f - sg));
            bv[i] = dh[i] * av[i] * sg;
            av[i] = da;
          }
          staged_store32(stg, av, da13 + c, p.ld_out, pol_out);
          staged_store32(stg, bv, da13 + p.F + c, p.ld_out, pol_out);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (!PAIR || leader) mbar_arrive(acce_bar(acc));
        else mbar_arrive_remote(mapa(acce_bar(acc), 0));   // the leader's barrier
      }
      if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
    }
  }
  if constexpr (kTmaOut || kTmaBwd || kTmaF32) {
    if (warp >= 2 && lane == 0) bulk_wait_all();   // this warp's output stores are written
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // the leader's MMAs into both CTAs are done
  tc_fence_after();
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

}  // namespace tc
}  // namespace moe
