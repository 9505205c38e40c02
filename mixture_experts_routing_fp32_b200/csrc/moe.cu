// libmoe.so: the extern "C" entry points declared in include/moe.h.
// One translation unit (the device error word is a single __device__
// variable); the kernels live in the .cuh files beside this one.
#include <cuda.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <numeric>
#include <type_traits>
#include <utility>

#include "common.cuh"
#include "router.cuh"
#include "dispatch.cuh"
#include "combine.cuh"
#include "expert_choice.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "router_tc.cuh"

using namespace moe;

namespace {

thread_local int g_last_cuda_error = 0;
thread_local int64_t g_launches = 0;

// Optional per-launch timing: a begin and an end event recorded on the
// launching stream around every kernel (moe_profile_* entry points).
constexpr int kProfMax = 256;
struct Prof {
  cudaEvent_t ev[2 * kProfMax];
  const char* name[kProfMax];
  int side[kProfMax];
  int n = 0, cap = 0;
};
thread_local Prof g_prof;

// Under stream capture the records must be real event-record nodes
// (cudaEventRecordExternal; re-recorded on every replay), not the
// capture-internal dependency markers a plain record becomes; outside
// capture that flag is invalid, so a plain record is used.
inline void prof_record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, s);
}
inline void prof_begin(cudaStream_t s) {
  if (g_prof.n < g_prof.cap) prof_record(g_prof.ev[2 * g_prof.n], s);
}
bool is_side_stream(cudaStream_t s);
inline void prof_end(cudaStream_t s, const char* name) {
  if (g_prof.n < g_prof.cap) {
    g_prof.side[g_prof.n] = is_side_stream(s) ? 1 : 0;
    prof_record(g_prof.ev[2 * g_prof.n + 1], s);
    g_prof.name[g_prof.n++] = name;
  }
}

#define MOE_CK(expr)                                   \
  do {                                                 \
    cudaError_t e__ = (expr);                          \
    if (e__ != cudaSuccess) {                          \
      g_last_cuda_error = (int)e__;                    \
      return MOE_ERR_CUDA;                             \
    }                                                  \
  } while (0)
#define MOE_LAUNCHED(s, name)                          \
  do {                                                 \
    ++g_launches;                                      \
    cudaError_t e__ = cudaGetLastError();              \
    if (e__ != cudaSuccess) {                          \
      g_last_cuda_error = (int)e__;                    \
      return MOE_ERR_CUDA;                             \
    }                                                  \
    prof_end((s), (name));                             \
  } while (0)
#define MOE_TRY(expr)                                  \
  do {                                                 \
    int r__ = (expr);                                  \
    if (r__ != MOE_OK) return r__;                     \
  } while (0)

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

size_t act_bytes(const moe_config_t* c) { return c->dtype == MOE_BF16 ? 2 : 4; }

int validate(const moe_config_t* c) {
  if (c == nullptr) return MOE_ERR_ARG;
  if (c->T < 1 || c->D < 8 || (c->D % 8) || c->F < 8 || (c->F % 8)) return MOE_ERR_ARG;
  if (c->E < 1 || c->E > kMaxExperts) return MOE_ERR_ARG;
  if (c->expert_choice != 0 && c->expert_choice != 1) return MOE_ERR_ARG;
  if (c->expert_choice) {
    // expert choice in the slot layout: one slot per (token, expert) pair
    if (c->K != c->E || c->score_fn != MOE_SOFTMAX || c->renorm != 0 || c->n_groups != 1 ||
        !(c->capacity_factor > 0.f) || c->aux_alpha != 0.f || c->seq_len != 0 ||
        c->route_scale != 1.f)
      return MOE_ERR_ARG;
  } else if (c->K < 1 || c->K > c->E || c->K > kMaxK) {
    return MOE_ERR_ARG;
  }
  if (c->n_shared != 0 && c->n_shared != 1) return MOE_ERR_ARG;
  if (c->dtype != MOE_FP32 && c->dtype != MOE_BF16) return MOE_ERR_ARG;
  if (c->score_fn != MOE_SOFTMAX && c->score_fn != MOE_SIGMOID) return MOE_ERR_ARG;
  if (c->renorm != 0 && c->renorm != 1) return MOE_ERR_ARG;
  if (c->n_groups < 1 || c->n_groups > 32 || (c->E % c->n_groups)) return MOE_ERR_ARG;
  if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return MOE_ERR_ARG;
  if ((int64_t)c->topk_groups * (c->E / c->n_groups) < c->K) return MOE_ERR_ARG;
  if (c->group_score != MOE_GMAX && c->group_score != MOE_GTOP2SUM) return MOE_ERR_ARG;
  if (c->n_groups > 1 && c->group_score == MOE_GTOP2SUM && c->E / c->n_groups < 2)
    return MOE_ERR_ARG;
  if (c->seq_len < 0 || (c->seq_len > 0 && (c->T % c->seq_len))) return MOE_ERR_ARG;
  // the batch aux loss is defined for softmax scores; the sequence-wise
  // one also for sigmoid affinities (normalised over experts)
  if (c->aux_alpha != 0.f && c->score_fn != MOE_SOFTMAX && c->seq_len == 0) return MOE_ERR_ARG;
  if (!(c->route_scale == c->route_scale) || c->min_capacity < 0) return MOE_ERR_ARG;
  if ((int64_t)c->T * c->K > (int64_t)INT32_MAX / 2) return MOE_ERR_ARG;
  if (c->gemm_impl != MOE_GEMM_AUTO && c->gemm_impl != MOE_GEMM_SIMT) return MOE_ERR_ARG;
  // globally scoped batch losses: N >= T tokens; not for the sequence-wise
  // loss (its sequences live on one rank) or expert choice
  if (c->loss_tokens < 0 || (c->loss_tokens > 0 && c->loss_tokens < c->T)) return MOE_ERR_ARG;
  if (c->loss_tokens > 0 && (c->seq_len != 0 || c->expert_choice)) return MOE_ERR_ARG;
  // expert shards: a range of the routed experts, on the tensor-core path,
  // token choice, no shared expert
  if (c->expert_base < 0 || c->n_local_experts < 0 ||
      (int64_t)c->expert_base + c->n_local_experts > c->E)
    return MOE_ERR_ARG;
  if (c->expert_base > 0 && c->n_local_experts == 0) return MOE_ERR_ARG;
  if (c->n_local_experts > 0 &&
      (c->expert_choice || c->n_shared || c->seq_len || c->dtype != MOE_BF16 ||
       c->gemm_impl != MOE_GEMM_AUTO ||
       (c->D % 128) || (c->F % 128)))
    return MOE_ERR_ARG;
  return MOE_OK;
}

// Routed experts this call's expert FFN holds (expert parallelism), and the first.
int local_E(const moe_config_t* c) { return c->n_local_experts > 0 ? c->n_local_experts : c->E; }
int expert_base(const moe_config_t* c) { return c->n_local_experts > 0 ? c->expert_base : 0; }

// Token count the batch aux and z losses average over.
int64_t loss_tokens_of(const moe_config_t* c) { return c->loss_tokens > 0 ? c->loss_tokens : c->T; }

// Expert choice: tokens each expert picks, C = min(T, max(ceil(c*T/E), min_capacity)).
int64_t ec_capacity(const moe_config_t* c) {
  const double v = std::ceil((double)c->capacity_factor * (double)c->T / (double)c->E);
  return std::min<int64_t>(c->T, std::max<int64_t>((int64_t)v, c->min_capacity));
}

// Token-choice drop capacity (-1: none; expert choice never drops in the
// dispatch, its picks already hold C slots per expert).
int64_t capacity_of(const moe_config_t* c) {
  if (c->expert_choice) return -1;
  if (!(c->capacity_factor > 0.f)) return -1;
  const double v = std::ceil((double)c->capacity_factor * (double)((int64_t)c->T * c->K) /
                             (double)c->E);
  return std::max<int64_t>((int64_t)v, c->min_capacity);
}

bool use_tc(const moe_config_t* c) {
  return c->dtype == MOE_BF16 && c->gemm_impl == MOE_GEMM_AUTO && (c->D % 128) == 0 &&
         (c->F % 128) == 0;
}

int64_t capacity_of(const moe_config_t* c);

// The router's fp32 products (logits, dW_r, the router part of dx) run on
// tensor cores as bf16 MMAs over three-way bf16 splits of the fp32 operand
// when the expert GEMMs do and E >= 8; below that the SIMT kernels are as
// fast.  Ep = E rounded up to 64 (split width).
bool router_tc(const moe_config_t* c) { return use_tc(c) && c->E >= 8; }
// The backward's router part of dx on CUDA cores inside the unpermute-sum
// (bf16 token choice, E <= 8, K in {1, 2, 4, 8}); MOE_ROUTER_DX_TC=1 keeps
// the tensor-core product for E = 8 (for cross-checks).
bool small_router_dx(const moe_config_t* c) {
  static const bool force_tc = [] {
    const char* v = std::getenv("MOE_ROUTER_DX_TC");
    return v != nullptr && v[0] == '1';
  }();
  return !force_tc && c->dtype == MOE_BF16 && !c->expert_choice && c->E <= 8 &&
         (c->K == 1 || c->K == 2 || c->K == 4 || c->K == 8);
}
bool router_dx_tc(const moe_config_t* c) {
  return router_tc(c) && (c->expert_choice || !small_router_dx(c));
}
// dW_r = ds^T x on tensor cores (three-way bf16 splits of ds, token-range
// split) on the tensor-core path; for E < 8 with token choice only (the
// expert-choice backward forms both router splits together), where it
// measured level with the two-stage SIMT form on the MiniMind shape
// (25.5 us either way, the step 1 us shorter); MOE_ROUTER_DW_TC=0 keeps
// the SIMT form there.
bool router_dw_tc(const moe_config_t* c) {
  static const bool small = [] {
    const char* v = std::getenv("MOE_ROUTER_DW_TC");
    return !(v != nullptr && v[0] == '0');
  }();
  return router_tc(c) || (small && use_tc(c) && !c->expert_choice);
}
// Token-choice routing inside the tensor-core logits kernel: up to 64
// experts, no group limit, K in {1, 2, 4, 8} (MOE_ROUTER_FUSED=0: for
// E >= 8 the partial-logit GEMM and a separate routing kernel instead, for
// fewer experts the CUDA-core router; for cross-checks).
bool router_fused_tc(const moe_config_t* c) {
  static const bool on = [] {
    const char* v = std::getenv("MOE_ROUTER_FUSED");
    return !(v != nullptr && v[0] == '0');
  }();
  return on && use_tc(c) && !c->expert_choice && c->E <= 64 && c->n_groups == 1 &&
         (c->K == 1 || c->K == 2 || c->K == 4 || c->K == 8);
}
int64_t router_ep(const moe_config_t* c) { return (c->E + 63) / 64 * 64; }
// Token ranges of the tensor-core dW_r product (a K split): with few output
// tiles (3 Ep / 128 x D / 128, E <= 64 and a narrow D) up to four ranges,
// so about one tile per SM of the 148 runs; the partials are summed in
// range order.  Returns the rows per range (a multiple of 64).
int dwr_split_rows(const moe_config_t* c) {
  const int64_t tiles = ceil_div(3 * router_ep(c), 128) * ceil_div(c->D, 128);
  const int64_t want = std::max<int64_t>(1, std::min<int64_t>(4, 148 / tiles));
  return (int)round_up(ceil_div(c->T, want), 64);
}
int dwr_splits(const moe_config_t* c) {
  return (int)ceil_div(c->T, dwr_split_rows(c));
}

// Row GEMMs run on CTA pairs (two SMs share each 256-row MMA) when experts
// hold enough rows that aligning their segments to 256 rows wastes little
// and the extra operand reuse pays (at least 1536 rows on average: measured
// faster for the OLMoE- and Mixtral-shaped layers, slower for 1024-row
// experts); the permuted row space is then 256-row aligned.  Otherwise
// segments are 128-row aligned and single-CTA tiles run.
bool pair_rows(const moe_config_t* c) {
  if (!use_tc(c)) return false;
  const int64_t C = capacity_of(c);
  const int64_t slots = (int64_t)c->T * c->K;
  const int64_t kept = c->expert_choice ? (int64_t)c->E * ec_capacity(c)
                       : C < 0          ? slots
                                        : std::min<int64_t>(slots, (int64_t)c->E * C);
  return kept / c->E >= 1536;
}

int row_align(const moe_config_t* c) { return pair_rows(c) ? 256 : kRowTile; }

struct Layout {
  int64_t rows_max, tiles_max, C, n_slots;
  int n_disp_blocks, n_aux_chunks, n_dwr_chunks, dwr_chunk, align;
  size_t off_bhist, off_bsent, off_aux, off_dg, off_ds, off_dwr, off_dO, off_dA13, off_dX,
      off_dH, total;
  // tensor-core router products (router_tc)
  int64_t Ep;
  size_t off_wf, off_wb, off_rparts, off_dsf, off_dsb, off_dwr3, off_rdx;
  // sequence-wise aux (seq_len > 0): per-sequence f [n_seq, E]; partial
  // counts / sums of n_split pieces of each sequence
  int64_t n_seq, n_split;
  size_t off_seqf, off_seqc, off_seqq, off_seqz, off_seqs;
};
constexpr int kAuxChunk = 128;

// Tokens per dW_r partial: enough chunks that the (E x D) tiles of all
// chunks fill about two waves of 148 SMs; one chunk when the tiles alone do.
int64_t dwr_chunk_tokens(const moe_config_t* c) {
  const int64_t tiles = (c->E <= 8) ? ceil_div(c->D, 256)
                                    : ceil_div(c->D, 64) * ceil_div(c->E, 64);
  const int64_t want = std::max<int64_t>(1, ceil_div(2 * 148, tiles));
  return std::max<int64_t>(32, round_up(ceil_div(c->T, want), 32));
}

Layout layout_of(const moe_config_t* c) {
  Layout L{};
  L.C = capacity_of(c);
  L.n_slots = (int64_t)c->T * c->K;
  const int64_t El = local_E(c);
  const int64_t kept_total = c->expert_choice ? (int64_t)c->E * ec_capacity(c)
                             : L.C < 0        ? L.n_slots
                                              : std::min<int64_t>(L.n_slots, El * L.C);
  const int64_t align = row_align(c);
  const int64_t pad = (align - 1) * std::min<int64_t>(El, kept_total);
  L.rows_max = round_up(kept_total + pad, align) + (c->n_shared ? round_up(c->T, align) : 0);
  if (L.rows_max == 0) L.rows_max = align;
  L.align = (int)align;
  L.tiles_max = L.rows_max / kRowTile;
  L.n_disp_blocks = (int)ceil_div(L.n_slots, kDispChunk);
  L.n_aux_chunks = (int)ceil_div(c->T, kAuxChunk);
  L.dwr_chunk = (int)dwr_chunk_tokens(c);
  L.n_dwr_chunks = (int)ceil_div(c->T, L.dwr_chunk);
  const size_t a = act_bytes(c);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += round_up((int64_t)bytes, 256); return o; };
  L.off_bhist = take((size_t)L.n_disp_blocks * c->E * 4);
  L.off_bsent = take((size_t)L.n_disp_blocks * 4);
  L.off_aux = take((size_t)L.n_aux_chunks * (c->E + 1) * 4);
  L.off_dg = take((size_t)L.n_slots * 4);
  L.off_ds = take((size_t)c->T * c->E * 4);
  L.off_dwr = take((size_t)L.n_dwr_chunks * c->E * c->D * 4);
  L.off_dO = take((size_t)L.rows_max * c->D * a);
  L.off_dA13 = take((size_t)L.rows_max * 2 * c->F * a);
  L.off_dX = take((size_t)L.rows_max * c->D * a);
  L.off_dH = use_tc(c) ? off : take((size_t)L.rows_max * c->F * a);
  if (router_tc(c) || router_fused_tc(c) || router_dw_tc(c)) L.Ep = router_ep(c);
  if (router_tc(c) || router_fused_tc(c)) L.off_wf = take((size_t)3 * L.Ep * c->D * 2);
  if (router_tc(c)) L.off_rparts = take((size_t)c->T * 3 * L.Ep * 4);
  if (router_dw_tc(c)) {
    L.off_dsf = take((size_t)c->T * 3 * L.Ep * 2);
    L.off_dwr3 = take((size_t)dwr_splits(c) * 3 * L.Ep * c->D * 4);
  }
  if (router_dx_tc(c)) {   // the router part of dx on tensor cores
    L.off_wb = take((size_t)3 * L.Ep * c->D * 2);
    L.off_dsb = take((size_t)c->T * 3 * L.Ep * 2);
    L.off_rdx = take((size_t)c->T * c->D * 4);
  }
  if (c->seq_len > 0) {
    L.n_seq = c->T / c->seq_len;
    // pieces of up to 32 tokens, about two waves of blocks over all sequences
    L.n_split = std::max<int64_t>(1, std::min<int64_t>(ceil_div(c->seq_len, 32),
                                                       ceil_div(2 * 148, L.n_seq)));
    L.off_seqf = take((size_t)L.n_seq * c->E * 4);
    L.off_seqc = take((size_t)L.n_seq * L.n_split * c->E * 4);
    L.off_seqq = take((size_t)L.n_seq * L.n_split * c->E * 4);
    L.off_seqz = take((size_t)L.n_seq * L.n_split * 4);
    L.off_seqs = take((size_t)L.n_seq * 4);
  }
  L.total = off;
  return L;
}

template <typename T>
T* wsp(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor [n3][rows][cols] (n3 = 1 for 2D), box {64, box_rows}, 128B swizzle.
int make_map(CUtensorMap* m, const void* ptr, int64_t n3, int64_t rows, int64_t cols,
             uint32_t box_rows, bool three_d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) { g_last_cuda_error = (int)cudaErrorNotSupported; return MOE_ERR_CUDA; }
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)n3};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)(rows * cols * 2)};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, three_d ? 3 : 2, const_cast<void*>(ptr),
                  dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { g_last_cuda_error = (int)cudaErrorInvalidValue; return MOE_ERR_CUDA; }
  return MOE_OK;
}

// Programmatic dependent launch on by default (MOE_PDL=0 turns it off):
// every kernel waits for its stream predecessor with griddepcontrol.wait
// before its first global access, so the launch attribute only lets the
// next kernel be scheduled, and its set-up run, while this one drains.
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_PDL");
    return !(v != nullptr && v[0] == '0');
  }();
  return on;
}

template <typename... KP, typename... A>
cudaError_t launch_k(void (*kern)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     A&&... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&lc, kern, std::forward<A>(args)...);
}

// Tensors the epilogues move through TMA (SwiGLU: a13, h; plain store: out;
// weight gradient: the routed experts' [E * rows, cols] and the shared
// expert's; SwiGLU backward: the saved a13 it loads, dA13), see
// make_store_map.
struct OutMaps {
  CUtensorMap o1, o2;
};

// bf16 tensor [rows][cols] for the epilogues' TMA loads and stores: box
// {32, 32}, 64-byte swizzle.
int make_store_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) { g_last_cuda_error = (int)cudaErrorNotSupported; return MOE_ERR_CUDA; }
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { g_last_cuda_error = (int)cudaErrorInvalidValue; return MOE_ERR_CUDA; }
  return MOE_OK;
}

// fp32 tensor [rows][cols] as TMA-store target: box {32, 32}, 128-byte swizzle.
int make_store_map_f32(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) { g_last_cuda_error = (int)cudaErrorNotSupported; return MOE_ERR_CUDA; }
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { g_last_cuda_error = (int)cudaErrorInvalidValue; return MOE_ERR_CUDA; }
  return MOE_OK;
}

template <int BN, int ST, int MODE, bool AMN, bool BMN, int EPI, bool PAIR, bool GATHER>
int launch_tc(const char* name, const CUtensorMap& a, const CUtensorMap& b,
              const CUtensorMap& bs, const tc::Params& p, int64_t total_max, int total_hint,
              cudaStream_t s, const OutMaps* om) {
  using S = tc::KernelSmem<BN, ST, MODE, PAIR, GATHER>;
  auto k = tc::gemm_kernel<BN, ST, MODE, AMN, BMN, EPI, PAIR, GATHER>;
  // the SwiGLU, plain-store, weight-gradient and SwiGLU-backward epilogues
  // move their blocks through TMA (all tile widths but 192)
  constexpr bool tma_out = BN != 192 && (EPI == tc::EPI_SWIGLU || EPI == tc::EPI_STORE ||
                                         EPI == tc::EPI_WGRAD || EPI == tc::EPI_SWIGLU_BWD ||
                                         EPI == tc::EPI_F32);
  if (tma_out && om == nullptr) return MOE_ERR_ARG;
  const CUtensorMap& o1 = om != nullptr ? om->o1 : a;
  const CUtensorMap& o2 = om != nullptr ? om->o2 : a;
  MOE_CK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes));
  if constexpr (PAIR) {
    // as many CTA pairs as can be resident at once (one per two SMs of a GPC)
    static int max_pairs = 0;
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.blockDim = dim3(tc::kThreads);
    lc.dynamicSmemBytes = S::kBytes;
    lc.stream = s;
    lc.attrs = attr;
    lc.numAttrs = 1;
    if (max_pairs == 0) {
      lc.gridDim = dim3(2 * (num_sms() / 2));
      int n = 0;
      MOE_CK(cudaOccupancyMaxActiveClusters(&n, k, &lc));
      max_pairs = n > 0 ? n : num_sms() / 2;
    }
    const int pairs = (int)std::min<int64_t>(max_pairs, total_max);
    if (pairs <= 0) return MOE_OK;
    lc.gridDim = dim3(2 * pairs);
    lc.numAttrs = pdl_enabled() ? 2 : 1;
    prof_begin(s);
    MOE_CK(cudaLaunchKernelEx(&lc, k, a, b, bs, o1, o2, p, total_hint));
    MOE_LAUNCHED(s, name);
  } else {
    const int grid = (int)std::min<int64_t>(num_sms(), total_max);
    if (grid <= 0) return MOE_OK;
    prof_begin(s);
    MOE_CK((launch_k(k, grid, tc::kThreads, S::kBytes, s, a, b, bs, o1, o2, p, total_hint)));
    MOE_LAUNCHED(s, name);
  }
  return MOE_OK;
}

template <int MODE, bool AMN, bool BMN, int EPI, bool PAIR = false, bool GATHER = false>
int run_tc(int bn, const char* name, const CUtensorMap& a, const CUtensorMap& b,
           const CUtensorMap& bs, const tc::Params& p, int64_t total_max, int total_hint,
           cudaStream_t s, const OutMaps* om = nullptr) {
  if constexpr (PAIR) {
    // per CTA: A 16 KB + half of B per stage
    if constexpr (!GATHER) {
      if (bn == 512)   // two stages of two k blocks (tc::stage_kb)
        return launch_tc<512, 2, MODE, AMN, BMN, EPI, true, false>(name, a, b, bs, p, total_max,
                                                                  total_hint, s, om);
    }
    if constexpr (!GATHER) {
      if (bn == 256)   // two k blocks per stage (tc::stage_kb)
        return launch_tc<256, 3, MODE, AMN, BMN, EPI, true, false>(name, a, b, bs, p, total_max,
                                                                  total_hint, s, om);
    }
    if (bn == 256)
      return launch_tc<256, 6, MODE, AMN, BMN, EPI, true, GATHER>(name, a, b, bs, p, total_max,
                                                                 total_hint, s, om);
    if constexpr (!GATHER) {
      if (bn == 128)
        return launch_tc<128, 4, MODE, AMN, BMN, EPI, true, false>(name, a, b, bs, p, total_max,
                                                                  total_hint, s, om);
    }
    if (bn == 128)
      return launch_tc<128, 8, MODE, AMN, BMN, EPI, true, GATHER>(name, a, b, bs, p, total_max,
                                                                 total_hint, s, om);
    return MOE_ERR_ARG;
  } else {
    if (bn == 256)
      return launch_tc<256, 4, MODE, AMN, BMN, EPI, false, GATHER>(name, a, b, bs, p, total_max,
                                                                  total_hint, s, om);
    if constexpr (EPI != tc::EPI_SWIGLU) {
      if (bn == 192)
        return launch_tc<192, 5, MODE, AMN, BMN, EPI, false, GATHER>(name, a, b, bs, p,
                                                                    total_max, total_hint, s, om);
    }
    if constexpr (!GATHER) {
      if (bn == 128)
        return launch_tc<128, 3, MODE, AMN, BMN, EPI, false, false>(name, a, b, bs, p, total_max,
                                                                   total_hint, s, om);
    }
    if (bn == 128)
      return launch_tc<128, 6, MODE, AMN, BMN, EPI, false, GATHER>(name, a, b, bs, p, total_max,
                                                                  total_hint, s, om);
    return MOE_ERR_ARG;
  }
}

// Expected 128-row tiles of the permuted rows (half a tile of padding per
// expert on average), used only to choose tile widths.
int64_t row_tiles_estimate(const moe_config_t* c, const Layout& L) {
  const int64_t kept_total = c->expert_choice ? (int64_t)c->E * ec_capacity(c)
                             : L.C < 0        ? L.n_slots
                                              : std::min<int64_t>(L.n_slots, (int64_t)local_E(c) * L.C);
  const int64_t rows = kept_total + 64 * std::min<int64_t>(local_E(c), kept_total);
  return ceil_div(rows, kRowTile) + (c->n_shared ? ceil_div(c->T, kRowTile) : 0);
}

// Output tile width BN in {512, 256, 192, 128} minimising the busiest SM's
// time, waves x BN / efficiency(BN): a narrower tile loads the same A rows
// for fewer columns, so it moves more bytes per FLOP and keeps the tensor
// pipe less busy (measured: BN=128 about 0.8 of BN=256 per column; a
// 256-row CTA pair with BN=256 is limited by operand delivery into the SM,
// which BN=512 halves per MMA).  BN=512 runs on CTA pairs with one
// accumulator, so its epilogue is not overlapped: it is offered only for
// tiles of at least kMinKb512 k blocks (nk; 0 = unknown).  Ties keep the
// wider tile.  SwiGLU tiles hold BN/2 gate and BN/2 up columns of F.
constexpr int64_t kMinKb512 = 48;
bool bn512_enabled();
int pick_bn(int64_t N, int64_t mtiles, bool swiglu, int64_t F, bool pair = false,
            int64_t nk = 0) {
  const int64_t sms = pair ? num_sms() / 2 : num_sms();
  if (pair) mtiles = ceil_div(mtiles, 2);
  int best = 0;
  int64_t best_cost = INT64_MAX;
  for (int bn : {512, 256, 192, 128}) {
    if (pair && bn == 192) continue;
    if (bn == 512 && !(pair && nk >= kMinKb512 && bn512_enabled())) continue;
    const int64_t eff_pct = bn == 512 ? 125 : bn == 256 ? 100 : bn == 192 ? 95 : 80;
    int64_t nt;
    if (swiglu) {
      if (bn == 192 || F % (bn / 2)) continue;
      nt = F / (bn / 2);
    } else {
      if (N % bn) continue;
      nt = N / bn;
    }
    const int64_t cost = ceil_div(mtiles * nt, sms) * bn * 100 / eff_pct;
    if (cost < best_cost) { best_cost = cost; best = bn; }
  }
  return best;
}

int grid_for(int64_t items_per_8, int cap_mult = 8) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(items_per_8, 8), (int64_t)num_sms() * cap_mult));
}

// ---------------------------------------------------------------------------
// router
// ---------------------------------------------------------------------------
int group_rows(int64_t Kd, bool pair = false);

// Routing of each token from logits (or from the tensor-core partial
// logits), one warp per token.
int route_launch(const moe_config_t* c, const RouteArgs& a, const float* logits,
                 const float* parts, int64_t Ep, const float* off, cudaStream_t s) {
  // from the partial logits with E a multiple of 32 and groups (if any) of
  // 32 experts: E / 32 lanes per token, one per 32-expert chunk
  const int L = c->E / 32;
  if (parts != nullptr && c->E % 32 == 0 && L <= 32 && (L & (L - 1)) == 0 &&
      (c->n_groups == 1 || c->E / c->n_groups == 32) && c->K <= 8) {
    auto go = [&](auto l, auto km) -> int {
      constexpr int LL = decltype(l)::value, KM = decltype(km)::value;
      const int grid = (int)ceil_div((int64_t)c->T * LL, 256);
      prof_begin(s);
      MOE_CK((launch_k(router_route_lanes_kernel<LL, KM>, grid, 256, 0, s, parts, (int)Ep, off, a)));
      MOE_LAUNCHED(s, "router_route");
      return MOE_OK;
    };
    auto by_k = [&](auto l) -> int {
      if (c->K <= 2) return go(l, std::integral_constant<int, 2>{});
      if (c->K <= 4) return go(l, std::integral_constant<int, 4>{});
      return go(l, std::integral_constant<int, 8>{});
    };
    switch (L) {
      case 1: return by_k(std::integral_constant<int, 1>{});
      case 2: return by_k(std::integral_constant<int, 2>{});
      case 4: return by_k(std::integral_constant<int, 4>{});
      case 8: return by_k(std::integral_constant<int, 8>{});
      case 16: return by_k(std::integral_constant<int, 16>{});
      default: return by_k(std::integral_constant<int, 32>{});
    }
  }
  const size_t sm = 8 * (size_t)c->E * 4;
  const int grid = grid_for(c->T);
  auto go = [&](auto nv) -> int {
    constexpr int NV = decltype(nv)::value;
    prof_begin(s);
    if (parts != nullptr)
      MOE_CK((launch_k(router_route_parts_kernel<NV>, grid, 256, sm, s, parts, (int)Ep, off, a)));
    else
      MOE_CK((launch_k(router_route_kernel<NV>, grid, 256, sm, s, logits, a)));
    MOE_LAUNCHED(s, "router_route");
    return MOE_OK;
  };
  if (c->E <= 32) return go(std::integral_constant<int, 1>{});
  if (c->E <= 64) return go(std::integral_constant<int, 2>{});
  if (c->E <= 128) return go(std::integral_constant<int, 4>{});
  if (c->E <= 256) return go(std::integral_constant<int, 8>{});
  return go(std::integral_constant<int, 16>{});
}

template <typename TX>
int router_impl(const moe_config_t* c, const TX* x, const float* w_r, const float* off,
                const float* bias, float* logits, float* probs, float* lse, int32_t* idx,
                float* w, int32_t* ties, void* ws, cudaStream_t s) {
  RouteArgs a{c->T, c->E, c->K, c->score_fn, c->renorm, c->n_groups, c->topk_groups,
              c->group_score, c->route_scale, bias, logits, probs, lse, idx, w, ties};
  MOE_CK(cudaMemsetAsync(ties, 0, sizeof(int32_t), s));
  if (router_fused_tc(c)) {
    // logits on tensor cores (the three splits stacked along N of one MMA)
    // and the routing in the same kernel's epilogue
    const Layout L = layout_of(c);
    // split width: E rounded up to 8, 16, 32 or 64 (fewer W_r bytes per
    // tile for few experts)
    const int EP = c->E <= 8 ? 8 : c->E <= 16 ? 16 : c->E <= 32 ? 32 : 64;
    auto* wf = wsp<__nv_bfloat16>(ws, L.off_wf);
    prof_begin(s);
    MOE_CK((launch_k(split_w_kernel, grid_for((int64_t)EP * c->D / 256), 256, 0, s, w_r, c->E,
                     EP, c->D, wf, (__nv_bfloat16*)nullptr)));
    MOE_LAUNCHED(s, "router_split_w");
    // E > 16: CTA pairs (each CTA streams half of the split rows)
    const bool pair = EP >= 32;
    // Tile height: as many 128-token rounds as the token count needs over
    // all CTAs, then the tokens spread evenly over them (a multiple of 8,
    // at least 64 so that few tokens do not spread over many CTAs that each
    // stream all of W_r).
    if (c->T == 0) return MOE_OK;
    static int max_pairs = 0;   // resident CTA pairs (the same for every split width)
    if (pair && max_pairs == 0) {
      auto k = rtc::router_tc_kernel<64, 8, true>;
      constexpr int sm = rtc::Smem<64, true>::kBytes;
      MOE_CK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, sm));
      cudaLaunchConfig_t lc = {};
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      lc.gridDim = dim3(2 * (num_sms() / 2));
      lc.blockDim = dim3(rtc::kThreads);
      lc.dynamicSmemBytes = sm;
      lc.attrs = at;
      lc.numAttrs = 1;
      int n = 0;
      MOE_CK(cudaOccupancyMaxActiveClusters(&n, k, &lc));
      max_pairs = n > 0 ? n : num_sms() / 2;
    }
    const int ctas = pair ? 2 * max_pairs : num_sms();
    const int64_t rounds = ceil_div(c->T, (int64_t)128 * ctas);
    int bm = (int)round_up(ceil_div(c->T, rounds * ctas), 8);
    bm = std::max(64, std::min(128, bm));
    const int64_t units = ceil_div(c->T, (int64_t)(pair ? 2 * bm : bm));
    const int NA = (3 * EP + 15) / 16 * 16;
    CUtensorMap mX, mW;
    MOE_TRY(make_map(&mX, x, 1, c->T, c->D, (uint32_t)bm, false));
    MOE_TRY(make_map(&mW, wf, 1, 3 * EP, c->D, (uint32_t)(pair ? NA / 2 : 3 * EP), false));
    auto go = [&](auto kern, size_t smem, auto pr) -> int {
      constexpr bool PR = decltype(pr)::value;
      MOE_CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      if constexpr (PR) {
        cudaLaunchConfig_t lc = {};
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        lc.blockDim = dim3(rtc::kThreads);
        lc.dynamicSmemBytes = smem;
        lc.stream = s;
        lc.attrs = attr;
        lc.gridDim = dim3((unsigned)(2 * std::min<int64_t>(max_pairs, units)));
        lc.numAttrs = pdl_enabled() ? 2 : 1;
        prof_begin(s);
        MOE_CK(cudaLaunchKernelEx(&lc, kern, mX, mW, a, off, c->D, bm));
      } else {
        prof_begin(s);
        MOE_CK((launch_k(kern, (int)std::min<int64_t>(num_sms(), units), rtc::kThreads, smem, s,
                         mX, mW, a, off, c->D, bm)));
      }
      MOE_LAUNCHED(s, "router_tc");
      return MOE_OK;
    };
    auto by_k = [&](auto ep, auto pr) -> int {
      constexpr int P = decltype(ep)::value;
      constexpr bool PR = decltype(pr)::value;
      constexpr size_t sm = rtc::Smem<P, PR>::kBytes;
      switch (c->K) {
        case 1: return go(rtc::router_tc_kernel<P, 1, PR>, sm, pr);
        case 2: return go(rtc::router_tc_kernel<P, 2, PR>, sm, pr);
        case 4: return go(rtc::router_tc_kernel<P, 4, PR>, sm, pr);
        default: return go(rtc::router_tc_kernel<P, 8, PR>, sm, pr);
      }
    };
    using NoPair = std::false_type;
    using Pair = std::true_type;
    if (EP == 8) return by_k(std::integral_constant<int, 8>{}, NoPair{});
    if (EP == 16) return by_k(std::integral_constant<int, 16>{}, NoPair{});
    if (EP == 32) return by_k(std::integral_constant<int, 32>{}, Pair{});
    return by_k(std::integral_constant<int, 64>{}, Pair{});
  }
  if (router_tc(c)) {
    // logits parts = x . (W_hi | W_mid | W_lo)^T on tensor cores (dense GEMM,
    // fp32 out), then routing sums the parts
    const Layout L = layout_of(c);
    const int64_t Ep = L.Ep, n3 = 3 * Ep;
    auto* wf = wsp<__nv_bfloat16>(ws, L.off_wf);
    float* parts = wsp<float>(ws, L.off_rparts);
    prof_begin(s);
    MOE_CK((launch_k(split_w_kernel, grid_for(Ep * c->D / 256), 256, 0, s, w_r, c->E, (int)Ep,
                     c->D, wf, (__nv_bfloat16*)nullptr)));
    MOE_LAUNCHED(s, "router_split_w");
    const int64_t mtiles = ceil_div(c->T, kRowTile);
    const int bn = pick_bn(n3, mtiles, false, 0, false);
    CUtensorMap mA, mB;
    MOE_TRY(make_map(&mA, x, 1, c->T, c->D, 128, false));
    MOE_TRY(make_map(&mB, wf, 1, n3, c->D, bn, true));       // dims {D, 3Ep, 1}
    tc::Params p{};
    p.E = 1; p.Kd = c->D; p.nN = (int)(n3 / bn); p.group_m = group_rows(c->D);
    p.dense_m = c->T;
    p.out_f32 = parts; p.ld_f32 = n3;
    OutMaps om;   // the partial logits as TMA-store target
    MOE_TRY(make_store_map_f32(&om.o1, parts, c->T, n3));
    om.o2 = om.o1;
    MOE_TRY((run_tc<tc::MODE_ROWS, false, false, tc::EPI_F32>(
        bn, "router_logits_tc", mA, mB, mB, p, mtiles * p.nN, 0, s, &om)));
    return route_launch(c, a, nullptr, parts, Ep, off, s);
  }
  const size_t fused_smem = 8 * (size_t)c->E * 4;
  if (c->E <= 32) {
    const int grid = grid_for(c->T);
    auto go = [&](auto kern) -> int {
      prof_begin(s);
      MOE_CK((launch_k(kern, grid, 256, fused_smem, s, x, w_r, off, c->D, a)));
      MOE_LAUNCHED(s, "router_fused");
      return MOE_OK;
    };
    if (c->K == 1 && c->E <= 4) return go(router_fused_kernel<TX, 4, 1>);
    if (c->K == 1 && c->E <= 8) return go(router_fused_kernel<TX, 8, 1>);
    if (c->E <= 4) return go(router_fused_kernel<TX, 4>);
    if (c->E <= 8) return go(router_fused_kernel<TX, 8>);
    if (c->E <= 16) return go(router_fused_kernel<TX, 16>);
    return go(router_fused_kernel<TX, 32>);
  }
  dim3 g1((unsigned)ceil_div(c->T, 64), (unsigned)ceil_div(c->E, 64));
  prof_begin(s);
  MOE_CK((launch_k(router_logits_kernel<TX>, g1, 256, 0, s, x, w_r, off, logits, c->T, c->D,
                   c->E)));
  MOE_LAUNCHED(s, "router_logits");
  return route_launch(c, a, logits, nullptr, 0, nullptr, s);
}

// ---------------------------------------------------------------------------
// aux / z loss
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
aux_partial_kernel(const float* __restrict__ probs, const float* __restrict__ lse, int T, int E,
                   float* __restrict__ part) {
  pdl_begin();
  // chunk c of kAuxChunk tokens: column sums of probs and the sum of lse^2,
  // each reduced in a fixed order (deterministic)
  __shared__ float red[256];
  const int c = blockIdx.x, tid = threadIdx.x;
  const int t0 = c * kAuxChunk, t1 = min(T, t0 + kAuxChunk);
  for (int e0 = 0; e0 < E; e0 += 256) {
    const int EB = min(256, E - e0);
    const int S = 256 / EB;             // token sub-streams per expert
    float s = 0.f;
    if (tid < S * EB) {
      const int e = e0 + tid % EB, sub = tid / EB;
      for (int t = t0 + sub; t < t1; t += S) s += probs[(size_t)t * E + e];
    }
    red[tid] = s;
    __syncthreads();
    if (tid < EB) {
      float acc = 0.f;
      for (int k = 0; k < S; ++k) acc += red[k * EB + tid];
      part[(size_t)c * (E + 1) + e0 + tid] = acc;
    }
    __syncthreads();
  }
  float z = 0.f;
  for (int t = t0 + tid; t < t1; t += 256) z += lse[t] * lse[t];
  red[tid] = z;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) red[tid] += red[tid + o];
    __syncthreads();
  }
  if (tid == 0) part[(size_t)c * (E + 1) + E] = red[0];
}

__global__ void __launch_bounds__(512)
aux_final_kernel(const float* __restrict__ part, const int32_t* __restrict__ counts, int n_chunks,
                 int T, int E, float alpha, float lambda, float* __restrict__ losses) {
  pdl_begin();
  // Every sum below runs in a fixed order that does not depend on timing:
  // a warp sums one expert's chunk partials (lane-strided, then a fixed
  // butterfly), the z partials likewise, then fixed-order block sums.
  __shared__ float red[512];
  __shared__ float fp_s[kMaxExperts];
  __shared__ float z_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float cnt = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt += (float)counts[e];
  red[threadIdx.x] = cnt;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  const float ctot = red[0];
  __syncthreads();
  for (int e = warp; e <= E; e += nw) {        // e == E: the z partials
    float v = 0.f;
    for (int c = lane; c < n_chunks; c += 32) v += part[(size_t)c * (E + 1) + e];
    v = warp_sum(v);
    if (lane == 0) {
      if (e < E) fp_s[e] = (ctot > 0.f ? (float)counts[e] / ctot : 0.f) * (v / (float)T);
      else z_s = v;
    }
  }
  __syncthreads();
  float acc = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) acc += fp_s[e];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    losses[0] = alpha * (float)E * red[0];
    losses[1] = lambda * z_s / (float)T;
  }
}

// Column sums of the aux partials: sums[e] = sum_t probs[t,e] (e < E),
// sums[E] = sum_t lse_t^2, each in aux_final_kernel's fixed order (a warp per
// column, lane-strided over the chunks, then the butterfly), so that
// aux_final_kernel on these sums (one "chunk") reproduces the local loss.
__global__ void __launch_bounds__(512)
aux_sums_kernel(const float* __restrict__ part, int n_chunks, int E, float* __restrict__ sums) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int e = warp; e <= E; e += nw) {
    float v = 0.f;
    for (int c = lane; c < n_chunks; c += 32) v += part[(size_t)c * (E + 1) + e];
    v = warp_sum(v);
    if (lane == 0) sums[e] = v;
  }
}

// ---------------------------------------------------------------------------
// expert FFN / backward GEMM sequences
// ---------------------------------------------------------------------------
template <typename TE>
int simt_rows(const moe_config_t* c, const Layout& L, const void* A, int64_t lda, const void* B,
              int64_t sbn, int64_t sbk, int64_t strideBE, const void* Bs, void* C, int64_t ldc,
              int N, int Kd, const int32_t* tile_expert, const int32_t* stats, cudaStream_t s) {
  SimtGemm g{};
  g.A = A; g.lda = lda; g.B = B; g.sbn = sbn; g.sbk = sbk; g.strideBE = strideBE;
  g.Bs = Bs ? Bs : B; g.C = C; g.ldc = ldc; g.N = N; g.Kd = Kd;
  g.tile_expert = tile_expert; g.stats = stats; g.E = c->E;
  dim3 grid((unsigned)(L.tiles_max * 2), (unsigned)ceil_div(N, 64));
  prof_begin(s);
  MOE_CK((launch_k(simt_rows_kernel<TE>, grid, 256, 0, s, g)));
  MOE_LAUNCHED(s, "simt_rows_gemm");
  return MOE_OK;
}

template <typename TE>
int simt_wgrad(const moe_config_t* c, const void* A, int64_t lda, const void* B, int64_t ldb,
               int Mo, int No, void* C, void* Cs, const int32_t* offsets, const int32_t* kept,
               cudaStream_t s) {
  SimtGemm g{};
  g.A = A; g.lda = lda; g.B = B; g.ldb = ldb; g.Mo = Mo; g.No = No;
  g.C = C; g.Cs = Cs; g.offsets = offsets; g.kept = kept; g.T = c->T; g.E = c->E;
  g.strideCE = (int64_t)Mo * No;
  dim3 grid((unsigned)ceil_div(No, 64), (unsigned)ceil_div(Mo, 64), (unsigned)(c->E + c->n_shared));
  prof_begin(s);
  MOE_CK((launch_k(simt_wgrad_kernel<TE>, grid, 256, 0, s, g)));
  MOE_LAUNCHED(s, "simt_wgrad_gemm");
  return MOE_OK;
}

// Side streams for the independent chains inside moe_backward (forked from
// and joined back into the caller's stream within the call; under stream
// capture the fork and join become graph edges).  Created once per host
// thread and device, on first use.
constexpr int kMaxSideDevices = 64;
struct Side {
  cudaStream_t st[3];
  cudaEvent_t ev[8];
  bool ok = false;
};
thread_local Side g_side[kMaxSideDevices];
thread_local bool g_side_enabled = true;   // moe_set_side_streams

thread_local const cudaStream_t* g_caller_side = nullptr;   // moe_set_backward_streams
thread_local cudaStream_t g_caller_side_st[3];

int side_streams(Side** out) {
  int dev = 0;
  MOE_CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxSideDevices) return MOE_ERR_ARG;
  Side& sd = g_side[dev];
  if (!sd.ok) {
    for (auto& st : sd.st) MOE_CK(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
    for (auto& ev : sd.ev) MOE_CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    sd.ok = true;
  }
  *out = &sd;
  return MOE_OK;
}

bool is_side_stream(cudaStream_t s) {
  if (g_caller_side != nullptr &&
      (s == g_caller_side[0] || s == g_caller_side[1] || s == g_caller_side[2]))
    return true;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return false;
  const Side& sd = g_side[dev];
  return sd.ok && (s == sd.st[0] || s == sd.st[1] || s == sd.st[2]);
}

// `to` waits for everything issued so far on `from`.
int fork_join(cudaEvent_t ev, cudaStream_t from, cudaStream_t to) {
  MOE_CK(cudaEventRecord(ev, from));
  MOE_CK(cudaStreamWaitEvent(to, ev, 0));
  return MOE_OK;
}

// 512-wide CTA-pair tiles (MOE_BN512=0 keeps BN <= 256, for comparison).
bool bn512_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_BN512");
    return !(v != nullptr && v[0] == '0');
  }();
  return on;
}

// Tile width of the weight-gradient GEMMs: pick_bn's choice, or
// MOE_WGRAD_BN (128, 256, or 512 on CTA pairs without the row gather, if it
// divides the output width) for tuning.
int wgrad_bn(int bn, int64_t n_out, bool pair512) {
  static const int forced = [] {
    const char* v = std::getenv("MOE_WGRAD_BN");
    return v != nullptr ? std::atoi(v) : 0;
  }();
  if ((forced == 128 || forced == 256 || (forced == 512 && pair512)) && n_out % forced == 0)
    return forced;
  return bn;
}

// Row tiles per rasterisation group: as many A row tiles of depth Kd as fit
// in about 24 MiB of L2, so they stay resident while the group sweeps the
// weight column slices (48 MiB measured 1-3% slower per step on the
// Mixtral and OLMoE shapes: the A tiles were read from DRAM again).
int group_rows(int64_t Kd, bool pair) {
  const int64_t rows = pair ? 256 : 128;
  return (int)std::max<int64_t>(1, std::min<int64_t>(64, (24ll << 20) / (rows * Kd * 2)));
}

tc::Params rows_params(const moe_config_t* c, int Kd, int nN, const int32_t* tile_expert,
                       const int32_t* stats, bool pair = false) {
  tc::Params p{};
  p.E = local_E(c); p.F = c->F; p.Kd = Kd; p.nN = nN; p.group_m = group_rows(Kd, pair);
  p.tile_expert = tile_expert; p.stats = stats; p.T = c->T;
  return p;
}

}  // namespace

// Dispatch passes: one block (histogram, scan and rank together) when the
// slots fit it, else the three multi-block passes through the per-block
// histograms in bhist/bsent; then the gather of x rows.
int dispatch_impl(const moe_config_t* c, const Layout& L, const int32_t* topk_idx,
                  const uint8_t* sentinel_mask, const void* x, int32_t* counts, int32_t* kept,
                  int32_t* offsets, int32_t* slot_row, int32_t* row_slot, int32_t* tile_expert,
                  int32_t* stats, void* x_perm, int32_t* bhist, int32_t* bsent, cudaStream_t s) {
  const int E = c->E, eb = expert_base(c), El = local_E(c);
  if (L.n_slots <= kSmallSlots) {
    const size_t smem = ((size_t)kSmallWarps * E + 2 * E + 1) * sizeof(int32_t);
    MOE_CK(cudaFuncSetAttribute(disp_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
    prof_begin(s);
    MOE_CK((launch_k(disp_small_kernel, 1, kSmallWarps * 32, smem, s, topk_idx, sentinel_mask,
                     L.n_slots, E, eb, El, c->T, c->n_shared, L.C, L.rows_max, L.align, counts,
                     kept, offsets, tile_expert, stats, slot_row, row_slot)));
    MOE_LAUNCHED(s, "dispatch_small");
  } else {
    prof_begin(s);
    MOE_CK((launch_k(disp_hist_kernel, L.n_disp_blocks, 256, E * sizeof(int32_t), s, topk_idx,
                     sentinel_mask, L.n_slots, E, bhist, bsent)));
    MOE_LAUNCHED(s, "dispatch_hist");
    prof_begin(s);
    MOE_CK((launch_k(disp_scan_kernel, 1, 1024, (2 * E + 1) * sizeof(int32_t), s, bhist, bsent,
                     L.n_disp_blocks, E, eb, El, c->T, c->n_shared, L.C, L.rows_max, L.align,
                     counts, kept, offsets, tile_expert, stats, row_slot)));
    MOE_LAUNCHED(s, "dispatch_scan");
    prof_begin(s);
    MOE_CK((launch_k(disp_rank_kernel, L.n_disp_blocks, 256,
                     (size_t)(kDispWarps + 1) * E * sizeof(int32_t), s, topk_idx, sentinel_mask,
                     L.n_slots, E, eb, El, L.C, L.rows_max, bhist, offsets, slot_row, row_slot)));
    MOE_LAUNCHED(s, "dispatch_rank");
  }
  if (x_perm == nullptr) return MOE_OK;   // layout only: the GEMMs gather x rows
  if (!c->expert_choice && (c->K == 1 || c->K == 2 || c->K == 4 || c->K == 8)) {
    // token order: each token's row of x read once for all its slots
    auto go = [&](auto tx, auto kt) -> int {
      using TX = decltype(tx);
      constexpr int KT = decltype(kt)::value;
      prof_begin(s);
      MOE_CK((launch_k(disp_gather_tok_kernel<TX, KT>, grid_for(c->T), 256, 0, s,
                       static_cast<const TX*>(x), c->D, El, c->T, c->n_shared, offsets, stats,
                       slot_row, row_slot, static_cast<TX*>(x_perm))));
      MOE_LAUNCHED(s, "dispatch_gather");
      return MOE_OK;
    };
    auto by_k = [&](auto tx) -> int {
      switch (c->K) {
        case 1: return go(tx, std::integral_constant<int, 1>{});
        case 2: return go(tx, std::integral_constant<int, 2>{});
        case 4: return go(tx, std::integral_constant<int, 4>{});
        default: return go(tx, std::integral_constant<int, 8>{});
      }
    };
    if (c->dtype == MOE_BF16) return by_k(__nv_bfloat16{});
    return by_k(float{});
  }
  const int grid = grid_for(L.rows_max);
  prof_begin(s);
  if (c->dtype == MOE_BF16)
    MOE_CK((launch_k(disp_gather_kernel<__nv_bfloat16>, grid, 256, 0, s,
                     static_cast<const __nv_bfloat16*>(x), c->D, c->K, El, c->T, offsets, stats,
                     row_slot, static_cast<__nv_bfloat16*>(x_perm))));
  else
    MOE_CK((launch_k(disp_gather_kernel<float>, grid, 256, 0, s, static_cast<const float*>(x),
                     c->D, c->K, El, c->T, offsets, stats, row_slot,
                     static_cast<float*>(x_perm))));
  MOE_LAUNCHED(s, "dispatch_gather");
  return MOE_OK;
}

// ===========================================================================
// extern "C" entry points
// ===========================================================================
extern "C" {

// x and W_r are read with 16-byte vector loads (and x through TMA).
static bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) != 0; }

int moe_get_sizes(const moe_config_t* cfg, moe_sizes_t* out) {
  MOE_TRY(validate(cfg));
  if (out == nullptr) return MOE_ERR_ARG;
  const Layout L = layout_of(cfg);
  out->rows_max = L.rows_max;
  out->tiles_max = L.tiles_max;
  out->capacity = L.C;
  out->ws_bytes = L.total;
  out->row_align = L.align;
  return MOE_OK;
}

int moe_router(const moe_config_t* c, const void* x, const float* w_r, const float* logit_offset,
               const float* sel_bias, float* logits, float* probs, float* lse, int32_t* topk_idx,
               float* topk_w, int32_t* near_ties, void* ws, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!x || !w_r || !logits || !probs || !lse || !topk_idx || !topk_w || !near_ties)
    return MOE_ERR_ARG;
  if (misaligned16(x) || misaligned16(w_r)) return MOE_ERR_ARG;
  if (c->expert_choice) return MOE_ERR_ARG;   // moe_route_expert_choice
  if ((router_tc(c) || router_fused_tc(c)) && ws == nullptr) return MOE_ERR_ARG;
  if (c->dtype == MOE_BF16)
    return router_impl(c, static_cast<const __nv_bfloat16*>(x), w_r, logit_offset, sel_bias,
                       logits, probs, lse, topk_idx, topk_w, near_ties, ws, s);
  return router_impl(c, static_cast<const float*>(x), w_r, logit_offset, sel_bias, logits, probs,
                     lse, topk_idx, topk_w, near_ties, ws, s);
}

}  // extern "C"

// Sequence-wise aux partials over (piece, sequence) blocks, then the final
// reduction: losses (if given) and the per-sequence f (if given).
int seq_aux_launch(const moe_config_t* c, const Layout& L, const float* probs, const float* lse,
                   const int32_t* topk_idx, const int32_t* slot_row, int norm, float* losses,
                   float* f_out, void* ws, cudaStream_t s) {
  int32_t* cnt = wsp<int32_t>(ws, L.off_seqc);
  float* qp = wsp<float>(ws, L.off_seqq);
  float* zp = wsp<float>(ws, L.off_seqz);
  const dim3 grid((unsigned)L.n_split, (unsigned)L.n_seq);
  auto go = [&](auto nv) -> int {
    prof_begin(s);
    MOE_CK((launch_k(seq_aux_partial_kernel<decltype(nv)::value>, grid, 256, 0, s, probs, lse,
                     topk_idx, slot_row, c->seq_len, c->K, c->E, norm, cnt, qp, zp)));
    MOE_LAUNCHED(s, "seq_aux_partial");
    return MOE_OK;
  };
  if (c->E <= 32) MOE_TRY(go(std::integral_constant<int, 1>{}));
  else if (c->E <= 64) MOE_TRY(go(std::integral_constant<int, 2>{}));
  else if (c->E <= 128) MOE_TRY(go(std::integral_constant<int, 4>{}));
  else if (c->E <= 256) MOE_TRY(go(std::integral_constant<int, 8>{}));
  else MOE_TRY(go(std::integral_constant<int, 16>{}));
  float* part = wsp<float>(ws, L.off_seqs);
  prof_begin(s);
  MOE_CK((launch_k(seq_aux_seq_kernel, (int)L.n_seq, 256, 0, s, cnt, qp, (int)L.n_split,
                   c->seq_len, c->E, part, f_out)));
  MOE_LAUNCHED(s, "seq_aux_seq");
  if (losses != nullptr) {
    prof_begin(s);
    MOE_CK((launch_k(seq_aux_final_kernel, 1, 256, 0, s, part, zp, (int)L.n_seq,
                     (int)(L.n_seq * L.n_split), c->T, c->E, c->aux_alpha, c->z_lambda,
                     losses)));
    MOE_LAUNCHED(s, "seq_aux_final");
  }
  return MOE_OK;
}

template <typename TX>
int route_ec_impl(const moe_config_t* c, const TX* x, const float* w_r, const float* off,
                  float* logits, float* probs, float* lse, int32_t* idx, float* w,
                  uint8_t* mask, int32_t* ties, void* ws, cudaStream_t s) {
  MOE_CK(cudaMemsetAsync(ties, 0, sizeof(int32_t), s));
  const int E = c->E;
  const float* parts = nullptr;
  int64_t Ep = 0;
  if (router_tc(c)) {
    const Layout L = layout_of(c);
    Ep = L.Ep;
    const int64_t n3 = 3 * Ep;
    auto* wf = wsp<__nv_bfloat16>(ws, L.off_wf);
    float* pt = wsp<float>(ws, L.off_rparts);
    prof_begin(s);
    MOE_CK((launch_k(split_w_kernel, grid_for(Ep * c->D / 256), 256, 0, s, w_r, E, (int)Ep,
                     c->D, wf, (__nv_bfloat16*)nullptr)));
    MOE_LAUNCHED(s, "router_split_w");
    const int64_t mtiles = ceil_div(c->T, kRowTile);
    const int bn = pick_bn(n3, mtiles, false, 0, false);
    CUtensorMap mA, mB;
    MOE_TRY(make_map(&mA, x, 1, c->T, c->D, 128, false));
    MOE_TRY(make_map(&mB, wf, 1, n3, c->D, bn, true));
    tc::Params p{};
    p.E = 1; p.Kd = c->D; p.nN = (int)(n3 / bn); p.group_m = group_rows(c->D);
    p.dense_m = c->T;
    p.out_f32 = pt; p.ld_f32 = n3;
    OutMaps om;   // the partial logits as TMA-store target
    MOE_TRY(make_store_map_f32(&om.o1, pt, c->T, n3));
    om.o2 = om.o1;
    MOE_TRY((run_tc<tc::MODE_ROWS, false, false, tc::EPI_F32>(
        bn, "router_logits_tc", mA, mB, mB, p, mtiles * p.nN, 0, s, &om)));
    parts = pt;
  } else {
    dim3 g1((unsigned)ceil_div(c->T, 64), (unsigned)ceil_div(E, 64));
    prof_begin(s);
    MOE_CK((launch_k(router_logits_kernel<TX>, g1, 256, 0, s, x, w_r, off, logits, c->T, c->D,
                     E)));
    MOE_LAUNCHED(s, "router_logits");
  }
  auto go = [&](auto nv) -> int {
    prof_begin(s);
    MOE_CK((launch_k(ec_scores_kernel<decltype(nv)::value>, grid_for(c->T), 256, 0, s, parts,
                     (int)Ep, parts != nullptr ? off : nullptr, c->T, E, logits, probs, lse,
                     idx, w)));
    MOE_LAUNCHED(s, "ec_scores");
    return MOE_OK;
  };
  if (E <= 32) MOE_TRY(go(std::integral_constant<int, 1>{}));
  else if (E <= 64) MOE_TRY(go(std::integral_constant<int, 2>{}));
  else if (E <= 128) MOE_TRY(go(std::integral_constant<int, 4>{}));
  else if (E <= 256) MOE_TRY(go(std::integral_constant<int, 8>{}));
  else MOE_TRY(go(std::integral_constant<int, 16>{}));
  prof_begin(s);
  MOE_CK((launch_k(ec_select_kernel, E, kEcThreads, 0, s, probs, c->T, E, (int)ec_capacity(c),
                   mask, ties)));
  MOE_LAUNCHED(s, "ec_select");
  return MOE_OK;
}

extern "C" {

int moe_route_expert_choice(const moe_config_t* c, const void* x, const float* w_r,
                                       const float* logit_offset, float* logits, float* probs,
                                       float* lse, int32_t* topk_idx, float* topk_w,
                                       uint8_t* sentinel_mask, int32_t* near_ties, void* ws,
                                       cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!c->expert_choice || !x || !w_r || !logits || !probs || !lse || !topk_idx || !topk_w ||
      !sentinel_mask || !near_ties)
    return MOE_ERR_ARG;
  if (misaligned16(x) || misaligned16(w_r)) return MOE_ERR_ARG;
  if (router_tc(c) && ws == nullptr) return MOE_ERR_ARG;
  if (c->dtype == MOE_BF16)
    return route_ec_impl(c, static_cast<const __nv_bfloat16*>(x), w_r, logit_offset, logits,
                         probs, lse, topk_idx, topk_w, sentinel_mask, near_ties, ws, s);
  return route_ec_impl(c, static_cast<const float*>(x), w_r, logit_offset, logits, probs, lse,
                       topk_idx, topk_w, sentinel_mask, near_ties, ws, s);
}

int moe_dispatch(const moe_config_t* c, const int32_t* topk_idx, const uint8_t* sentinel_mask,
                 const void* x, int32_t* counts, int32_t* kept, int32_t* offsets,
                 int32_t* slot_row, int32_t* row_slot, int32_t* tile_expert, int32_t* stats,
                 void* x_perm, void* ws, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!topk_idx || !x || !counts || !kept || !offsets || !slot_row || !row_slot ||
      !tile_expert || !stats || !ws)
    return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  return dispatch_impl(c, L, topk_idx, sentinel_mask, x, counts, kept, offsets, slot_row,
                       row_slot, tile_expert, stats, x_perm, wsp<int32_t>(ws, L.off_bhist),
                       wsp<int32_t>(ws, L.off_bsent), s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free dispatch.
//
// Some callers are handed only their input and output buffers and may not
// allocate device memory themselves: a plugin or custom-op host that offers
// no workspace hook and forbids cudaMalloc inside the op, or a serving
// runtime whose device memory plan is fixed before the first request.  They
// cannot provide the workspace moe_dispatch takes, so this variant keeps its
// only scratch (per-block expert histograms and sentinel counts) in the
// file-scope device array below.  Every GPU that loads the library holds the
// array until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t moe_static_scratch[MOE_STATIC_SCRATCH_BYTES / sizeof(int32_t)];

namespace {
constexpr int kMaxStaticDevices = 64;
std::mutex g_static_mu;
int32_t* g_static_scratch_ptr[kMaxStaticDevices] = {};

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// with the device current.  Outside stream capture it is looked up on every
// call (so a context torn down and re-created on the same ordinal, e.g.
// after cudaDeviceReset, gets the new address) and remembered; inside a
// capture the remembered address is used, so the first call on a device
// must come before any capture on it (MOE_ERR_ARG otherwise).
int static_scratch_ptr(cudaStream_t s, int32_t** out) {
  int dev = 0;
  MOE_CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxStaticDevices) return MOE_ERR_ARG;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  MOE_CK(cudaStreamIsCapturing(s, &cap));
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    MOE_CK(cudaGetSymbolAddress(&p, moe_static_scratch));
    g_static_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  if (g_static_scratch_ptr[dev] == nullptr) return MOE_ERR_ARG;
  *out = g_static_scratch_ptr[dev];
  return MOE_OK;
}
}  // namespace

extern "C" {

int moe_dispatch_static(const moe_config_t* c, const int32_t* topk_idx,
                        const uint8_t* sentinel_mask, const void* x, int32_t* counts,
                        int32_t* kept, int32_t* offsets, int32_t* slot_row, int32_t* row_slot,
                        int32_t* tile_expert, int32_t* stats, void* x_perm, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!topk_idx || !x || !counts || !kept || !offsets || !slot_row || !row_slot ||
      !tile_expert || !stats)
    return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  // scratch: n_blocks x E histogram entries + n_blocks sentinel counts.  Both
  // are written in full by the histogram kernel before anything reads them,
  // so nothing has to start at zero.
  const size_t need = ((size_t)L.n_disp_blocks * c->E + (size_t)L.n_disp_blocks) * sizeof(int32_t);
  if (need > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_ARG;
  int32_t* base = nullptr;
  MOE_TRY(static_scratch_ptr(s, &base));
  return dispatch_impl(c, L, topk_idx, sentinel_mask, x, counts, kept, offsets, slot_row,
                       row_slot, tile_expert, stats, x_perm, base,
                       base + (size_t)L.n_disp_blocks * c->E, s);
}

int moe_aux_loss(const moe_config_t* c, const float* probs, const float* lse,
                 const int32_t* counts, float* losses, void* ws, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!probs || !lse || !counts || !losses || !ws) return MOE_ERR_ARG;
  if (c->seq_len > 0) return MOE_ERR_ARG;   // moe_aux_loss_seq
  const Layout L = layout_of(c);
  float* part = wsp<float>(ws, L.off_aux);
  prof_begin(s);
  MOE_CK((launch_k(aux_partial_kernel, L.n_aux_chunks, 256, 0, s, probs, lse, c->T, c->E, part)));
  MOE_LAUNCHED(s, "aux_partial");
  prof_begin(s);
  MOE_CK((launch_k(aux_final_kernel, 1, 512, 0, s, part, counts, L.n_aux_chunks, c->T, c->E, c->aux_alpha,
                                     c->z_lambda, losses)));
  MOE_LAUNCHED(s, "aux_final");
  return MOE_OK;
}

int moe_aux_stats(const moe_config_t* c, const float* probs, const float* lse, float* sums,
                  void* ws, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!probs || !lse || !sums || !ws || c->seq_len > 0 || c->expert_choice) return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  float* part = wsp<float>(ws, L.off_aux);
  prof_begin(s);
  MOE_CK((launch_k(aux_partial_kernel, L.n_aux_chunks, 256, 0, s, probs, lse, c->T, c->E, part)));
  MOE_LAUNCHED(s, "aux_partial");
  prof_begin(s);
  MOE_CK((launch_k(aux_sums_kernel, 1, 512, 0, s, part, L.n_aux_chunks, c->E, sums)));
  MOE_LAUNCHED(s, "aux_sums");
  return MOE_OK;
}

int moe_aux_loss_global(const moe_config_t* c, const int32_t* counts, const float* sums,
                        float* losses, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!counts || !sums || !losses || c->seq_len > 0 || c->expert_choice) return MOE_ERR_ARG;
  prof_begin(s);
  MOE_CK((launch_k(aux_final_kernel, 1, 512, 0, s, sums, counts, 1, (int)loss_tokens_of(c), c->E,
                   c->aux_alpha, c->z_lambda, losses)));
  MOE_LAUNCHED(s, "aux_final");
  return MOE_OK;
}

int moe_aux_loss_seq(const moe_config_t* c, const float* probs, const float* lse,
                     const int32_t* topk_idx, const int32_t* slot_row, float* losses, void* ws,
                     cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!probs || !lse || !topk_idx || !slot_row || !losses || !ws || c->seq_len <= 0)
    return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  const int norm = c->score_fn == MOE_SOFTMAX ? 0 : 1;
  MOE_TRY(seq_aux_launch(c, L, probs, lse, topk_idx, slot_row, norm, losses, nullptr, ws, s));
  return MOE_OK;
}

int moe_bias_update(const moe_config_t* c, const int32_t* counts, float* sel_bias, float gamma,
                    cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!counts || !sel_bias || !(gamma == gamma)) return MOE_ERR_ARG;
  prof_begin(s);
  MOE_CK((launch_k(bias_update_kernel, 1, 256, 0, s, counts, c->E, gamma, sel_bias)));
  MOE_LAUNCHED(s, "bias_update");
  return MOE_OK;
}

}  // extern "C"

namespace {
// gate/up + SwiGLU and down on the tensor cores.  The gate/up A rows are
// read from x_perm, or, with x_perm == nullptr, gathered from the token rows
// of x by the GEMM itself (row_slot, offsets[E] for the shared group).
// With y != nullptr (one slot per token, no shared expert) the down GEMM
// also writes the combined output y[t] = g_t o[row(t)] from its epilogue.
int expert_ffn_tc(const moe_config_t* c, const Layout& L, const void* x_perm, const void* x,
                  const int32_t* row_slot, const int32_t* offsets, const int32_t* tile_expert,
                  const int32_t* stats, const void* w13, const void* w_down, const void* w13_s,
                  const void* w_down_s, void* a13, void* h, void* o, cudaStream_t s,
                  const int32_t* slot_row = nullptr, const float* topk_w = nullptr,
                  void* y = nullptr) {
  const int D = c->D, F = c->F, E = local_E(c);
  const bool gather = x_perm == nullptr;
  CUtensorMap mA, mB, mBs;
  const int64_t mt = row_tiles_estimate(c, L);
  const bool pr = pair_rows(c);                 // CTA-pair row tiles
  const int64_t units = pr ? L.tiles_max / 2 : L.tiles_max;
  // gate/up + SwiGLU: A = x_perm [rows, D] (or rows of x [T, D] copied by
  // the GEMM's producer warp: mapA unused); B = w13 [E, 2F, D] K-major
  // (512-wide tiles load their rows by TMA box only: not with the gather)
  const int bn1 = pick_bn(2 * F, mt, true, F, pr, gather ? 0 : D / 64);
  MOE_TRY(make_map(&mA, gather ? x : x_perm, 1, gather ? c->T : L.rows_max, D, 128, false));
  // B boxes: the gate / up rows of one MMA block (at most 128 per CTA)
  const uint32_t box1 = (uint32_t)std::min(bn1 / 2, 128);
  MOE_TRY(make_map(&mB, w13, E, 2 * F, D, box1, true));
  MOE_TRY(make_map(&mBs, c->n_shared ? w13_s : w13, 1, 2 * F, D, box1, true));
  tc::Params p = rows_params(c, D, F / (bn1 / 2), tile_expert, stats, pr);
  p.out = static_cast<__nv_bfloat16*>(a13); p.ld_out = 2 * F;
  p.out2 = static_cast<__nv_bfloat16*>(h); p.ld_out2 = F;
  p.offsets = offsets; p.row_slot = row_slot; p.gK = c->K;
  p.shared_T = c->n_shared ? c->T : 0;
  p.gx = static_cast<const __nv_bfloat16*>(x);
  const char* n1 = "tc_gate_up_swiglu";
  const int64_t tot1 = units * p.nN;
  OutMaps om1;   // a13 and h as TMA-store targets
  MOE_TRY(make_store_map(&om1.o1, a13, L.rows_max, 2 * F));
  MOE_TRY(make_store_map(&om1.o2, h, L.rows_max, F));
  if (pr && gather)
    MOE_TRY((run_tc<tc::MODE_ROWS, false, false, tc::EPI_SWIGLU, true, true>(bn1, n1, mA, mB, mBs, p, tot1, 0, s, &om1)));
  else if (pr)
    MOE_TRY((run_tc<tc::MODE_ROWS, false, false, tc::EPI_SWIGLU, true>(bn1, n1, mA, mB, mBs, p, tot1, 0, s, &om1)));
  else if (gather)
    MOE_TRY((run_tc<tc::MODE_ROWS, false, false, tc::EPI_SWIGLU, false, true>(bn1, n1, mA, mB, mBs, p, tot1, 0, s, &om1)));
  else
    MOE_TRY((run_tc<tc::MODE_ROWS, false, false, tc::EPI_SWIGLU>(bn1, n1, mA, mB, mBs, p, tot1, 0, s, &om1)));
  // down: A = h [rows, F]; B = w_down [E, D, F] K-major (a pair CTA loads
  // half of the BN rows)
  const int bn2 = pick_bn(D, mt, false, F, pr, F / 64);
  const uint32_t box2 = pr ? (uint32_t)std::min(bn2 / 2, 128) : (uint32_t)bn2;
  MOE_TRY(make_map(&mA, h, 1, L.rows_max, F, 128, false));
  MOE_TRY(make_map(&mB, w_down, E, D, F, box2, true));
  MOE_TRY(make_map(&mBs, c->n_shared ? w_down_s : w_down, 1, D, F, box2, true));
  tc::Params q = rows_params(c, F, D / bn2, tile_expert, stats, pr);
  q.out = static_cast<__nv_bfloat16*>(o); q.ld_out = D;
  if (y != nullptr) {
    q.row_slot = row_slot; q.slot_row = slot_row; q.tw = topk_w;
    q.tout = static_cast<__nv_bfloat16*>(y);
    const char* n2 = "tc_down_combine";
    if (pr)
      return run_tc<tc::MODE_ROWS, false, false, tc::EPI_COMBINE1, true>(
          bn2, n2, mA, mB, mBs, q, units * q.nN, 0, s);
    return run_tc<tc::MODE_ROWS, false, false, tc::EPI_COMBINE1>(
        bn2, n2, mA, mB, mBs, q, units * q.nN, 0, s);
  }
  OutMaps om2;   // o as TMA-store target
  MOE_TRY(make_store_map(&om2.o1, o, L.rows_max, D));
  om2.o2 = om2.o1;
  if (pr)
    return run_tc<tc::MODE_ROWS, false, false, tc::EPI_STORE, true>(
        bn2, "tc_down", mA, mB, mBs, q, units * q.nN, 0, s, &om2);
  return run_tc<tc::MODE_ROWS, false, false, tc::EPI_STORE>(
      bn2, "tc_down", mA, mB, mBs, q, units * q.nN, 0, s, &om2);
}

// One slot per token and no shared expert: the combine and the
// unpermute-sum are row scatters, done in the down / dgrad gate-up GEMM
// epilogues (bf16 tensor-core layers; dx only with the CUDA-core router
// term, E < 8).
bool token_epilogues(const moe_config_t* c) {
  return use_tc(c) && c->K == 1 && c->n_shared == 0 && !c->expert_choice;
}
}  // namespace

extern "C" {

int moe_expert_ffn(const moe_config_t* c, const void* x_perm, const int32_t* offsets,
                   const int32_t* tile_expert, const int32_t* stats, const void* w13,
                   const void* w_down, const void* w13_s, const void* w_down_s, void* a13,
                   void* h, void* o, void* ws, cudaStream_t s) {
  (void)ws;
  MOE_TRY(validate(c));
  if (!x_perm || !tile_expert || !stats || !w13 || !w_down || !a13 || !h || !o)
    return MOE_ERR_ARG;
  if (c->n_shared && (!w13_s || !w_down_s)) return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  const int D = c->D, F = c->F;
  if (use_tc(c))
    return expert_ffn_tc(c, L, x_perm, nullptr, nullptr, offsets, tile_expert, stats, w13,
                         w_down, w13_s, w_down_s, a13, h, o, s);
  auto go = [&](auto tag) -> int {
    using TE = decltype(tag);
    MOE_TRY(simt_rows<TE>(c, L, x_perm, D, w13, D, 1, (int64_t)2 * F * D, w13_s, a13, 2 * F,
                          2 * F, D, tile_expert, stats, s));
    prof_begin(s);
    MOE_CK((launch_k(swiglu_fwd_kernel<TE>, num_sms() * 8, 256, 0, s, static_cast<const TE*>(a13),
                                                         static_cast<TE*>(h), stats, F)));
    MOE_LAUNCHED(s, "swiglu_fwd");
    return simt_rows<TE>(c, L, h, F, w_down, F, 1, (int64_t)D * F, w_down_s, o, D, D, F,
                         tile_expert, stats, s);
  };
  if (c->dtype == MOE_BF16) return go(__nv_bfloat16{});
  return go(float{});
}

int moe_expert_ffn_gather(const moe_config_t* c, const void* x, const int32_t* row_slot,
                          const int32_t* offsets, const int32_t* tile_expert,
                          const int32_t* stats, const void* w13, const void* w_down,
                          const void* w13_s, const void* w_down_s, void* a13, void* h, void* o,
                          void* ws, cudaStream_t s) {
  (void)ws;
  MOE_TRY(validate(c));
  if (!use_tc(c)) return MOE_ERR_ARG;   // the gather rides on the tensor-core GEMM
  if (!x || !row_slot || !offsets || !tile_expert || !stats || !w13 || !w_down || !a13 || !h ||
      !o)
    return MOE_ERR_ARG;
  if (c->n_shared && (!w13_s || !w_down_s)) return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  return expert_ffn_tc(c, L, nullptr, x, row_slot, offsets, tile_expert, stats, w13, w_down,
                       w13_s, w_down_s, a13, h, o, s);
}

int moe_expert_ffn_combine(const moe_config_t* c, const void* x, const void* x_perm,
                           const int32_t* offsets, const int32_t* slot_row,
                           const int32_t* row_slot, const float* topk_w,
                           const int32_t* tile_expert, const int32_t* stats, const void* w13,
                           const void* w_down, const void* w13_s, const void* w_down_s,
                           void* a13, void* h, void* o, void* y, void* ws, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!offsets || !slot_row || !row_slot || !topk_w || !tile_expert || !stats || !w13 ||
      !w_down || !a13 || !h || !o || !y)
    return MOE_ERR_ARG;
  if (!x_perm && (!x || !use_tc(c))) return MOE_ERR_ARG;
  if (c->n_shared && (!w13_s || !w_down_s)) return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  if (token_epilogues(c))
    return expert_ffn_tc(c, L, x_perm, x, row_slot, offsets, tile_expert, stats, w13, w_down,
                         w13_s, w_down_s, a13, h, o, s, slot_row, topk_w, y);
  if (x_perm)
    MOE_TRY(moe_expert_ffn(c, x_perm, offsets, tile_expert, stats, w13, w_down, w13_s, w_down_s,
                           a13, h, o, ws, s));
  else
    MOE_TRY(moe_expert_ffn_gather(c, x, row_slot, offsets, tile_expert, stats, w13, w_down,
                                  w13_s, w_down_s, a13, h, o, ws, s));
  return moe_combine(c, o, slot_row, topk_w, offsets, y, s);
}

int moe_combine(const moe_config_t* c, const void* o, const int32_t* slot_row,
                const float* topk_w, const int32_t* offsets, void* y, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!o || !slot_row || !topk_w || !offsets || !y) return MOE_ERR_ARG;
  const int grid = grid_for(c->T);
  if (c->expert_choice) {
    prof_begin(s);
    if (c->dtype == MOE_BF16)
      MOE_CK((launch_k(ec_combine_kernel<__nv_bfloat16>, grid, 256, 0, s,
                       static_cast<const __nv_bfloat16*>(o), slot_row, topk_w, offsets,
                       c->n_shared, c->T, c->D, c->E, static_cast<__nv_bfloat16*>(y))));
    else
      MOE_CK((launch_k(ec_combine_kernel<float>, grid, 256, 0, s, static_cast<const float*>(o),
                       slot_row, topk_w, offsets, c->n_shared, c->T, c->D, c->E,
                       static_cast<float*>(y))));
    MOE_LAUNCHED(s, "combine");
    return MOE_OK;
  }
  if (c->dtype == MOE_BF16 && (c->K == 1 || c->K == 2 || c->K == 4 || c->K == 8)) {
    auto go = [&](auto kt) -> int {
      prof_begin(s);
      constexpr int KT = decltype(kt)::value;
      auto kern = [] {
        if constexpr (KT <= 2) return combine_bf16_wide_kernel<KT>;
        else return combine_bf16_kernel<KT>;
      }();
      MOE_CK((launch_k(kern, grid, 256, 0, s,
                       static_cast<const __nv_bfloat16*>(o), slot_row, topk_w, offsets,
                       c->n_shared, c->T, c->D, local_E(c), static_cast<__nv_bfloat16*>(y))));
      MOE_LAUNCHED(s, "combine");
      return MOE_OK;
    };
    if (c->K == 1) return go(std::integral_constant<int, 1>{});
    if (c->K == 2) return go(std::integral_constant<int, 2>{});
    if (c->K == 4) return go(std::integral_constant<int, 4>{});
    return go(std::integral_constant<int, 8>{});
  }
  prof_begin(s);
  if (c->dtype == MOE_BF16)
    MOE_CK((launch_k(combine_kernel<__nv_bfloat16>, grid, 256, 0, s,
        static_cast<const __nv_bfloat16*>(o), slot_row, topk_w, offsets, c->n_shared, c->T,
        c->D, c->K, local_E(c), static_cast<__nv_bfloat16*>(y))));
  else
    MOE_CK((launch_k(combine_kernel<float>, grid, 256, 0, s, static_cast<const float*>(o), slot_row, topk_w,
                                               offsets, c->n_shared, c->T, c->D, c->K, local_E(c),
                                               static_cast<float*>(y))));
  MOE_LAUNCHED(s, "combine");
  return MOE_OK;
}

int moe_backward(const moe_config_t* c, const void* x, const float* w_r, const float* logits,
                 const float* probs, const float* lse, const int32_t* topk_idx,
                 const float* topk_w, const int32_t* counts, const int32_t* kept,
                 const int32_t* offsets, const int32_t* slot_row, const int32_t* row_slot,
                 const int32_t* tile_expert, const int32_t* stats, const void* x_perm,
                 const void* a13, const void* h, const void* o, const void* w13,
                 const void* w_down, const void* w13_s, const void* w_down_s, const void* dy,
                 void* dx, float* dw_r, void* dw13, void* dw_down, void* dw13_s,
                 void* dw_down_s, float* dg_out, float* dlogits_out, void* ws, cudaStream_t s) {
  MOE_TRY(validate(c));
  if (!x || !w_r || !logits || !probs || !lse || !topk_idx || !topk_w || !counts || !kept ||
      !offsets || !slot_row || !row_slot || !tile_expert || !stats || !a13 || !h ||
      !o || !w13 || !w_down || !dy || !dx || !dw_r || !dw13 || !dw_down || !ws)
    return MOE_ERR_ARG;
  if (misaligned16(x) || misaligned16(w_r)) return MOE_ERR_ARG;
  if (!x_perm && !use_tc(c)) return MOE_ERR_ARG;   // only the tensor-core wgrad gathers
  if (c->n_shared && (!w13_s || !w_down_s || !dw13_s || !dw_down_s)) return MOE_ERR_ARG;
  const Layout L = layout_of(c);
  const int D = c->D, F = c->F, E = c->E, T = c->T, K = c->K;
  const int El = local_E(c);   // routed experts of the expert GEMMs (E unless sharded)
  float* dg = wsp<float>(ws, L.off_dg);
  float* ds = wsp<float>(ws, L.off_ds);
  float* dwr_part = wsp<float>(ws, L.off_dwr);
  void* dO = wsp<void>(ws, L.off_dO);
  void* dA13 = wsp<void>(ws, L.off_dA13);
  void* dXp = wsp<void>(ws, L.off_dX);
  void* dH = wsp<void>(ws, L.off_dH);
  const bool bf = c->dtype == MOE_BF16;
  // the router's backward products (dW_r, the router part of dx) on tensor
  // cores from E >= 8 (measured faster than the CUDA-core forms at E = 8)
  const bool rtc = router_tc(c);
  const bool dx1 = token_epilogues(c) && !rtc;   // dx from the dgrad gate/up epilogue
  // the router part of dx from the tensor-core product (fp32 R [T, D], then
  // a gather-sum) unless E <= 8 with bf16 token choice: there the
  // unpermute-sum kernel forms ds . W_r itself in fp32 (8 FMAs per element)
  // and the [T, D] fp32 round trip disappears
  const bool dx_tc = router_dx_tc(c);
  const bool dw_tc = router_dw_tc(c);

  // 1. per row: gate gradient dg = <o, dy>, and dO = g * dy (token order:
  // each token's dy row read once for all its slots)
  if (bf && !c->expert_choice && (K == 1 || K == 2 || K == 4 || K == 8)) {
    auto go = [&](auto kt) -> int {
      constexpr int KT = decltype(kt)::value;
      prof_begin(s);
      MOE_CK((launch_k(bwd_tok_kernel<KT>, grid_for(T), 256, 0, s,
                       static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dy),
                       topk_w, slot_row, row_slot, offsets, stats, c->n_shared, El, T, D, dg,
                       static_cast<__nv_bfloat16*>(dO))));
      MOE_LAUNCHED(s, "bwd_gate_grad_rows");
      return MOE_OK;
    };
    if (K == 1) MOE_TRY(go(std::integral_constant<int, 1>{}));
    else if (K == 2) MOE_TRY(go(std::integral_constant<int, 2>{}));
    else if (K == 4) MOE_TRY(go(std::integral_constant<int, 4>{}));
    else MOE_TRY(go(std::integral_constant<int, 8>{}));
  } else {
    const int grid = grid_for(L.rows_max);
    prof_begin(s);
    if (bf)
      MOE_CK((launch_k(bwd_rows_kernel<__nv_bfloat16>, grid, 256, 0, s,
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dy), topk_w,
          row_slot, offsets, stats, K, El, T, D, dg, static_cast<__nv_bfloat16*>(dO))));
    else
      MOE_CK((launch_k(bwd_rows_kernel<float>, grid, 256, 0, s,
          static_cast<const float*>(o), static_cast<const float*>(dy), topk_w, row_slot, offsets,
          stats, K, El, T, D, dg, static_cast<float*>(dO))));
    MOE_LAUNCHED(s, "bwd_gate_grad_rows");
  }
  // The router gradient chain (2, 7) runs on side stream r, concurrently
  // with the expert GEMMs (3-6).  The weight-gradient GEMMs run on side
  // streams: w1 (dW_down, which needs only dO and h) from here on, w2
  // (dW13) once the SwiGLU-backward GEMM is done.  The dx kernel (8) waits
  // only for ds; every side stream joins back into s before returning.
  // With large expert GEMMs everything runs in order on s instead: two
  // persistent GEMMs at once only share the SMs and stretch each other's
  // last wave (measured 2-4% slower per step on the Mixtral- and
  // DeepSeek-shaped layers, whose weight-gradient GEMMs are 4-12 TFLOP;
  // 1.3% faster on the OLMoE shape at 1 TFLOP).
  Side* sd = nullptr;
  MOE_TRY(side_streams(&sd));
  cudaStream_t r = sd->st[0], w1 = sd->st[1], w2 = sd->st[2];
  if (g_caller_side != nullptr) {
    r = g_caller_side[0]; w1 = g_caller_side[1]; w2 = g_caller_side[2];
  }
  const double wgrad_flops =
      use_tc(c) ? 4.0 * (double)row_tiles_estimate(c, L) * kRowTile * c->F * c->D : 0.0;
  if (!g_side_enabled || wgrad_flops >= 2e12) r = w1 = w2 = s;
  MOE_TRY(fork_join(sd->ev[0], s, r));
  if (use_tc(c)) MOE_TRY(fork_join(sd->ev[1], s, w1));
  // 2. router backward: dlogits
  {
    RouterBwdArgs a{T, E, K, c->score_fn, c->renorm, c->route_scale, c->aux_alpha, c->z_lambda,
                    logits, probs, lse, topk_idx, topk_w, slot_row, dg, counts, ds, dlogits_out,
                    dg_out, 0, nullptr, nullptr, nullptr, 0, (float)loss_tokens_of(c)};
    if (c->seq_len > 0 && c->aux_alpha != 0.f) {
      // per-sequence f for the sequence-wise aux gradient
      a.seq_len = c->seq_len;
      a.seq_f = wsp<float>(ws, L.off_seqf);
      MOE_TRY(seq_aux_launch(c, L, probs, lse, topk_idx, slot_row,
                             c->score_fn == MOE_SOFTMAX ? 0 : 1, nullptr,
                             wsp<float>(ws, L.off_seqf), ws, r));
    }
    if (dw_tc) {
      a.dsf = wsp<__nv_bfloat16>(ws, L.off_dsf);
      a.dsb = dx_tc ? wsp<__nv_bfloat16>(ws, L.off_dsb) : nullptr;
      a.Ep = (int)L.Ep;
    }
    const int grid = grid_for(T);
    {
    cudaStream_t s = r;
    if (c->expert_choice) {
      // dp = dg on the picked pairs, then the softmax backward
      auto go = [&](auto nv) -> int {
        prof_begin(s);
        MOE_CK((launch_k(ec_router_bwd_kernel<decltype(nv)::value>, grid, 256, 0, s, probs,
                         logits, lse, slot_row, dg, T, E, c->z_lambda, ds, dlogits_out, dg_out,
                         a.dsf, a.dsb, a.Ep)));
        MOE_LAUNCHED(s, "router_bwd");
        return MOE_OK;
      };
      if (E <= 32) MOE_TRY(go(std::integral_constant<int, 1>{}));
      else if (E <= 64) MOE_TRY(go(std::integral_constant<int, 2>{}));
      else if (E <= 128) MOE_TRY(go(std::integral_constant<int, 4>{}));
      else if (E <= 256) MOE_TRY(go(std::integral_constant<int, 8>{}));
      else MOE_TRY(go(std::integral_constant<int, 16>{}));
    } else {
    prof_begin(s);
    if (E <= 32) MOE_CK((launch_k(router_bwd_kernel<1>, grid, 256, 0, s, a)));
    else if (E <= 64) MOE_CK((launch_k(router_bwd_kernel<2>, grid, 256, 0, s, a)));
    else if (E <= 128) MOE_CK((launch_k(router_bwd_kernel<4>, grid, 256, 0, s, a)));
    else if (E <= 256) MOE_CK((launch_k(router_bwd_kernel<8>, grid, 256, 0, s, a)));
    else MOE_CK((launch_k(router_bwd_kernel<16>, grid, 256, 0, s, a)));
    MOE_LAUNCHED(s, "router_bwd");
    }
    if (dx_tc) {
      // (hi; mid; hi) split of W_r for the router part of dx
      prof_begin(s);
      MOE_CK((launch_k(split_w_kernel, grid_for(L.Ep * D / 256), 256, 0, s, w_r, E, (int)L.Ep, D,
                       (__nv_bfloat16*)nullptr, wsp<__nv_bfloat16>(ws, L.off_wb))));
      MOE_LAUNCHED(s, "router_split_w");
    }
    MOE_CK(cudaEventRecord(sd->ev[6], r));   // ds (and its splits) ready
    }
  }
  // 3-6. expert GEMMs
  if (use_tc(c)) {
    CUtensorMap mA, mB, mBs;
    const int64_t mt = row_tiles_estimate(c, L);
    const int groups = El + c->n_shared;
    const bool pr = pair_rows(c);                 // CTA-pair row tiles
    const int64_t units = pr ? L.tiles_max / 2 : L.tiles_max;
    // 3. dgrad down + SwiGLU backward: dA13 = swiglu'(dO . w_down[e])
    // (BN = 512 leaves this epilogue -- a13 read, dA13 written -- unoverlapped:
    // measured slower than BN = 256 on the Mixtral-shaped layer)
    const int bn3 = pick_bn(F, mt, false, F, pr, 0);
    // k blocks of an average weight-gradient tile (the group's rows)
    const int64_t wg_kb = ceil_div(row_tiles_estimate(c, L) * kRowTile, (int64_t)groups * 64);
    MOE_TRY(make_map(&mA, dO, 1, L.rows_max, D, 128, false));
    MOE_TRY(make_map(&mB, w_down, El, D, F, 64, true));                // dims {F, D, El}
    MOE_TRY(make_map(&mBs, c->n_shared ? w_down_s : w_down, 1, D, F, 64, true));
    {
      tc::Params p = rows_params(c, D, F / bn3, tile_expert, stats, pr);
      p.out = static_cast<__nv_bfloat16*>(dA13); p.ld_out = 2 * F;
      p.aux = static_cast<const __nv_bfloat16*>(a13); p.ld_aux = 2 * F;
      OutMaps om3;   // the saved a13 (TMA loads) and dA13 (TMA stores)
      MOE_TRY(make_store_map(&om3.o1, a13, L.rows_max, 2 * F));
      MOE_TRY(make_store_map(&om3.o2, dA13, L.rows_max, 2 * F));
      if (pr)
        MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_SWIGLU_BWD, true>(
            bn3, "tc_dgrad_down_swiglu_bwd", mA, mB, mBs, p, units * p.nN, 0, s, &om3)));
      else
        MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_SWIGLU_BWD>(
            bn3, "tc_dgrad_down_swiglu_bwd", mA, mB, mBs, p, units * p.nN, 0, s, &om3)));
    }
    MOE_TRY(fork_join(sd->ev[2], s, w2));
    // 4. wgrad down: dW_down[e] = dO^T h over the expert's rows (CTA pairs
    // split the 256-row output tiles)
    const bool pw4 = (D % 256) == 0;
    const int bn4 = wgrad_bn(pick_bn(F, (int64_t)groups * (D / 128), false, F, pw4, wg_kb), F, pw4);
    MOE_TRY(make_map(&mA, dO, 1, L.rows_max, D, 64, false));
    MOE_TRY(make_map(&mB, h, 1, L.rows_max, F, 64, false));
    {
      tc::Params p{};
      p.E = El; p.F = F; p.offsets = offsets; p.kept = kept; p.T = T;
      p.n_groups = groups; p.nMo = D / (pw4 ? 256 : 128); p.nNo = F / bn4; p.No = F;
      p.strideCE = (int64_t)D * F;
      p.out = static_cast<__nv_bfloat16*>(dw_down);
      p.out_shared = static_cast<__nv_bfloat16*>(dw_down_s);
      const int total = p.n_groups * p.nMo * p.nNo;
      OutMaps om4;   // dW_down as [El * D, F] and the shared expert's [D, F]
      MOE_TRY(make_store_map(&om4.o1, dw_down, (int64_t)El * D, F));
      if (c->n_shared) MOE_TRY(make_store_map(&om4.o2, dw_down_s, D, F));
      else om4.o2 = om4.o1;
      if (pw4)
        MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD, true>(
            bn4, "tc_wgrad_down", mA, mB, mB, p, total, total, w1, &om4)));
      else
        MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD>(
            bn4, "tc_wgrad_down", mA, mB, mB, p, total, total, w1, &om4)));
    }
    // 5. dgrad gate/up: dX_perm = dA13 . w13[e]; with one slot per token
    // (no shared expert, CUDA-core router term) the epilogue writes dx
    // itself: dx[t] = dX_perm[row(t)] + ds_t . W_r, once ds is ready
    const int bn5 = pick_bn(D, mt, false, F, pr, 2 * F / 64);
    MOE_TRY(make_map(&mA, dA13, 1, L.rows_max, 2 * F, 128, false));
    MOE_TRY(make_map(&mB, w13, El, 2 * F, D, 64, true));                 // dims {D, 2F, El}
    MOE_TRY(make_map(&mBs, c->n_shared ? w13_s : w13, 1, 2 * F, D, 64, true));
    {
      tc::Params p = rows_params(c, 2 * F, D / bn5, tile_expert, stats, pr);
      p.out = static_cast<__nv_bfloat16*>(dXp); p.ld_out = D;
      if (dx1) {
        MOE_CK(cudaStreamWaitEvent(s, sd->ev[6], 0));
        p.row_slot = row_slot; p.slot_row = slot_row; p.tout = static_cast<__nv_bfloat16*>(dx);
        p.ds = ds; p.w_r = w_r; p.Er = E;
        if (pr)
          MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_DX1, true>(
              bn5, "tc_dgrad_gate_up_dx", mA, mB, mBs, p, units * p.nN, 0, s)));
        else
          MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_DX1>(
              bn5, "tc_dgrad_gate_up_dx", mA, mB, mBs, p, units * p.nN, 0, s)));
      } else {
        OutMaps om5;   // dX_perm as TMA-store target
        MOE_TRY(make_store_map(&om5.o1, dXp, L.rows_max, D));
        om5.o2 = om5.o1;
        if (pr)
          MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_STORE, true>(
              bn5, "tc_dgrad_gate_up", mA, mB, mBs, p, units * p.nN, 0, s, &om5)));
        else
          MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_STORE>(
              bn5, "tc_dgrad_gate_up", mA, mB, mBs, p, units * p.nN, 0, s, &om5)));
      }
    }
    // 6. wgrad gate/up: dW13[e] = dA13^T x_perm (x_perm == nullptr: the
    // producer warp copies the B rows from x by row_slot; mapB unused)
    const bool pw6 = ((2 * F) % 256) == 0;
    const bool g6 = x_perm == nullptr;
    const int bn6 =
        wgrad_bn(pick_bn(D, (int64_t)groups * (2 * F / 128), false, F, pw6, g6 ? 0 : wg_kb), D,
                 pw6 && !g6);
    MOE_TRY(make_map(&mA, dA13, 1, L.rows_max, 2 * F, 64, false));
    MOE_TRY(make_map(&mB, g6 ? x : x_perm, 1, g6 ? T : L.rows_max, D, 64, false));
    {
      tc::Params p{};
      p.E = El; p.F = F; p.offsets = offsets; p.kept = kept; p.T = T;
      p.n_groups = groups; p.nMo = 2 * F / (pw6 ? 256 : 128); p.nNo = D / bn6; p.No = D;
      p.strideCE = (int64_t)2 * F * D;
      p.out = static_cast<__nv_bfloat16*>(dw13);
      p.out_shared = static_cast<__nv_bfloat16*>(dw13_s);
      p.row_slot = row_slot; p.gK = K; p.shared_T = c->n_shared ? T : 0;
      p.gx = static_cast<const __nv_bfloat16*>(x);
      const int total = p.n_groups * p.nMo * p.nNo;
      const char* n6 = "tc_wgrad_gate_up";
      OutMaps om6;   // dW13 as [El * 2F, D] and the shared expert's [2F, D]
      MOE_TRY(make_store_map(&om6.o1, dw13, (int64_t)El * 2 * F, D));
      if (c->n_shared) MOE_TRY(make_store_map(&om6.o2, dw13_s, 2 * F, D));
      else om6.o2 = om6.o1;
      if (pw6 && g6)
        MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD, true, true>(
            bn6, n6, mA, mB, mB, p, total, total, w2, &om6)));
      else if (pw6)
        MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD, true>(
            bn6, n6, mA, mB, mB, p, total, total, w2, &om6)));
      else if (g6)
        MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD, false, true>(
            bn6, n6, mA, mB, mB, p, total, total, w2, &om6)));
      else
        MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD>(
            bn6, n6, mA, mB, mB, p, total, total, w2, &om6)));
    }
  } else {
    auto go = [&](auto tag) -> int {
      using TE = decltype(tag);
      // 3. dH = dO . w_down[e]  (B(n=j, k=d) = w_down[e][d][j])
      MOE_TRY(simt_rows<TE>(c, L, dO, D, w_down, 1, F, (int64_t)D * F, w_down_s, dH, F, F, D,
                            tile_expert, stats, s));
      prof_begin(s);
      MOE_CK((launch_k(swiglu_bwd_kernel<TE>, num_sms() * 8, 256, 0, s,
          static_cast<const TE*>(dH), static_cast<const TE*>(a13), static_cast<TE*>(dA13),
          stats, F)));
      MOE_LAUNCHED(s, "swiglu_bwd");
      // 4. dW_down[e] = dO^T h
      MOE_TRY(simt_wgrad<TE>(c, dO, D, h, F, D, F, dw_down, dw_down_s, offsets, kept, s));
      // 5. dX_perm = dA13 . w13[e]  (B(n=d, k=j) = w13[e][j][d])
      MOE_TRY(simt_rows<TE>(c, L, dA13, 2 * F, w13, 1, D, (int64_t)2 * F * D, w13_s, dXp, D, D,
                            2 * F, tile_expert, stats, s));
      // 6. dW13[e] = dA13^T x_perm
      return simt_wgrad<TE>(c, dA13, 2 * F, x_perm, D, 2 * F, D, dw13, dw13_s, offsets, kept, s);
    };
    if (bf) MOE_TRY(go(__nv_bfloat16{}));
    else MOE_TRY(go(float{}));
  }
  // 7. dW_r = ds^T x on the router stream: on tensor cores as
  // (ds_hi | ds_mid | ds_lo)^T x then the sum of the three parts; else two
  // deterministic SIMT stages
  if (dw_tc) {
    cudaStream_t s = r;
    const int64_t n3 = 3 * L.Ep;
    CUtensorMap mA, mB;
    MOE_TRY(make_map(&mA, wsp<__nv_bfloat16>(ws, L.off_dsf), 1, T, n3, 64, false));
    MOE_TRY(make_map(&mB, x, 1, T, D, 64, false));
    const int64_t nmo = ceil_div(n3, kRowTile);
    const int bn = pick_bn(D, nmo, false, 0, false);
    tc::Params p{};
    p.E = 1; p.dense_rows = T; p.T = T;
    p.n_groups = dwr_splits(c); p.dense_split = dwr_split_rows(c);   // token ranges
    p.strideCE = n3 * D;                                            // partial stride
    p.nMo = (int)nmo; p.nNo = D / bn; p.No = D;
    p.m_limit = (int)n3;
    p.out_f32 = wsp<float>(ws, L.off_dwr3); p.ld_f32 = D;
    const int total = p.n_groups * p.nMo * p.nNo;
    MOE_TRY((run_tc<tc::MODE_WGRAD, true, true, tc::EPI_WGRAD_F32>(
        bn, "router_dw_tc", mA, mB, mB, p, total, total, s)));
    prof_begin(s);
    MOE_CK((launch_k(dwr_reduce3_kernel, grid_for((int64_t)E * D / 32), 256, 0, s,
                     wsp<const float>(ws, L.off_dwr3), E, (int)L.Ep, D, dwr_splits(c), dw_r)));
    MOE_LAUNCHED(s, "router_dw_reduce3");
  } else {
    cudaStream_t s = r;
    const int nc = L.n_dwr_chunks;
    prof_begin(s);
    if (E <= 8) {
      dim3 g((unsigned)ceil_div(D, 256), 1, (unsigned)nc);
      if (bf) MOE_CK((launch_k(dwr_partial_kernel<__nv_bfloat16, 8, 256, 2, 4>, g, 256, 0, s,
          ds, static_cast<const __nv_bfloat16*>(x), T, E, D, L.dwr_chunk, dwr_part)));
      else MOE_CK((launch_k(dwr_partial_kernel<float, 8, 256, 2, 4>, g, 256, 0, s,
          ds, static_cast<const float*>(x), T, E, D, L.dwr_chunk, dwr_part)));
    } else {
      dim3 g((unsigned)ceil_div(D, 64), (unsigned)ceil_div(E, 64), (unsigned)nc);
      if (bf) MOE_CK((launch_k(dwr_partial_kernel<__nv_bfloat16, 64, 64, 4, 4>, g, 256, 0, s,
          ds, static_cast<const __nv_bfloat16*>(x), T, E, D, L.dwr_chunk, dwr_part)));
      else MOE_CK((launch_k(dwr_partial_kernel<float, 64, 64, 4, 4>, g, 256, 0, s,
          ds, static_cast<const float*>(x), T, E, D, L.dwr_chunk, dwr_part)));
    }
    MOE_LAUNCHED(s, "router_dw_partial");
    const int64_t n = (int64_t)E * D;
    prof_begin(s);
    MOE_CK((launch_k(dwr_reduce_kernel, (int)std::min<int64_t>(ceil_div(n, 256), num_sms() * 8), 256, 0, s,
        dwr_part, nc, n, dw_r)));
    MOE_LAUNCHED(s, "router_dw_reduce");
  }
  // 8. dx = unpermute-sum(dX_perm) + shared + ds . w_r, once ds is ready
  // (already written by the dgrad gate/up epilogue when dx1);
  // on tensor cores the router part R = (ds_hi | ds_hi | ds_mid) .
  // (W_hi; W_mid; W_hi) is written in fp32 and a gather kernel adds the
  // dX_perm rows
  MOE_CK(cudaStreamWaitEvent(s, sd->ev[6], 0));
  float* Rdx = nullptr;
  if (rtc && c->expert_choice) {
    // expert choice: the router term R on tensor cores, then a ballot-based
    // gather over each token's picked rows
    const int64_t n3 = 3 * L.Ep;
    Rdx = wsp<float>(ws, L.off_rdx);
    CUtensorMap mA, mB;
    MOE_TRY(make_map(&mA, wsp<__nv_bfloat16>(ws, L.off_dsb), 1, T, n3, 128, false));
    MOE_TRY(make_map(&mB, wsp<__nv_bfloat16>(ws, L.off_wb), 1, n3, D, 64, true));
    const int64_t mtiles = ceil_div(T, kRowTile);
    const int bn = pick_bn(D, mtiles, false, 0, false);
    tc::Params p{};
    p.E = 1; p.Kd = (int)n3; p.nN = D / bn; p.group_m = group_rows(n3);
    p.dense_m = T;
    p.out_f32 = Rdx; p.ld_f32 = D;
    OutMaps om;   // R as TMA-store target
    MOE_TRY(make_store_map_f32(&om.o1, Rdx, T, D));
    om.o2 = om.o1;
    MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_F32>(
        bn, "router_dx_tc", mA, mB, mB, p, mtiles * p.nN, 0, s, &om)));
  }
  if (dx1) {
    // done
  } else if (c->expert_choice) {
    prof_begin(s);
    if (bf)
      MOE_CK((launch_k(ec_dx_kernel<__nv_bfloat16>, grid_for(T), 256, 0, s, Rdx, ds, w_r,
                       static_cast<const __nv_bfloat16*>(dXp), slot_row, offsets, c->n_shared,
                       T, D, E, static_cast<__nv_bfloat16*>(dx))));
    else
      MOE_CK((launch_k(ec_dx_kernel<float>, grid_for(T), 256, 0, s, Rdx, ds, w_r,
                       static_cast<const float*>(dXp), slot_row, offsets, c->n_shared, T, D, E,
                       static_cast<float*>(dx))));
    MOE_LAUNCHED(s, "dx_unpermute_sum");
  } else if (dx_tc) {
    const int64_t n3 = 3 * L.Ep;
    float* R = wsp<float>(ws, L.off_rdx);
    CUtensorMap mA, mB;
    MOE_TRY(make_map(&mA, wsp<__nv_bfloat16>(ws, L.off_dsb), 1, T, n3, 128, false));
    MOE_TRY(make_map(&mB, wsp<__nv_bfloat16>(ws, L.off_wb), 1, n3, D, 64, true));  // {D, 3Ep, 1}
    const int64_t mtiles = ceil_div(T, kRowTile);
    const int bn = pick_bn(D, mtiles, false, 0, false);
    tc::Params p{};
    p.E = 1; p.Kd = (int)n3; p.nN = D / bn; p.group_m = group_rows(n3);
    p.dense_m = T;
    p.out_f32 = R; p.ld_f32 = D;
    OutMaps om;   // R as TMA-store target
    MOE_TRY(make_store_map_f32(&om.o1, R, T, D));
    om.o2 = om.o1;
    MOE_TRY((run_tc<tc::MODE_ROWS, false, true, tc::EPI_F32>(
        bn, "router_dx_tc", mA, mB, mB, p, mtiles * p.nN, 0, s, &om)));
    auto go = [&](auto kt) -> int {
      prof_begin(s);
      MOE_CK((launch_k(dx_sum_kernel<decltype(kt)::value>, grid_for(T), 256, 0, s, R,
                       static_cast<const __nv_bfloat16*>(dXp), slot_row, offsets, c->n_shared,
                       T, D, El, K, static_cast<__nv_bfloat16*>(dx))));
      MOE_LAUNCHED(s, "dx_unpermute_sum");
      return MOE_OK;
    };
    if (K == 1) MOE_TRY(go(std::integral_constant<int, 1>{}));
    else if (K == 2) MOE_TRY(go(std::integral_constant<int, 2>{}));
    else if (K == 4) MOE_TRY(go(std::integral_constant<int, 4>{}));
    else if (K == 8) MOE_TRY(go(std::integral_constant<int, 8>{}));
    else MOE_TRY(go(std::integral_constant<int, 0>{}));
  } else if (bf && E <= 8 && (K == 1 || K == 2 || K == 4 || K == 8)) {
    // blocks (16 slices of 256 columns, token group g), one per SM (each
    // holds a ring of cp.async stages per warp in shared memory)
    const int nch = (int)ceil_div(ceil_div(D, 256), 16);
    const int groups = (int)std::max<int64_t>(1, std::min<int64_t>(T, num_sms() / nch));
    auto go = [&](auto kt) -> int {
      constexpr int KT = decltype(kt)::value;
      constexpr int sm = DxRing<KT>::kBytes;
      MOE_CK(cudaFuncSetAttribute(dx_small_kernel<KT>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, sm));
      prof_begin(s);
      MOE_CK((launch_k(dx_small_kernel<KT>, dim3((unsigned)nch, (unsigned)groups), 512, sm, s, ds,
                       w_r, static_cast<const __nv_bfloat16*>(dXp), slot_row, offsets,
                       c->n_shared, T, D, E, El, static_cast<__nv_bfloat16*>(dx))));
      MOE_LAUNCHED(s, "dx_unpermute_router");
      return MOE_OK;
    };
    if (K == 1) MOE_TRY(go(std::integral_constant<int, 1>{}));
    else if (K == 2) MOE_TRY(go(std::integral_constant<int, 2>{}));
    else if (K == 4) MOE_TRY(go(std::integral_constant<int, 4>{}));
    else MOE_TRY(go(std::integral_constant<int, 8>{}));
  } else {
    dim3 g((unsigned)ceil_div(T, 64), (unsigned)ceil_div(D, 128));
    prof_begin(s);
    if (bf)
      MOE_CK((launch_k(dx_kernel<__nv_bfloat16>, g, 256, 0, s, ds, w_r, static_cast<const __nv_bfloat16*>(dXp),
                                                 slot_row, offsets, c->n_shared, T, D, E, K,
                                                 static_cast<__nv_bfloat16*>(dx))));
    else
      MOE_CK((launch_k(dx_kernel<float>, g, 256, 0, s, ds, w_r, static_cast<const float*>(dXp), slot_row,
                                         offsets, c->n_shared, T, D, E, K,
                                         static_cast<float*>(dx))));
    MOE_LAUNCHED(s, "dx_unpermute_router");
  }
  // join the router chain and the weight-gradient streams (the latter are
  // no-ops on the SIMT path)
  MOE_TRY(fork_join(sd->ev[3], r, s));
  MOE_TRY(fork_join(sd->ev[4], w1, s));
  MOE_TRY(fork_join(sd->ev[5], w2, s));
  return MOE_OK;
}

int moe_check_status(cudaStream_t s, uint32_t* bits) {
  MOE_CK(cudaStreamSynchronize(s));
  unsigned v = 0, zero = 0;
  MOE_CK(cudaMemcpyFromSymbol(&v, moe::g_dev_error, sizeof(v)));
  MOE_CK(cudaMemcpyToSymbol(moe::g_dev_error, &zero, sizeof(zero)));
  if (bits) *bits = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

const char* moe_status_string(int st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument or unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA error (see moe_last_cuda_error)";
    case MOE_ERR_DEVICE: return "device error word set (bad expert id, timeout or row overflow)";
    case MOE_ERR_TIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
  }
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

int moe_set_backward_streams(const cudaStream_t* streams) {
  if (streams == nullptr) {
    g_caller_side = nullptr;
    return MOE_OK;
  }
  for (int i = 0; i < 3; ++i) g_caller_side_st[i] = streams[i];
  g_caller_side = g_caller_side_st;
  return MOE_OK;
}

int moe_set_side_streams(int enable) {
  const int prev = g_side_enabled ? 1 : 0;
  g_side_enabled = enable != 0;
  return prev;
}

int moe_profile_enable(int max_launches) {
  if (max_launches < 1 || max_launches > kProfMax) return MOE_ERR_ARG;
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  g_prof.cap = 0;
  g_prof.n = 0;
  for (int i = 0; i < 2 * max_launches; ++i) MOE_CK(cudaEventCreate(&g_prof.ev[i]));
  g_prof.cap = max_launches;
  return MOE_OK;
}

int moe_profile_reset(void) {
  g_prof.n = 0;
  return MOE_OK;
}

int moe_profile_read(float* ms, int max) {
  if (ms == nullptr) return MOE_ERR_ARG;
  const int n = std::min(g_prof.n, max);
  for (int i = 0; i < n; ++i)
    MOE_CK(cudaEventElapsedTime(&ms[i], g_prof.ev[2 * i], g_prof.ev[2 * i + 1]));
  return n;
}

int moe_profile_starts(float* ms, int max) {
  if (ms == nullptr) return MOE_ERR_ARG;
  const int n = std::min(g_prof.n, max);
  for (int i = 0; i < n; ++i)
    MOE_CK(cudaEventElapsedTime(&ms[i], g_prof.ev[0], g_prof.ev[2 * i]));
  return n;
}

const char* moe_profile_name(int i) {
  return (i >= 0 && i < g_prof.n) ? g_prof.name[i] : "";
}

int moe_profile_side(int i) {
  return (i >= 0 && i < g_prof.n) ? g_prof.side[i] : -1;
}

int moe_profile_disable(void) {
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  g_prof.cap = 0;
  g_prof.n = 0;
  return MOE_OK;
}

int64_t moe_launch_count(int reset) {
  const int64_t v = g_launches;
  if (reset) g_launches = 0;
  return v;
}

}  // extern "C"
