/*
 * moe.h — C ABI of the B200 (sm_100a) token-choice MoE layer library
 * (libmoe.so): router, dispatch, expert FFN, combine, aux/z losses and the
 * full backward of one layer on one GPU.
 *
 * Pages this follows (cited by title and section):
 *   [STA324]  "08 MoE：容量、路由、梯度、均衡和系统实现" (STA324 notes), §8.1-§8.9
 *   [TRAIN]   "MoE 训练：稀疏计算背后的路由与通信" (MoE training course page)
 *   [8MOE]    "8-MoE" lecture notes (Router / Gating Network, KeepTopK,
 *             Expert Capacity, GShard, Switch Transformers, ST-MoE,
 *             MoE 高效推理 — token grouping and permutation)
 *   [HF48687] "Wrong router gradient with experts_implementation=batched_mm
 *             under expert parallelism" (transformers issue summary)
 *   [MM858]   "[Bug] num_experts_per_tok=1 时 MoE 路由器收不到梯度" (MiniMind issue)
 *
 * Conventions (all entry points):
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise;
 *     `cfg` is a HOST pointer.  All buffers are owned and allocated by the
 *     caller; the library never allocates or frees memory.
 *   - All layouts are row-major and contiguous.  T tokens, D model dim,
 *     E routed experts, K experts per token, F expert FFN dim.  On the
 *     tensor-core path the kernels read and write activation, expert-weight
 *     and gradient buffers through TMA, so each must start on a 16-byte
 *     boundary (any cudaMalloc'd or torch buffer does); a misaligned one
 *     makes the call return MOE_ERR_CUDA when its tensor map is built
 *     (kernels of that call that come earlier may already have run).  x
 *     and W_r, which every path reads with 16-byte loads, are checked
 *     first: moe_router, moe_route_expert_choice and moe_backward return
 *     MOE_ERR_ARG, having launched nothing, when either is misaligned.
 *     "act" = activation / expert-weight element type, cfg->dtype:
 *     MOE_BF16 (__nv_bfloat16) or MOE_FP32 (float).  The router is fp32.
 *   - Calls are asynchronous on `stream` and never synchronise, except
 *     moe_check_status().  They may issue cudaMemsetAsync on `stream`.
 *   - Return value: MOE_OK (0) or a negative moe_status; on MOE_ERR_ARG
 *     nothing was launched.  Errors detected on the device (an expert id
 *     outside [-1, E), a pipeline wait that timed out) set a device error
 *     word that moe_check_status() reads and clears.
 *   - Permuted row space: routed expert e owns rows
 *     [offsets[e], offsets[e+1]); its kept slots occupy the first kept[e]
 *     rows in flat-slot order, the rest up to the next multiple of
 *     row_align (128, or 256 when the expert GEMMs run on CTA pairs; see
 *     moe_get_sizes) are zero padding.  The shared expert (n_shared = 1) owns rows
 *     [offsets[E], offsets[E+1]) = its T tokens in order, then padding.
 *     Buffers indexed by row are sized rows_max (moe_get_sizes).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = -1,          /* invalid argument / unsupported configuration */
  MOE_ERR_CUDA = -2,         /* a CUDA call or launch failed (moe_last_cuda_error) */
  MOE_ERR_DEVICE = -3,       /* device error word set (see moe_check_status) */
  MOE_ERR_TIMEOUT = -4       /* reserved: a bounded device wait gave up */
} moe_status;

enum { MOE_FP32 = 0, MOE_BF16 = 1 };             /* cfg.dtype */
enum { MOE_SOFTMAX = 0, MOE_SIGMOID = 1 };       /* cfg.score_fn */
enum { MOE_GMAX = 0, MOE_GTOP2SUM = 1 };         /* cfg.group_score */
enum { MOE_GEMM_AUTO = 0, MOE_GEMM_SIMT = 1 };   /* cfg.gemm_impl */

/* Device error word bits (moe_check_status). */
#define MOE_DEVERR_EXPERT_ID  1u   /* an expert id outside [-1, E): slot treated as sentinel */
#define MOE_DEVERR_TIMEOUT    2u   /* a tensor-core pipeline wait gave up */
#define MOE_DEVERR_ROWS       4u   /* permuted rows exceeded rows_max */

/*
 * Layer configuration.
 *   score_fn   MOE_SOFTMAX: p = softmax(s), top-K on s          [STA324 §8.2]
 *              MOE_SIGMOID: p = sigmoid(s), top-K on p + b      [STA324 §8.6]
 *   renorm     0 = variant A (g = p_sel, no renormalisation),
 *              1 = variant B (g = softmax over the selected logits; for
 *                  sigmoid g = p_sel / (sum p_sel + 1e-20))     [STA324 §8.2]
 *   n_groups, topk_groups, group_score
 *              group-limited routing: E splits into n_groups contiguous
 *              groups scored by their max (MOE_GMAX) or the sum of their
 *              two largest (MOE_GTOP2SUM) selection scores; only experts of
 *              the topk_groups best groups are eligible.  1,1 = off.
 *              [STA324 §8.2], [TRAIN] (capacity, dropless and group routing)
 *   capacity_factor, min_capacity
 *              C = max(ceil(c*T*K/E), min_capacity); c <= 0: no limit.
 *              [STA324 §8.5], [8MOE] Expert Capacity
 *   route_scale multiplies g after renormalisation               [TRAIN]
 *   aux_alpha  Switch load-balance loss alpha*E*sum_e f_e P_e
 *              [STA324 §8.5], [TRAIN]; over the whole batch (softmax
 *              scores only) or, with seq_len > 0, per sequence
 *   seq_len    > 0: sequence-wise aux loss, the same loss on each group of
 *              seq_len consecutive tokens, averaged over the groups; with
 *              sigmoid scores P uses the affinities divided by their sum
 *              over experts [STA324 §8.6], [TRAIN] (DeepSeek-V3's
 *              complementary sequence-wise term); seq_len divides T
 *   z_lambda   router z-loss lambda*mean_t lse_t^2           [8MOE] ST-MoE
 *   n_shared   0 or 1: a shared SwiGLU expert on every token, weight 1,
 *              no top-K slot                                 [STA324 §8.7]
 *   expert_choice
 *              1: every expert picks C = min(T, max(ceil(c*T/E),
 *              min_capacity)) tokens, the ones with the largest softmax
 *              probability p[t,e] (equal scores: lower token first); the
 *              gate weight is p[t,e]; a token may be picked by several
 *              experts or none.  [STA324 §8.4]  The layer then runs in the
 *              token-choice layout with one slot per (t, e) pair: K must
 *              equal E, topk_idx[t,e] = e, and the pairs an expert did not
 *              pick are sentinel slots.  Requires softmax, renorm = 0,
 *              capacity_factor > 0, no groups, no aux loss, route_scale 1.
 *   gemm_impl  MOE_GEMM_AUTO: tcgen05 tensor cores for bf16 when D and F
 *              are multiples of 128, CUDA-core SIMT otherwise (fp32 always);
 *              MOE_GEMM_SIMT: force the SIMT kernels (cross-checks).
 *   loss_tokens  0, or the global token count N >= T when the batch aux
 *              loss and the z-loss are scoped over all data-parallel ranks
 *              ([STA324 §8.5]: the balance statistic may be taken over the
 *              whole batch or all devices): the aux gradient then uses the
 *              counts passed to moe_backward (the all-reduced ones) and both
 *              gradients divide by N.  Requires seq_len = 0, expert_choice = 0.
 *   expert_base, n_local_experts
 *              expert parallelism ([HF48687]: under expert parallelism every
 *              rank sees the global routing and the slots of experts it
 *              does not hold are sentinels, whose expert output is zero;
 *              [8MOE] DeepSpeed / [TRAIN] all-to-all flow).  With
 *              n_local_experts = El > 0 this call holds routed experts
 *              [expert_base, expert_base + El): moe_router, the aux / z
 *              losses and the router gradient stay over all E experts
 *              (logits, probs [T,E], counts [E]); moe_dispatch gives the
 *              slots of other experts slot_row = -2 (counted in stats[1])
 *              and lays out only the local experts (kept [El], offsets
 *              [El+2], tile_expert values < El, capacity still
 *              ceil(c*T*K/E)); the expert weights and their gradients are
 *              [El, ...].  y, dx, dW_r, dlogits and dg of the shards sum to
 *              those of the whole layer (add the aux / z losses on one shard
 *              only).  Requires the tensor-core path (bf16, D and F
 *              multiples of 128), n_shared = 0, seq_len = 0 and token
 *              choice.
 * Limits: 1 <= K <= min(E, 16) (expert choice: K = E); E <= 512; n_groups <= 32, E % n_groups == 0,
 * topk_groups * (E / n_groups) >= K; D % 8 == 0; F % 8 == 0.
 */
typedef struct {
  int32_t T, D, E, K, F, n_shared;
  int32_t dtype;
  int32_t score_fn, renorm;
  int32_t n_groups, topk_groups, group_score;
  float capacity_factor;
  int32_t min_capacity;
  float route_scale, aux_alpha, z_lambda;
  int32_t gemm_impl;
  int32_t seq_len;      /* 0: batch aux loss; > 0: sequence-wise aux loss over
                           consecutive groups of seq_len tokens (divides T) */
  int32_t expert_choice; /* 0: token choice (top-K per token); 1: expert choice
                            (moe_route_expert_choice) */
  int32_t loss_tokens;   /* tokens the batch aux and z losses average over:
                            0 = T (this call's batch); data-parallel ranks that
                            scope the losses over the global batch set the
                            global token count (>= T) and pass the all-reduced
                            counts (moe_aux_stats, moe_aux_loss_global) */
  int32_t expert_base;     /* expert parallelism: first routed expert this call's */
  int32_t n_local_experts; /* expert FFN holds (0 = all E experts, no sharding) */
} moe_config_t;

typedef struct {
  int64_t rows_max;     /* rows of every permuted-row buffer (multiple of 128) */
  int64_t tiles_max;    /* rows_max / 128 */
  int64_t capacity;     /* C, or -1 when unlimited */
  size_t ws_bytes;      /* workspace needed by any call (256-byte aligned base) */
  int64_t row_align;    /* expert segments start at multiples of this (128 or 256) */
} moe_sizes_t;

/* Buffer sizes for cfg.  Host-only, no CUDA calls. */
int moe_get_sizes(const moe_config_t* cfg, moe_sizes_t* out);

/*
 * moe_router — fp32 router logits, scores, group limit, top-K and gate
 * weights.  [STA324 §8.2, §8.6], [8MOE] Router / Gating Network, KeepTopK,
 * [TRAIN] (TopKRouter flow), [MM858] §2.
 *   x            [T,D] act
 *   w_r          [E,D] f32 router weight (logits s = x w_r^T)
 *   logit_offset [E] f32 or NULL: constant added to the logits
 *   sel_bias     [E] f32 or NULL: selection-only bias (sigmoid scoring)
 *   logits       [T,E] f32 out
 *   probs        [T,E] f32 out: softmax probabilities or sigmoid affinities
 *   lse          [T]   f32 out: logsumexp of the logits
 *   topk_idx     [T,K] i32 out: selected experts, best first; equal
 *                selection scores go to the lower expert index
 *   topk_w       [T,K] f32 out: gate weights g
 *   near_ties    [1] i32 out: tokens where two consecutive selection scores
 *                among the top K+1 (or the kept/next group scores) are
 *                closer than 1e-5: the choice or the slot order of such a
 *                token may differ from an exact computation
 *   ws           workspace (moe_get_sizes)
 */
int moe_router(const moe_config_t* cfg, const void* x, const float* w_r,
               const float* logit_offset, const float* sel_bias,
               float* logits, float* probs, float* lse,
               int32_t* topk_idx, float* topk_w, int32_t* near_ties,
               void* ws, cudaStream_t stream);

/*
 * moe_dispatch — counting-sort permutation with capacity drop and sentinel
 * slots, and the gather of token rows into expert order.
 * [8MOE] MoE 高效推理 (sort tokens by expert, gather), Expert Capacity,
 * GShard drop tokens; [STA324 §8.5, §8.8]; [HF48687] cause analysis.
 *   topk_idx      [T,K] i32: expert per slot; -1 = sentinel (no local expert)
 *   sentinel_mask [T*K] u8 or NULL: nonzero marks a slot as sentinel
 *   x             [T,D] act
 *   counts        [E] i32 out: valid slots per expert before drops
 *   kept          [E] i32 out: min(counts, C)
 *   offsets       [E+2] i32 out: permuted-row offsets (see header)
 *   slot_row      [T*K] i32 out: row of each slot, -1 if dropped, -2 if
 *                 sentinel
 *   row_slot      [rows_max] i32 out: slot of each routed row, -1 otherwise
 *   tile_expert   [tiles_max] i32 out: expert of each 128-row tile (E = shared)
 *   stats         [4] i32 out: n_dropped, n_sentinel, n_rows, n_tiles
 *   x_perm        [rows_max,D] act out: gathered rows, zero padding; NULL:
 *                 layout only (no gather launched), for the fused-gather
 *                 path (moe_expert_ffn_gather, moe_backward with NULL x_perm)
 * Slots of one expert are ranked in flat slot order j = t*K + k; ranks >= C
 * are dropped.
 */
int moe_dispatch(const moe_config_t* cfg, const int32_t* topk_idx,
                 const uint8_t* sentinel_mask, const void* x,
                 int32_t* counts, int32_t* kept, int32_t* offsets,
                 int32_t* slot_row, int32_t* row_slot, int32_t* tile_expert,
                 int32_t* stats, void* x_perm, void* ws, cudaStream_t stream);

/*
 * moe_dispatch_static — moe_dispatch without a workspace (allocates nothing).
 * The pages have no counterpart: this entry point serves callers that are
 * given only their input and output buffers and cannot allocate device
 * memory, such as a plugin or custom-op host with no workspace hook that
 * forbids cudaMalloc inside the op, or a serving runtime whose device memory
 * plan is fixed in advance.  Arguments, outputs and results are those of
 * moe_dispatch, minus `ws`.
 *   - Scratch (per-block expert histograms and sentinel counts) lives in a
 *     file-scope device array of MOE_STATIC_SCRATCH_BYTES that every GPU
 *     loading the library holds until the process exits.  It needs
 *     (ceil(T*K / 4096) * (E + 1)) * 4 bytes; larger problems are rejected
 *     with MOE_ERR_ARG before anything is launched (1 MiB covers, e.g.,
 *     T*K up to about 4.1 M slots at E = 256).
 *   - Each call outside stream capture looks up the array's device address
 *     (cudaGetSymbolAddress, with the calling thread's current device) and
 *     remembers it per device; a call made while `stream` is being captured
 *     uses the remembered address, so make the first call on each device
 *     before any stream capture on it (else MOE_ERR_ARG).
 *   - All calls share the one array and it keeps the last call's contents
 *     (every call rewrites what it reads, nothing must start at zero).
 *     Calls that overlap on the GPU — on different streams, or from
 *     different threads, at the same time — race on it: serialise them.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define MOE_STATIC_SCRATCH_BYTES (1u << 20)
int moe_dispatch_static(const moe_config_t* cfg, const int32_t* topk_idx,
                        const uint8_t* sentinel_mask, const void* x,
                        int32_t* counts, int32_t* kept, int32_t* offsets,
                        int32_t* slot_row, int32_t* row_slot, int32_t* tile_expert,
                        int32_t* stats, void* x_perm, cudaStream_t stream);

/*
 * moe_aux_loss — losses[0] = alpha*E*sum_e f_e P_e with f_e = counts_e /
 * sum(counts), P_e = mean_t probs[t,e]; losses[1] = lambda*mean_t lse_t^2.
 * [STA324 §8.5, §8.6], [TRAIN], [8MOE] ST-MoE.  losses: [2] f32 out.
 * Deterministic (fixed-order reductions).
 */
int moe_aux_loss(const moe_config_t* cfg, const float* probs, const float* lse,
                 const int32_t* counts, float* losses, void* ws,
                 cudaStream_t stream);

/*
 * moe_aux_stats — this batch's share of the load-balance statistics, for
 * aux and z losses scoped over several data-parallel ranks ([STA324 §8.5]:
 * the balance statistic over the whole batch or all devices).
 *   sums [E+1] f32 out: sums[e] = sum_t probs[t,e], sums[E] = sum_t lse_t^2,
 *        each reduced in a fixed order (deterministic)
 * The caller all-reduces (sums) `sums` and the dispatch's `counts` over the
 * ranks (NCCL), then calls moe_aux_loss_global; moe_backward with
 * cfg.loss_tokens = N and the all-reduced counts gives each rank's share of
 * the gradient of the global losses.
 */
int moe_aux_stats(const moe_config_t* cfg, const float* probs, const float* lse,
                  float* sums, void* ws, cudaStream_t stream);

/*
 * moe_aux_loss_global — losses from all-reduced statistics:
 * losses[0] = alpha*E*sum_e (counts_e / sum counts) (sums_e / N),
 * losses[1] = lambda * sums[E] / N, N = cfg.loss_tokens (T if 0).
 * [STA324 §8.5, §8.6], [TRAIN], [8MOE] ST-MoE.  counts [E] i32 and sums
 * [E+1] f32 summed over ranks; with one rank the result equals moe_aux_loss
 * bit for bit.  losses [2] f32 out.
 */
int moe_aux_loss_global(const moe_config_t* cfg, const int32_t* counts, const float* sums,
                        float* losses, cudaStream_t stream);

/*
 * moe_route_expert_choice — router of expert choice (cfg.expert_choice = 1,
 * K = E).  fp32 logits (tensor cores on bf16 splits of w_r, as moe_router),
 * probs = softmax, lse, then each expert's C picks.  [STA324 §8.4]
 *   logits, probs [T,E] f32 out; lse [T] f32 out
 *   topk_idx  [T,E] i32 out: e (slot (t,e) belongs to expert e)
 *   topk_w    [T,E] f32 out: p[t,e]
 *   sentinel_mask [T*E] u8 out: 1 where expert e did not pick token t
 *             (pass it to moe_dispatch)
 *   near_ties [1] i32 out: experts whose C-th and (C+1)-th scores differ by
 *             less than 1e-5
 */
int moe_route_expert_choice(const moe_config_t* cfg, const void* x, const float* w_r,
                            const float* logit_offset, float* logits, float* probs,
                            float* lse, int32_t* topk_idx, float* topk_w,
                            uint8_t* sentinel_mask, int32_t* near_ties, void* ws,
                            cudaStream_t stream);

/*
 * moe_aux_loss_seq — the sequence-wise aux loss (cfg.seq_len > 0):
 * losses[0] = alpha*E*mean_s sum_e f_{s,e} P_{s,e}, f_{s,e} = share of
 * sequence s's valid (non-sentinel, pre-drop) slots that chose e, P_{s,e} =
 * mean over its tokens of probs (softmax) or of probs / sum_e probs
 * (sigmoid affinities); losses[1] as in moe_aux_loss.  [STA324 §8.5, §8.6],
 * [TRAIN].  topk_idx and slot_row from moe_router / moe_dispatch (slot_row
 * -2 marks sentinels).  Deterministic; MOE_ERR_ARG if seq_len == 0.
 */
int moe_aux_loss_seq(const moe_config_t* cfg, const float* probs, const float* lse,
                     const int32_t* topk_idx, const int32_t* slot_row, float* losses,
                     void* ws, cudaStream_t stream);

/*
 * moe_bias_update — the selection-bias load-control step of sigmoid
 * routing: sel_bias[e] -= gamma * sign(counts[e] - mean(counts)) in place
 * (overloaded experts' bias goes down, underloaded ones' up; the sign is
 * taken exactly, on counts[e]*E - sum(counts)).  [STA324 §8.6], [TRAIN]
 * (DeepSeek-V3's dynamic expert bias).  counts from moe_dispatch (valid
 * slots, pre-drop); sel_bias [E] f32 in/out.
 */
int moe_bias_update(const moe_config_t* cfg, const int32_t* counts, float* sel_bias,
                    float gamma, cudaStream_t stream);

/*
 * moe_expert_ffn — grouped SwiGLU experts over the permuted rows.
 * [STA324 §8.1, §8.8] (SwiGLU ~3DF parameters; grouped GEMM over experts).
 *   x_perm   [rows_max,D] act (moe_dispatch)
 *   w13      [E,2F,D] act: rows 0..F-1 gate projection, F..2F-1 up
 *   w_down   [E,D,F]  act
 *   w13_s, w_down_s  [2F,D], [D,F] act: shared expert (NULL if n_shared=0)
 *   a13      [rows_max,2F] act out: pre-activations (saved for backward)
 *   h        [rows_max,F]  act out: silu(a) * b
 *   o        [rows_max,D]  act out: expert outputs h w_down^T
 * Tiles of experts without rows are skipped on the device (no host sync).
 */
int moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                   const int32_t* offsets,
                   const int32_t* tile_expert, const int32_t* stats,
                   const void* w13, const void* w_down,
                   const void* w13_s, const void* w_down_s,
                   void* a13, void* h, void* o, void* ws, cudaStream_t stream);

/*
 * moe_expert_ffn_gather — moe_expert_ffn without the permuted copy of x:
 * the gate/up GEMM's producer warp copies its A rows straight from the
 * token rows of x (16-byte cp.async copies into the swizzled layout a TMA
 * box would produce), so x_perm is never written or read.  Same method, one HBM round trip less: the pages
 * group tokens into contiguous per-expert blocks before the grouped GEMM
 * ([8MOE] MoE 高效推理; [STA324 §8.8]); here the grouping happens inside the
 * GEMM's operand load.
 *   x         [T,D] act: layer input (the tensor moe_dispatch was given)
 *   row_slot  [rows_max] i32 (moe_dispatch): permuted row r holds token
 *             row_slot[r] / K; rows of the shared group hold token
 *             r - offsets[E]; padding rows load as zeros
 *   offsets   [E+2] i32 (moe_dispatch)
 *   the rest as moe_expert_ffn; the outputs are identical to moe_expert_ffn
 *   on the x_perm that moe_dispatch would have written.
 * bf16 layers on the tensor-core path only (MOE_ERR_ARG for fp32 layers or
 * gemm_mode MOE_GEMM_SIMT).
 */
int moe_expert_ffn_gather(const moe_config_t* cfg, const void* x,
                          const int32_t* row_slot, const int32_t* offsets,
                          const int32_t* tile_expert, const int32_t* stats,
                          const void* w13, const void* w_down,
                          const void* w13_s, const void* w_down_s,
                          void* a13, void* h, void* o, void* ws, cudaStream_t stream);

/*
 * moe_expert_ffn_combine — moe_expert_ffn (x_perm != NULL) or
 * moe_expert_ffn_gather (x_perm == NULL) followed by moe_combine, in one
 * call.  With one slot per token (K = 1) and no shared expert on the
 * tensor-core path, the combine y_t = g_t o[slot_row[t]] is a row scatter:
 * the down-projection GEMM's epilogue writes y from its fp32 accumulator
 * (scaled by g, rounded once) next to o, and tokens whose slot holds no
 * row (sentinel, dropped) get y_t = 0 — no combine kernel runs.  Otherwise
 * the separate combine runs.  [8MOE] Router / Gating Network; [STA324
 * §8.7, §8.8].
 *   x, x_perm   as moe_expert_ffn_gather / moe_expert_ffn (x may be NULL
 *               when x_perm is given)
 *   slot_row, row_slot, topk_w, offsets, tile_expert, stats: moe_router /
 *               moe_dispatch outputs
 *   a13, h, o   as moe_expert_ffn;  y [T,D] act out, as moe_combine
 */
int moe_expert_ffn_combine(const moe_config_t* cfg, const void* x, const void* x_perm,
                           const int32_t* offsets, const int32_t* slot_row,
                           const int32_t* row_slot, const float* topk_w,
                           const int32_t* tile_expert, const int32_t* stats,
                           const void* w13, const void* w_down,
                           const void* w13_s, const void* w_down_s,
                           void* a13, void* h, void* o, void* y, void* ws,
                           cudaStream_t stream);

/*
 * moe_combine — y_t = sum_{k kept} g_{t,k} o[slot_row[t*K+k]] (k ascending,
 * fp32 accumulation) + o[offsets[E] + t] when n_shared.  Deterministic
 * gather, no atomics.  [8MOE] Router / Gating Network (y = sum G(x)_i
 * E_i(x)); [STA324 §8.7, §8.8].
 *   y [T,D] act out
 */
int moe_combine(const moe_config_t* cfg, const void* o,
                const int32_t* slot_row, const float* topk_w,
                const int32_t* offsets, void* y, cudaStream_t stream);

/*
 * moe_backward — all gradients of <y, dy> + L_aux + L_z.
 * [STA324 §8.3, §8.5], [MM858] §2-§3, [HF48687] cause analysis.
 * Inputs are the forward's inputs and outputs above, plus
 *   dy        [T,D] act: upstream gradient of y
 * Outputs:
 *   dx        [T,D] act: expert path + shared expert + router path
 *   dw_r      [E,D] f32
 *   dw13      [E,2F,D] act, dw_down [E,D,F] act (expert with no rows: 0)
 *   dw13_s, dw_down_s  shared expert grads (NULL if n_shared = 0)
 *   dg_out    [T,K] f32 or NULL: dL/dg = <o, dy>, 0 on sentinel/dropped
 *   dlogits_out [T,E] f32 or NULL: dL/ds
 * The gate gradient of a sentinel or dropped slot is zero (its expert
 * output is treated as zero), so such slots send no gradient to the router
 * through the gate path.  Deterministic: no floating-point atomics.
 * With one slot per token (K = 1), no shared expert and E < 8 on the
 * tensor-core path, dx is written by the dgrad gate/up GEMM's epilogue
 * (dX_perm row + ds_t . W_r, rounded once; tokens without a row get the
 * router part alone) instead of a separate unpermute-sum.  The router part
 * ds_t . W_r is formed in fp32 on CUDA cores for bf16 token choice with
 * E <= 8, else (E > 8, expert choice) on tensor cores from exact bf16
 * splits of ds and W_r (the three leading terms, fp32 accumulation).
 * x_perm may be NULL on the tensor-core path (bf16 layers): the gate/up
 * weight-gradient GEMM then copies its x rows by row_slot in its producer
 * warp (cp.async), as moe_expert_ffn_gather does (MOE_ERR_ARG for NULL
 * x_perm on the SIMT path).
 * Inside the call, independent chains (the router gradient, the two
 * weight-gradient GEMMs) are forked onto three side streams and joined back
 * into `stream` before the call returns, so the results are ordered on
 * `stream` like any other call.  When each weight-gradient GEMM is 2 TFLOP
 * or more (4·rows·F·D with the expected rows), everything runs in order on
 * `stream` instead: two persistent GEMMs at once only share the SMs.  The
 * fork/join still happens (events recorded on `stream` itself).  The side
 * streams are the caller's when set
 * with moe_set_backward_streams (recommended: one set per layer, so that
 * independent layers' backward passes do not queue behind one another);
 * otherwise the library creates three streams and eight events per host
 * thread and device on first use (make that first call outside stream
 * capture), shared by every call on that thread and device and kept until
 * the process exits — the one resource besides moe_profile_enable's events
 * that the library creates itself (no device memory).  The fork/join
 * events are always the library's (eight per host thread and device).
 * The counts argument feeds only the aux-loss gradient (f = counts/sum).
 */
int moe_backward(const moe_config_t* cfg,
                 const void* x, const float* w_r, const float* logits,
                 const float* probs, const float* lse,
                 const int32_t* topk_idx, const float* topk_w,
                 const int32_t* counts, const int32_t* kept,
                 const int32_t* offsets, const int32_t* slot_row,
                 const int32_t* row_slot, const int32_t* tile_expert,
                 const int32_t* stats,
                 const void* x_perm, const void* a13, const void* h,
                 const void* o,
                 const void* w13, const void* w_down,
                 const void* w13_s, const void* w_down_s,
                 const void* dy,
                 void* dx, float* dw_r, void* dw13, void* dw_down,
                 void* dw13_s, void* dw_down_s,
                 float* dg_out, float* dlogits_out,
                 void* ws, cudaStream_t stream);

/* Synchronises `stream`, reads and clears the device error word (bits in
 * *bits if non-NULL).  MOE_OK, MOE_ERR_DEVICE or MOE_ERR_CUDA. */
int moe_check_status(cudaStream_t stream, uint32_t* bits);

/* Text for a moe_status value (static storage). */
const char* moe_status_string(int status);

/* The cudaError_t behind the last MOE_ERR_CUDA on this thread. */
int moe_last_cuda_error(void);

/* Number of kernel launches issued by this thread since the last reset. */
int64_t moe_launch_count(int reset);

/*
 * Side streams inside moe_backward (default on).  With 0, every kernel of
 * moe_backward runs on the caller's stream in issue order: slower, but
 * each launch then has the GPU to itself (used to time kernels one by one).
 * Applies to later calls from this host thread; returns the previous value.
 */
int moe_set_side_streams(int enable);

/*
 * Caller-owned side streams for moe_backward on this host thread:
 * streams[3] (created by the caller on the device the calls run on, kept
 * alive while set), or NULL to return to the library's own.  Applies to
 * later moe_backward calls from this thread; a layer sets its own streams
 * before each of its backward calls.
 */
int moe_set_backward_streams(const cudaStream_t* streams);

/*
 * Per-launch timing (measurement support; not part of the layer's math).
 * While enabled, every kernel launch of this thread is bracketed by a begin
 * and an end cudaEvent recorded on the launching stream (inside a CUDA
 * graph capture they become event-record nodes, re-recorded on every
 * replay).  Up to max_launches launches (<= 256) are recorded after each
 * moe_profile_reset().
 *   moe_profile_enable  creates the events (the library's only resource
 *                       other than device code; no device memory)
 *   moe_profile_read    after the caller synchronised: writes the elapsed
 *                       milliseconds of each recorded launch to ms (host
 *                       array) and returns how many were written
 *   moe_profile_starts  like moe_profile_read, but writes the start of each
 *                       recorded launch relative to the start of launch 0
 *                       (a timeline of one step; gaps show launch overhead)
 *   moe_profile_name    kernel family name of recorded launch i
 *   moe_profile_side    1 if launch i ran on one of the library's side
 *                       streams (concurrently with other work, so its
 *                       duration includes sharing the GPU), 0 if on the
 *                       caller's stream, -1 if i is out of range
 */
int moe_profile_enable(int max_launches);
int moe_profile_reset(void);
int moe_profile_read(float* ms, int max);
int moe_profile_starts(float* ms, int max);
const char* moe_profile_name(int i);
int moe_profile_side(int i);
int moe_profile_disable(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
