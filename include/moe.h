/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE layer forward library (libmoe.so).
 *
 * The library computes the single-device forward of a token-choice top-k
 * mixture-of-experts layer with SwiGLU experts:
 *
 *   router (fp32 logits, softmax, top-k, optional renormalisation)
 *   -> dispatch of the routed copies into expert-major order
 *   -> [expert-parallel local regroup of a rank-major buffer]
 *   -> grouped SwiGLU  y = (silu(x w1^T) * (x w3^T)) w2^T  per expert segment
 *   -> weighted combine (scatter-add of every copy back to its token).
 *
 * Sources, by page and section:
 *   [HP] hyper_parallel platform/torch/common/moe.py coverage page:
 *        TokenChoiceTopKRouter.forward, MoE.permutation, MoE.unpermutation,
 *        _run_experts_for_loop, _run_experts_grouped_mm_gpu, GroupedExperts,
 *        MoE.forward.
 *   [QO] QwenLM/Qwen3-Omni issue #115: SpeedupMoeExperts.forward (training
 *        branch with index_add_), SpeedupMoeSparseMoeBlock.forward
 *        (norm_topk_prob renormalisation).
 *   [EP] huggingface/transformers PR #41053 "Qwen3 moe":
 *        Ep2DpParallel._token_dispatch (rank-major received buffer that has to
 *        be reshuffled back into expert order).
 *   [PF] PaddlePaddle/PaddleFormers PR #2702 "[Unified MoE Layer]: Add MoE
 *        Layer with DeepEP EP Support; Add Qwen3MoE EP", review of
 *        paddleformers/nn/moe_deepep/moe_gate.py: _probs_drop_policy (the
 *        capacity drop policy).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Ownership: every array argument is a DEVICE pointer owned by the caller,
 *   except where a comment says "host".  The library keeps no state between
 *   calls and allocates no device memory; scratch space is the caller's
 *   workspace `ws` of at least the size the matching *_workspace_size()
 *   returns (256-byte aligned).
 * Layout: row-major, contiguous.  `dt` is the element type of x, the expert
 *   weights, x_perm, the hidden activation, y and out.  Router logits and
 *   routing weights are always fp32; indices and counts are int32.
 * Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *   work is asynchronous on it and no entry point synchronises the host,
 *   except moe_get_device_status.
 * Errors: arguments are checked on the host before anything is launched;
 *   a bad argument returns MOE_ERR_INVALID_ARG and launches nothing.  Shapes
 *   the sm_100a kernels do not cover return MOE_ERR_UNSUPPORTED (there is no
 *   CPU fallback).  A failed launch returns MOE_ERR_CUDA.  Bad *data* found
 *   on the device (an expert id outside [0,E), regroup counts that do not sum
 *   to the row count, offsets that are not a valid segmentation, a pipeline
 *   wait that ran out of time) never traps: the kernels skip the offending
 *   element, keep every access in bounds and OR a MOE_DEV_* bit into the
 *   status word at the start of the workspace.  Each entry point that takes
 *   `ws` clears that word when it starts; read it with
 *   moe_get_device_status.  moe_last_error() describes the last host-side
 *   error of the calling thread.
 * Empty inputs: T == 0 (or N == 0) is a valid no-op that still writes the
 *   zero counts / offsets it is asked for.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_CUDA = 3,
  MOE_ERR_WORKSPACE = 4,
  MOE_ERR_DEVICE = 5
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

/* Score function of the router ([HP] TokenChoiceTopKRouter, score_func):
 * softmax over the E experts, or an element-wise sigmoid.  Other values
 * return MOE_ERR_INVALID_ARG. */
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_t;

/* Bits of the device status word. */
#define MOE_DEV_BAD_EXPERT 1   /* dispatch: expert id outside [0, E)            */
#define MOE_DEV_BAD_COUNTS 2   /* regroup: counts negative or not summing to rows */
#define MOE_DEV_BAD_OFFSETS 4  /* grouped_swiglu: offsets not 0..N non-decreasing;
                                  dispatch: a slot outside [0, T k) (its workspace
                                  changed while the call ran) */
#define MOE_DEV_TIMEOUT 8      /* a pipeline wait exceeded its time limit        */

/* Limits of this build. */
#define MOE_MAX_EXPERTS 512
#define MOE_MAX_TOPK 16

/* ------------------------------------------------------------------------
 * moe_router_topk -- [HP] TokenChoiceTopKRouter.forward without bias,
 * groups or scale; [QO] SpeedupMoeSparseMoeBlock.forward (norm_topk_prob).
 *
 *   scores  = logits_in            if logits_in != NULL
 *           = x @ w_router^T (fp32 accumulation, no rounding of the logits)
 *   p       = softmax(scores) over all E experts (score MOE_SCORE_SOFTMAX)
 *           = sigmoid(scores)                    (score MOE_SCORE_SIGMOID)
 *   topk_idx[t, 0..k-1] = the k largest scores, largest first; equal scores
 *             go to the lower expert index (selection is made on the fp32
 *             scores; p is increasing in them so this is the top-k of p)
 *   topk_w[t, j] = p[t, topk_idx[t, j]], divided by their sum over j when
 *             renormalize != 0
 *   counts[e] = number of (t, j) with topk_idx[t, j] == e
 *
 * x        [T, d]  dt, may be NULL when logits_in is given
 * w_router [E, d]  dt (the bias-free gate nn.Linear(d, E) weight)
 * logits_in  [T, E] fp32 or NULL
 * logits_out [T, E] fp32 or NULL (written when the GEMM runs)
 * topk_idx [T, k] int32, topk_w [T, k] fp32, counts [E] int32 or NULL.
 * NaN scores are treated as -inf for the selection.
 * Requires 1 <= top_k <= min(E, 16), E <= 512, d % 8 == 0 for bf16 (whole
 * 16-byte rows), 16-byte aligned x / w_router.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_router_workspace_size(int T, int d, int E, moe_dtype_t dt);
MOE_API moe_status_t moe_router_topk(const void* x, const void* w_router, const float* logits_in,
                             int T, int d, int E, int top_k, moe_score_t score,
                             int renormalize, moe_dtype_t dt, float* logits_out,
                             int32_t* topk_idx, float* topk_w, int32_t* counts,
                             void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Router options -- the settings of [HP] TokenChoiceTopKRouter.__init__ and
 * of the MoE module around it (expert_bias, tokens_per_expert,
 * score_before_experts), taken by moe_router_topk_ex and moe_forward_ex.
 *
 * For token t with logits z (fp32) the router computes
 *   s      = softmax(z) over the E experts, or sigmoid(z)      (score)
 *   c      = s * route_scale
 *   c'     = c with every expert outside the topk_groups groups of largest
 *            max(c) set to -inf, when num_groups > 0 (node-limited routing;
 *            groups are the num_groups equal runs of consecutive experts;
 *            equal group maxima go to the lower group index)
 *   key    = c' + expert_bias          (expert_bias may be NULL = 0)
 *   topk_idx[t, :] = the k largest keys, largest first, ties to the lower
 *            expert index
 *   topk_w[t, j]   = s[topk_idx[t, j]] (the unbiased score, before the
 *            scale), divided by the sum over j when renormalize != 0, then
 *            times route_scale
 *   tokens_per_expert[e] += number of (t, j) with topk_idx[t, j] == e
 *   *aux_loss = E * sum_e f_e * P_e, f_e = #{(t, j): topk_idx = e} / (T k),
 *            P_e = sum of those copies' topk_w / T: the load-balance loss of
 *            this call ([HP] _compute_load_balance_loss without the
 *            sequence-partition reduction; 0 for T = 0; P_e is summed with
 *            fp32 atomics, so its last bits depend on the order of blocks)
 * Keys are compared in fp32.  Without expert_bias and with route_scale > 0
 * the keys are increasing functions of z, and the selection (groups
 * included) is made on z itself, so it is exact.
 *
 * score_before_experts (moe_forward_ex only; [HP] MoE.forward): the routed
 * row of copy (t, j) is multiplied by topk_w[t, j] before the experts
 * (fp32 product, rounded once to dt) and the combine is unweighted.
 * moe_router_options_init sets the defaults: softmax, no renormalisation,
 * route_scale 1, no bias, no groups, no histogram, and weights applied after
 * the experts (score_before_experts = 0, the semantics of moe_forward).
 *
 * Rules: route_scale finite and != 0; num_groups = 0, or 1 <= num_groups
 * <= 32 dividing E with 1 <= topk_groups <= num_groups and
 * top_k <= topk_groups * (E / num_groups); expert_bias [E] fp32 device or
 * NULL; tokens_per_expert [E] fp32 device or NULL (accumulated, never
 * cleared by the library); aux_loss one fp32 device scalar or NULL (written).
 *
 * aux_loss_coef (backward only: moe_router_backward, moe_backward): a trainer
 * that adds aux_loss_coef * aux_loss to its objective ([HP] adds the
 * auxiliary loss to the training loss) gets its gradient here: the routing
 * weight of a copy routed to expert e receives aux_loss_coef * E * f_e / T
 * (f_e as above; the counts carry no gradient), added to d_topk_w before the
 * router's backward.  0 (the default) adds nothing.
 *
 * capacity ([PF] PaddleFormers moe_gate.py, _probs_drop_policy): 0 (the
 * default) keeps every copy.  With capacity > 0 a token keeps its copy for
 * expert e only if its score for e is among the `capacity` highest scores of
 * the copies routed to e (the score before renormalisation and route_scale;
 * equal scores to the lower token index): a dropped copy gets topk_idx = -1
 * and topk_w = 0, the kept weights are unchanged, and `counts` counts the
 * kept copies (tokens_per_expert and aux_loss still count the routed ones).
 * moe_dispatch skips -1 without an error; moe_combine and the backward
 * entry points skip the positions of dropped copies.  moe_forward_ex: bf16
 * and ep_ranks = 1 only; the training entry points take no capacity.
 *
 * topk_scores (output, [T, k] fp32 device, or NULL): the score of each
 * selected expert before renormalisation and route_scale (softmax or
 * sigmoid of the logits), the key the capacity policy ranks by.
 * ---------------------------------------------------------------------- */
typedef struct moe_router_options {
  moe_score_t score;
  int renormalize;
  float route_scale;
  const float* expert_bias;
  int num_groups;
  int topk_groups;
  float* tokens_per_expert;
  int score_before_experts;
  float* aux_loss;
  float aux_loss_coef;
  int capacity;
  float* topk_scores;
} moe_router_options_t;

MOE_API void moe_router_options_init(moe_router_options_t* opts);

/* moe_router_topk_ex -- moe_router_topk with the options above (opts NULL =
 * the defaults).  Same arguments, workspace, outputs and error rules as
 * moe_router_topk otherwise; score_before_experts is ignored here. */
MOE_API moe_status_t moe_router_topk_ex(const void* x, const void* w_router,
                                        const float* logits_in, int T, int d, int E, int top_k,
                                        const moe_router_options_t* opts, moe_dtype_t dt,
                                        float* logits_out, int32_t* topk_idx, float* topk_w,
                                        int32_t* counts, void* ws, size_t ws_bytes,
                                        void* stream);

/* ------------------------------------------------------------------------
 * moe_dispatch -- [HP] MoE.permutation (stable argsort of the flat expert
 * ids, bincount) and the gather routed_x = x_flat[token_indices].
 *
 * With f = t*k + j the flat index of copy (t, j):
 *   counts[e]    = #{f : topk_idx[f] == e}
 *   offsets[e]   = sum_{e' < e} counts[e'],  offsets[E] = T*k
 *   dst_pos[t,j] = offsets[e] + #{f' < f : topk_idx[f'] == e}   (slot of the copy)
 *   src_row[s]   = t for the copy in slot s
 *   x_perm[s, :] = x[src_row[s], :]   (skipped when x_perm == NULL)
 * The order inside an expert segment is increasing f, so the result is
 * unique and bit-exact.  topk_idx [T, k] int32; counts [E]; offsets [E+1];
 * src_row [T*k]; dst_pos [T, k]; x [T, d] and x_perm [T*k, d] dt.
 * An id of -1 is a copy the capacity policy dropped: it is skipped (dst_pos
 * = -1, no slot) without an error.  Other ids outside [0, E) set
 * MOE_DEV_BAD_EXPERT; such copies get dst_pos = -1,
 * take no slot, and the unused tail slots of src_row are -1.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_dispatch_workspace_size(int T, int E, int top_k);
MOE_API moe_status_t moe_dispatch(const void* x, const int32_t* topk_idx, int T, int d, int E,
                          int top_k, moe_dtype_t dt, int32_t* counts, int32_t* offsets,
                          int32_t* src_row, int32_t* dst_pos, void* x_perm, void* ws,
                          size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_dispatch_noalloc -- moe_dispatch without a caller workspace.  The
 * pages have no counterpart: it exists for callers that cannot allocate
 * device memory where they dispatch, e.g. an engine or plugin whose enqueue
 * path must not allocate, a server whose device memory is all reserved by
 * another framework's pool, or a latency-critical path that must never wait
 * on an allocator.
 *
 * Same arguments, outputs and error behaviour as moe_dispatch, minus ws.
 * Its scratch (status word and per-block histogram table) is a fixed
 * MOE_NOALLOC_SCRATCH_BYTES array inside the library, held by every GPU that
 * loads it until the process exits.  Sizes for which
 * moe_dispatch_workspace_size(T, E, top_k) exceeds MOE_NOALLOC_SCRATCH_BYTES
 * (for E = 128 about a million tokens) return MOE_ERR_UNSUPPORTED with a
 * message and launch nothing.  It allocates nothing: no cudaMalloc,
 * cudaFree or allocating library call.
 * Each call made outside stream capture looks the array's device address
 * up (cudaGetSymbolAddress, with the device current), so a device reset or a
 * re-created context is followed; a call on a capturing stream uses the
 * address of the last lookup on that device, so make one call on the device
 * before any capture.  All calls share the array and it keeps the last call's
 * contents (each call rewrites the status word and the table), so calls
 * that overlap on the GPU -- on different streams, or from several host
 * threads -- race; serialise them.  The device status word is not exposed:
 * ids outside [0, E) show up as dst_pos = -1 and offsets[E] < T*k.
 * ---------------------------------------------------------------------- */
#define MOE_NOALLOC_SCRATCH_BYTES (4 << 20)
MOE_API moe_status_t moe_dispatch_noalloc(const void* x, const int32_t* topk_idx, int T, int d,
                                          int E, int top_k, moe_dtype_t dt, int32_t* counts,
                                          int32_t* offsets, int32_t* src_row, int32_t* dst_pos,
                                          void* x_perm, void* stream);

/* ------------------------------------------------------------------------
 * moe_ep_dispatch_rank_major -- the layout in which R expert-parallel ranks
 * receive the routed copies ([EP] Ep2DpParallel._token_dispatch): source
 * rank r owns tokens [r*S, min(T, (r+1)*S)), S = ceil(T/R), and destination
 * rank g owns experts [g*L, (g+1)*L), L = E / R.  The buffer lists, for
 * g = 0..R-1, for r = 0..R-1, for l = 0..L-1, the copies of source r for
 * expert g*L + l in increasing flat index.  Produced on one GPU as if after
 * the all-to-all (no communication).
 *   counts_rm [R, R, L] (indexed [g][r][l]); offsets_rm [R*R*L + 1];
 *   src_row [T*k]; dst_pos [T, k]; x_rm [T*k, d] or NULL.
 * Requires E % R == 0 and E*R <= 8192.  Other rules as moe_dispatch.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_ep_dispatch_workspace_size(int T, int E, int top_k, int R);
MOE_API moe_status_t moe_ep_dispatch_rank_major(const void* x, const int32_t* topk_idx, int T, int d,
                                        int E, int top_k, int R, moe_dtype_t dt,
                                        int32_t* counts_rm, int32_t* offsets_rm,
                                        int32_t* src_row, int32_t* dst_pos, void* x_rm,
                                        void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_ep_local_regroup -- [EP] Ep2DpParallel._token_dispatch: the received
 * buffer "is not sorted by expert anymore" and "needs to be reshuffled back".
 *
 * in [rows, d] holds, for each destination block g, segments (r, l) in
 * source-rank-major order (r outer, l inner) of counts_rm[g][r][l] rows.
 * out [rows, d] holds the same rows local-expert-major (l outer, r inner):
 *   for g, for l, for r: segment (g, r, l)
 * perm [rows]: out row -> in row.  counts_em [G*L] = sum_r counts_rm[g][r][l];
 * offsets_em [G*L + 1].  perm_inv [rows] (in row -> out row) or NULL.
 * counts_rm [G, R, L] int32 device array.  If the counts are negative or do
 * not sum to rows, MOE_DEV_BAD_COUNTS is set and nothing is copied.
 * G*R*L <= 8192.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_regroup_workspace_size(int G, int R, int L);
MOE_API moe_status_t moe_ep_local_regroup(const void* in, const int32_t* counts_rm, int G, int R,
                                  int L, int rows, int d, moe_dtype_t dt, void* out,
                                  int32_t* counts_em, int32_t* offsets_em, int32_t* perm,
                                  int32_t* perm_inv, void* ws, size_t ws_bytes,
                                  void* stream);

/* ------------------------------------------------------------------------
 * moe_grouped_swiglu -- [HP] _run_experts_for_loop / _run_experts_grouped_mm_gpu
 * (GroupedExperts weights [E, out, in]).
 *
 * For every expert e with rows s in [offsets[e], offsets[e+1]):
 *   H[s] = silu(x_perm[s] . w1[e]^T) * (x_perm[s] . w3[e]^T)      (fp32 acc)
 *   y[s] = (H[s] . w2[e]^T) * (row_scale ? row_scale[s] : 1)        (fp32 acc)
 * bf16: H is rounded to bf16 once (it is the GEMM2 operand), y once.
 * fp32: everything in fp32.  Experts with no rows are skipped.
 * x_perm [N, d]; offsets [E+1] int32 (device); w1, w3 [E, h, d]; w2 [E, d, h];
 * row_scale [N] fp32 or NULL; y [N, d].
 * bf16 requires d % 64 == 0 and h % 64 == 0 (tcgen05 path); fp32 requires
 * d % 4 == 0 and h % 4 == 0.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_grouped_swiglu_workspace_size(int N, int d, int h, int E, moe_dtype_t dt);
MOE_API moe_status_t moe_grouped_swiglu(const void* x_perm, const int32_t* offsets, const void* w1,
                                const void* w3, const void* w2, const float* row_scale,
                                int N, int d, int h, int E, moe_dtype_t dt, void* y,
                                void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_grouped_swiglu_gather -- moe_grouped_swiglu without the expert-major
 * copy of the tokens: the rows of expert segment s are read straight from
 * x through src_row (the gather [HP] MoE.forward writes as
 * routed_x = x_flat[token_indices], fused into the first GEMM's loads).
 *   H[s] = silu(x[src_row[s]] . w1[e]^T) * (x[src_row[s]] . w3[e]^T), then
 *   y[s] as moe_grouped_swiglu.
 * x [T, d]; src_row [N] int32 (device; entries outside [0, T) read zeros);
 * offsets [E+1]; weights, row_scale, y, ws and the shape rules as
 * moe_grouped_swiglu (workspace: moe_grouped_swiglu_workspace_size).
 * ---------------------------------------------------------------------- */
MOE_API moe_status_t moe_grouped_swiglu_gather(const void* x, int T, const int32_t* src_row,
                                       const int32_t* offsets, const void* w1, const void* w3,
                                       const void* w2, const float* row_scale, int N, int d,
                                       int h, int E, moe_dtype_t dt, void* y, void* ws,
                                       size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_grouped_swiglu_combine -- the grouped SwiGLU with the combine folded
 * into GEMM2's epilogue ([HP] MoE.unpermutation's scatter_add done by the
 * expert GEMM itself): no y [N, d] is written.
 *   out[t] = sum_j w[t, j] * (H[s] . w2[e(s)]^T),  s = dst_pos[t, j]
 * with H as moe_grouped_swiglu (bf16) and w = topk_w (fp32) or 1 when
 * topk_w == NULL.  Each GEMM2 output row, times its weight, is added in
 * fp32 into the token's row of an fp32 buffer in the workspace (the order
 * of the k additions is not fixed, so results may differ run to run in the
 * last fp32 bits), which is rounded once to bf16 into out [T, d].
 * x_perm [N, d] with N = T * top_k, offsets [E+1], w1, w3 [E, h, d], w2
 * [E, d, h], dst_pos [T, top_k] from moe_dispatch (positions outside
 * [0, N) add nothing).  bf16 only, d % 64 == 0, h % 64 == 0, and only where
 * the grouped SwiGLU runs on CTA pairs (N >= 64 E); otherwise
 * MOE_ERR_UNSUPPORTED.  Workspace moe_grouped_swiglu_combine_workspace_size
 * (status word, H, the fp32 output, the slots' tokens and weights).
 * Measured slower on B200 than moe_grouped_swiglu + moe_combine (8-32 %
 * on the bf16 workloads: the fp32 reductions move twice the bytes of the
 * bf16 rows they replace), and not bitwise reproducible, so moe_forward
 * keeps the separate gather-reduce; this entry point serves callers that
 * cannot hold y [N, d].
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_grouped_swiglu_combine_workspace_size(int T, int top_k, int d, int h, int E,
                                                 moe_dtype_t dt);
MOE_API moe_status_t moe_grouped_swiglu_combine(const void* x_perm, const int32_t* offsets,
                                        const void* w1, const void* w3, const void* w2,
                                        const int32_t* dst_pos, const float* topk_w, int T,
                                        int top_k, int d, int h, int E, moe_dtype_t dt,
                                        void* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_combine -- [QO] SpeedupMoeExperts.forward training branch
 * (weighted index_add_); [HP] MoE.unpermutation (scatter_add).
 *
 *   out[t, :] = sum_{j=0..k-1} w[t, j] * y[r(t, j), :]
 *   r(t, j)   = row_map ? row_map[dst_pos[t, j]] : dst_pos[t, j]
 *   w         = topk_w (fp32) or 1 when topk_w == NULL
 * Accumulated in fp32 over j = 0..k-1 in order, rounded once to dt.
 * y [N, d]; dst_pos [T, k]; row_map [N] or NULL; out [T, d].  Positions
 * outside [0, N) (e.g. -1 from a bad expert id) contribute nothing.
 * ---------------------------------------------------------------------- */
MOE_API moe_status_t moe_combine(const void* y, const int32_t* dst_pos, const int32_t* row_map,
                         const float* topk_w, int T, int d, int N, int top_k,
                         moe_dtype_t dt, void* out, void* stream);

/* ------------------------------------------------------------------------
 * Training path: the backward of the experts, the combine and the dispatch.
 * The pages train these layers ([HP] MoE.forward under autograd, [QO]
 * SpeedupMoeExperts training branch); the gradients below are the
 * derivatives of the forward definitions above, by the chain rule.
 *
 * moe_grouped_swiglu_train -- moe_grouped_swiglu (no row_scale) that also
 * returns what the backward needs:
 *   H [N, h]   = silu(G) * U, in dt (the GEMM2 operand)
 *   gu [N, 2h] = G | U with G = x_perm[s] . w1[e]^T in columns [0, h) and
 *                U = x_perm[s] . w3[e]^T in [h, 2h), each rounded once to
 *                dt from the fp32 accumulator (bf16: tcgen05; fp32: CUDA
 *                cores, no rounding).
 * Shapes and alignment as moe_grouped_swiglu; rows of empty experts are not
 * written; y is bit-identical to moe_grouped_swiglu's.  No workspace beyond
 * a 256-byte device status word (ws, ws_bytes >= 256).
 *
 * moe_grouped_swiglu_backward -- for every expert e with rows S (the
 * segment of x_perm), G, U from gu and upstream gradient dY = dy[seg]:
 *   dA = dY . w2[e];  dU = dA * silu(G);  dG = dA * U * silu'(G)
 *   dx_perm[seg] = dG . w1[e] + dU . w3[e]                    [N, d]
 *   dw1[e] = dG^T . S,  dw3[e] = dU^T . S                      [E, h, d]
 *   dw2[e] = dY^T . H[seg]                                    [E, d, h]
 * silu'(g) = s(g) (1 + g (1 - s(g))), s the logistic sigmoid.  bf16: fp32
 * accumulation on tcgen05 tensor cores, dG and dU rounded to bf16 once
 * (they are operands of the next products), every output once; d % 64 == 0
 * and h % 64 == 0.  fp32: CUDA cores, fp32 throughout; d % 4 == 0 and
 * h % 4 == 0.  Experts with no rows get zero weight gradients.  All
 * pointers 16-byte aligned; workspace
 * moe_grouped_swiglu_backward_workspace_size (dG | dU [N, 2h] in dt plus
 * the status word).  Bad offsets set MOE_DEV_BAD_OFFSETS in the status
 * word (moe_get_device_status) and the outputs are not written.
 *
 * moe_combine_backward -- gradient of moe_combine (row_map NULL):
 *   dy[dst_pos[t, j]] = w[t, j] * dout[t]      (one rounding to dt)
 *   d_topk_w[t, j]    = <dout[t], y[dst_pos[t, j]]>   (fp32 accumulation)
 * w = topk_w or 1 when topk_w == NULL; d_topk_w may be NULL (not computed).
 * dout [T, d]; y, dy [N, d]; dst_pos [T, k].  Slots outside [0, N) are
 * skipped (their d_topk_w is 0).  bf16 or fp32; d a whole number of
 * 16-byte vectors.
 *
 * moe_dispatch_backward -- gradient of x_perm = x[src_row] with respect to
 * x: dx[t] = dx_add[t] + sum_j dx_perm[dst_pos[t, j]] (fp32 sum over j in
 * order, one rounding): the unweighted combine.  dx_add [T, d] or NULL (the
 * router's share of dx, from moe_router_backward).  Rules as moe_combine.
 *
 * moe_router_backward -- gradient of the routing weights of
 * moe_router_topk_ex with respect to the gate logits and the gate's inputs,
 * for upstream gradients d_topk_w [T, k] and the experts the forward
 * selected (topk_idx).  Selection has no gradient: the expert bias and the
 * group masking only choose experts.  Per token, with s the scores
 * (softmax or sigmoid of the saved fp32 logits [T, E], as opts->score), S
 * the selected experts and c = opts->route_scale:
 *   w_j = c s_j / sum_S s   (opts->renormalize)   or   w_j = c s_j
 *   ds_j = c (g_j - sum_S g s / sum_S s) / sum_S s   or   ds_j = c g_j
 *   (0 for experts outside S)
 *   dz = s * (ds - <s, ds>)   (softmax)   or   dz = ds * s * (1 - s)  (sigmoid)
 *   d_logits = dz (fp32, optional), dw_router = dz^T x [E, d] (optional),
 *   dx = dz w_router [T, d] (optional)
 * dt = MOE_BF16: the gate products run on tcgen05 from dz rounded once to
 * bf16, with fp32 accumulation (E % 8 == 0 and d % 64 == 0); dw_router is
 * reduced over token segments into fp32 partials summed in segment order
 * (deterministic).  dt = MOE_F32: fp32 x, w_router, dw_router and dx; the
 * products run on CUDA cores from dz in fp32.  opts NULL =
 * defaults (softmax, no renormalisation, scale 1).  E <= 512.  Workspace
 * moe_router_backward_workspace_size (dz, the partials and the status
 * word).  Entries of topk_idx outside [0, E) are skipped.
 * ---------------------------------------------------------------------- */
MOE_API moe_status_t moe_grouped_swiglu_train(const void* x_perm, const int32_t* offsets,
                                      const void* w1, const void* w3, const void* w2, int N,
                                      int d, int h, int E, moe_dtype_t dt, void* y, void* h_act,
                                      void* gu, void* ws, size_t ws_bytes, void* stream);
MOE_API size_t moe_grouped_swiglu_backward_workspace_size(int N, int d, int h, int E,
                                                  moe_dtype_t dt);
MOE_API moe_status_t moe_grouped_swiglu_backward(const void* x_perm, const int32_t* offsets,
                                         const void* w1, const void* w3, const void* w2,
                                         const void* h_act, const void* gu, const void* dy,
                                         int N, int d, int h, int E, moe_dtype_t dt,
                                         void* dx_perm, void* dw1, void* dw3, void* dw2,
                                         void* ws, size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_combine_backward(const void* dout, const void* y,
                                  const int32_t* dst_pos, const float* topk_w, int T, int d,
                                  int N, int top_k, moe_dtype_t dt, void* dy, float* d_topk_w,
                                  void* stream);
MOE_API moe_status_t moe_dispatch_backward(const void* dx_perm, const int32_t* dst_pos,
                                   const void* dx_add, int T, int d, int N, int top_k,
                                   moe_dtype_t dt, void* dx, void* stream);
MOE_API size_t moe_router_backward_workspace_size(int T, int d, int E);
MOE_API moe_status_t moe_router_backward(const float* logits, const int32_t* topk_idx,
                                 const float* d_topk_w, const void* x, const void* w_router,
                                 int T, int d, int E, int top_k,
                                 const moe_router_options_t* opts, moe_dtype_t dt,
                                 float* d_logits, void* dw_router, void* dx, void* ws,
                                 size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_forward_train / moe_backward -- the whole layer's training step in two
 * calls ([HP] MoE.forward trained under autograd).
 *
 * moe_forward_train computes `out` exactly as moe_forward (ep_ranks = 1, no
 * shared expert) and keeps in `state` (caller-owned, opaque, sized by
 * moe_train_state_size) what the backward needs: the router's fp32 logits,
 * the routing, the dispatch layout, x_perm, the experts' outputs, H and G | U.
 * The state must stay untouched until moe_backward has run on the stream.
 * logits_in (as moe_forward) replaces the gate; the state then keeps a copy.
 *
 * moe_backward, for an upstream gradient dout [T, d] of `out`, runs the
 * chain rule through every step (the entry points of the training path
 * above, in order: combine, experts, router, dispatch) and writes
 *   dw1, dw3 [E, h, d], dw2 [E, d, h]         the expert weight gradients
 *   dw_router [E, d] (NULL: not computed)      the gate's weight gradient
 *   dx [T, d]                                  the input gradient: the sum of
 *      each token's copies' gradients, plus the router's share dz w_router
 *      when dw_router is computed (a gate driven by logits_in has neither)
 *   d_logits [T, E] fp32 (NULL: not written)   the logits' gradient dz
 * `opts` must be the options of the forward (score, renormalize, route_scale
 * enter the router's derivative; bias and groups only selected;
 * aux_loss_coef adds the load-balance loss's gradient).  With
 * score_before_experts ([HP] MoE.forward) the forward scales the routed rows
 * by their weights and combines unweighted, and the backward takes the
 * weights' gradient from the scaled rows, d topk_w[t, j] =
 * <dx_perm[p(t, j)], x[t]>, and weights each copy's share of dx by topk_w
 * (x is then required).  bf16 only; d % 64 == 0, h % 64 == 0, E % 8 == 0.
 * Workspace: moe_backward_workspace_size.  Device errors: the status word of
 * `state` (forward) and of `ws` (backward).  A shared expert: the _ex forms
 * below.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_train_state_size(int T, int d, int E, int top_k, int h);
MOE_API moe_status_t moe_forward_train(const void* x, const void* w_router,
                                       const float* logits_in, const void* w1, const void* w3,
                                       const void* w2, int T, int d, int E, int top_k, int h,
                                       const moe_router_options_t* opts, moe_dtype_t dt,
                                       void* out, void* state, size_t state_bytes,
                                       void* stream);
MOE_API size_t moe_backward_workspace_size(int T, int d, int E, int top_k, int h);
MOE_API moe_status_t moe_backward(const void* dout, const void* x, const void* w_router,
                                  const void* w1, const void* w3, const void* w2, int T, int d,
                                  int E, int top_k, int h, const moe_router_options_t* opts,
                                  moe_dtype_t dt, const void* state, void* dx, float* d_logits,
                                  void* dw_router, void* dw1, void* dw3, void* dw2, void* ws,
                                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_forward -- [HP] MoE.forward with score_before_experts=False and no
 * shared expert: router -> dispatch -> grouped SwiGLU -> combine.
 * With ep_ranks R > 1 the routed rows are laid out as R simulated EP ranks
 * would receive them (moe_ep_dispatch_rank_major), regrouped
 * (moe_ep_local_regroup) and then run through the experts; the result is
 * the same function.  out [T, d]; topk_idx/topk_w/counts/logits_out are
 * optional copies of the router outputs.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_forward_workspace_size(int T, int d, int E, int top_k, int h, int ep_ranks,
                                  moe_dtype_t dt);
MOE_API moe_status_t moe_forward(const void* x, const void* w_router, const float* logits_in,
                         const void* w1, const void* w3, const void* w2, int T, int d, int E,
                         int top_k, int h, moe_score_t score, int renormalize, int ep_ranks,
                         moe_dtype_t dt, void* out, float* logits_out, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                         void* stream);

/* Shared expert of [HP] MoE.forward (shared_expert = FeedForward(dim,
 * hidden)): a dense SwiGLU on every token whose output is added to the routed
 * output,  out[t] += (silu(x[t] w1^T) * (x[t] w3^T)) w2^T.
 * w1, w3 [h, d] and w2 [d, h] in dt (device, 16-byte aligned); bf16 needs
 * h % 64 == 0, fp32 h % 4 == 0. */
typedef struct moe_shared_expert {
  const void* w1;
  const void* w3;
  const void* w2;
  int h;
} moe_shared_expert_t;

/* moe_forward_ex -- [HP] MoE.forward with the router options above (opts
 * NULL = the defaults) and an optional shared expert (shared NULL = none;
 * both NULL make it moe_forward).  With score_before_experts the routed rows
 * are scaled in the dispatch copy and the combine sums the expert outputs
 * unweighted.  The shared expert runs as a one-segment grouped SwiGLU over
 * x; the combine adds its row to each token's routed sum in fp32 before the
 * single rounding to dt.  Workspace: moe_forward_ex_workspace_size with
 * h_shared = shared->h (0 without a shared expert, which equals
 * moe_forward_workspace_size).  Other arguments and error rules as
 * moe_forward. */
MOE_API size_t moe_forward_ex_workspace_size(int T, int d, int E, int top_k, int h, int ep_ranks,
                                             moe_dtype_t dt, int h_shared);
MOE_API moe_status_t moe_forward_ex(const void* x, const void* w_router, const float* logits_in,
                                    const void* w1, const void* w3, const void* w2, int T, int d,
                                    int E, int top_k, int h, const moe_router_options_t* opts,
                                    const moe_shared_expert_t* shared, int ep_ranks,
                                    moe_dtype_t dt, void* out, float* logits_out,
                                    int32_t* topk_idx, float* topk_w, int32_t* counts, void* ws,
                                    size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_forward_train_ex / moe_backward_ex -- moe_forward_train / moe_backward
 * with a shared expert ([HP] MoE.forward: out = routed + shared_expert(x),
 * a dense SwiGLU FFN on every token; `shared` as moe_forward_ex, NULL =
 * none).  The forward keeps the shared expert's H [T, hs] and G | U
 * [T, 2hs] in the state (moe_train_state_size_ex); the backward runs its
 * backward as a one-segment grouped SwiGLU backward over all T tokens with
 * the layer's upstream gradient dout, writes dws1, dws3 [hs, d] and dws2
 * [d, hs] (required when `shared` is given) and adds its share of dx.
 * Workspace: moe_backward_workspace_size_ex.  h_shared = 0 gives the sizes
 * of the plain forms, which are these calls with shared = NULL.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_train_state_size_ex(int T, int d, int E, int top_k, int h, int h_shared);
MOE_API moe_status_t moe_forward_train_ex(const void* x, const void* w_router,
                                          const float* logits_in, const void* w1,
                                          const void* w3, const void* w2, int T, int d, int E,
                                          int top_k, int h, const moe_router_options_t* opts,
                                          const moe_shared_expert_t* shared, moe_dtype_t dt,
                                          void* out, void* state, size_t state_bytes,
                                          void* stream);
MOE_API size_t moe_backward_workspace_size_ex(int T, int d, int E, int top_k, int h,
                                              int h_shared);
MOE_API moe_status_t moe_backward_ex(const void* dout, const void* x, const void* w_router,
                                     const void* w1, const void* w3, const void* w2, int T, int d,
                                     int E, int top_k, int h, const moe_router_options_t* opts,
                                     const moe_shared_expert_t* shared, moe_dtype_t dt,
                                     const void* state, void* dx, float* d_logits,
                                     void* dw_router, void* dw1, void* dw3, void* dw2,
                                     void* dws1, void* dws3, void* dws2, void* ws,
                                     size_t ws_bytes, void* stream);

/* moe_selftest_timeout -- test of the failure path every pipeline of the
 * library shares (no counterpart on the pages).  Launches one thread that
 * waits, through the library's bounded mbarrier wait, on a shared-memory
 * barrier that nothing arrives at.  After the wait limit (2 s of
 * %globaltimer) the wait gives up, the kernel ORs MOE_DEV_TIMEOUT into the
 * status word at the start of ws (cleared first) and returns; nothing
 * faults or traps, and the context stays usable.  ws: device, >= 256 bytes.
 * Asynchronous on `stream` like every entry point. */
MOE_API moe_status_t moe_selftest_timeout(void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then copies the status word at the start of `ws`
 * into *code (host).  Returns MOE_ERR_CUDA if the copy fails. */
MOE_API moe_status_t moe_get_device_status(const void* ws, int* code, void* stream);

/* Static description of a status code (never NULL). */
MOE_API const char* moe_status_string(moe_status_t s);

/* Text of the last host-side error raised on the calling thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
MOE_API int moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_MOE_H */
