// Internal (non-exported) launchers shared by the translation units of libmoe.
// Every launcher enqueues on `stream`, never synchronises, and returns the
// cudaError_t of its launches.  `status` points at the device status word.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

namespace tc {
// 2-D bf16 tensor map over a row-major [rows, inner] array, box [box_rows, 64],
// 128-byte swizzle, zero fill outside the array.
bool make_tmap(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows);
}  // namespace tc

int num_sms();                               // SM count of the current device
void set_last_error(const char* fmt, ...);   // thread-local text for moe_last_error

// ---- router -------------------------------------------------------------
// The tcgen05 router GEMM splits the reduction over d so that the number of
// (128-token, K-split) tiles is close to kRouterTargetTiles (the SM count of
// a B200); the plan depends on the sizes only, so workspace sizes can be
// computed on the host without a device.
constexpr int kRouterTargetTiles = 148;
struct RouterPlan {
  int ksplit;         // number of K splits (partial logit buffers)
  int kb_per_split;   // 64-wide K blocks per split
};
RouterPlan router_plan(int T, int d);
// tcgen05 router GEMM (bf16, E <= 256): fp32 partial logits [ksplit, T, E].
cudaError_t launch_router_tc(const void* x, const void* w_router, int T, int d, int E,
                             float* logits_part, int* status, cudaStream_t s);
// Fused tcgen05 router (bf16, E <= 256, no node-limited groups): the gate
// contraction on clusters of C CTAs per 128-token tile, the partial logits
// reduced through distributed shared memory, then scores, top-k and weights
// by one thread per token -- one kernel.  `plan`/`blk` as launch_router_topk
// (the dispatch histogram); `counts` (or null) is written through the
// per-CTA table `counts_part` ([grid, E] ints) by a second kernel;
// tokens_per_expert and lb (2E floats) are added to.  With clear_status the
// kernel clears the status word itself (it is the call's only writer).
struct RouterFusedPlan {
  int bn;           // accumulator columns (E rounded up to 32, 64, 128 or 256)
  int tiles;        // 128-token tiles
  int C;            // CTAs per tile (cluster size)
  int kb_total, kb_per_cta;
  int pitch;        // fp32 row pitch of the partial logits in shared memory
  int region;       // shared bytes before the barriers (stages / exchange)
  int smem;         // dynamic shared memory of a CTA
  int grid;
  bool ok;          // the plan fits the kernel's shared memory
};
struct DispatchPlan;
RouterFusedPlan router_fused_plan(int T, int d, int E, const DispatchPlan* plan);
// The dispatch plan of a whole-layer call: token blocks small enough that
// every CTA of the fused router owns whole blocks.
DispatchPlan layer_dispatch_plan(int T, int d, int E, int top_k, int R, moe_dtype_t dt);
struct RouterOptions;
cudaError_t launch_router_fused(const void* x, const void* w_router, int T, int d, int E,
                                int top_k, int renorm, const RouterOptions& o, float* logits_out,
                                int32_t* topk_idx, float* topk_w, int32_t* counts,
                                int32_t* counts_part, float* tokens_per_expert, float* lb,
                                const DispatchPlan* plan, int32_t* blk, int* status,
                                bool clear_status, cudaStream_t s);
// CUDA-core fp32 logits (x fp32 or bf16) into `logits` [T, E].
cudaError_t launch_router_logits_simt(const void* x, const void* w_router, int T, int d, int E,
                                      moe_dtype_t dt, float* logits, cudaStream_t s);
// ---- dispatch plan ----------------------------------------------------------
struct DispatchPlan {
  int T, k, E, R, L, S;   // R = 1: plain dispatch; R > 1: rank-major EP layout
  int nbins;              // E or E * R
  int tb;                 // tokens per block
  int nblk;
};
// max_tb caps the tokens per block (a power of two >= 8): inside the layer
// the fused router writes the histogram table, and each of its CTAs owns
// 128 / C tokens (layer_dispatch_plan).
DispatchPlan make_dispatch_plan(int T, int E, int top_k, int R, int max_tb = 128);
size_t dispatch_ws_bytes(const DispatchPlan& p);
// Host-side argument rules shared by every dispatch entry point (returns
// MOE_OK or MOE_ERR_INVALID_ARG with the text for moe_last_error set).
moe_status_t check_dispatch_args(const void* x, const int32_t* topk_idx, int T, int d, int E,
                                 int top_k, int R, moe_dtype_t dt, const int32_t* counts,
                                 const int32_t* offsets, const int32_t* src_row,
                                 const int32_t* dst_pos, const void* x_perm);

// Scoring options of the top-k kernel (moe_router_options_t without the
// host-only fields).  sigmoid: score function; scale: route_scale; bias:
// expert_bias [E] or null; groups / topk_groups: node-limited routing (0 =
// off).
struct RouterOptions {
  int sigmoid = 0;
  float scale = 1.0f;
  const float* bias = nullptr;
  int groups = 0;
  int topk_groups = 0;
  // [T, k] or null: the score of each selected expert before renormalisation
  // and scale (the key of the capacity drop policy)
  float* scores_out = nullptr;
};

// Sum of `nsplit` partial logit arrays [nsplit, T, E] (in split order), then
// scores / top-k / weights as `o` says; writes the logits if asked.  With
// `plan` and `blk` it also writes the dispatch histogram table of `plan`
// (so launch_dispatch can skip its histogram kernel).  The expert histogram
// is added to `counts` (int) and to `tokens_per_expert` (fp32) when given;
// with `lb` (2E zeroed floats) it adds the copies per expert to lb[0..E)
// and their routing weights to lb[E..2E).
cudaError_t launch_router_topk(const float* parts, int nsplit, int T, int E, int top_k,
                               int renorm, const RouterOptions& o, float* logits_out,
                               int32_t* topk_idx, float* topk_w, int32_t* counts,
                               float* tokens_per_expert, const DispatchPlan* plan,
                               int32_t* blk, cudaStream_t s, float* lb = nullptr);
// *loss = E * sum_e (lb[e] / (T k)) * (lb[E + e] / T), or 0 for T = 0.
cudaError_t launch_lb_loss(const float* lb, int E, int T, int top_k, float* loss, cudaStream_t s);

// ---- dispatch -------------------------------------------------------------
// hist_done: the histogram table in `ws` was already written (by the router).
// row_w [T*k] (or null): copy f = t*k + j of row t is multiplied by row_w[f]
// (fp32 product, one rounding to dt) as it is written to x_perm.
// own_status: the call's only kernels (the dispatch entry points): the
// column scan writes the whole status word (MOE_DEV_BAD_EXPERT or 0), so no
// clearing is needed before the call; otherwise nothing is written to it.
cudaError_t launch_dispatch(const DispatchPlan& p, const void* x, const int32_t* topk_idx,
                            int d, moe_dtype_t dt, int32_t* counts, int32_t* offsets,
                            int32_t* src_row, int32_t* dst_pos, void* x_perm, void* ws,
                            int* status, cudaStream_t s, bool hist_done = false,
                            const float* row_w = nullptr, bool own_status = false);

// ---- regroup ----------------------------------------------------------------
// One kernel (the segment tables are rebuilt in every block's shared
// memory).  own_status: the call's only kernel, which writes the whole status
// word (no clearing before it); otherwise it only adds MOE_DEV_BAD_COUNTS.
size_t regroup_ws_bytes(int G, int R, int L);
cudaError_t launch_regroup(const void* in, const int32_t* counts_rm, int G, int R, int L,
                           int rows, int d, moe_dtype_t dt, void* out, int32_t* counts_em,
                           int32_t* offsets_em, int32_t* perm, int32_t* perm_inv, void* ws,
                           int* status, cudaStream_t s, bool own_status = false);

// ---- combine ----------------------------------------------------------------
// shared, shared2 [T, d] (or null): rows added to each token's weighted sum
// in fp32 before the rounding (the shared expert's output; in the backward
// the router's and the shared expert's shares of dx).
cudaError_t launch_combine(const void* y, const int32_t* dst_pos, const int32_t* row_map,
                           const float* topk_w, int T, int d, int N, int top_k, moe_dtype_t dt,
                           void* out, cudaStream_t s, const void* shared = nullptr,
                           const void* shared2 = nullptr);
// Backward of the combine: dy [N, d] (every slot p(t, j) = w[t, j] dout[t];
// w = 1 when topk_w is null) and, if d_topk_w is given, the fp32 dot products
// <dout[t], y[p(t, j)]> ([T, k]).
cudaError_t launch_combine_backward(const void* dout, const void* y, const int32_t* dst_pos,
                                    const float* topk_w, int T, int d, int N, int top_k,
                                    moe_dtype_t dt, void* dy, float* d_topk_w, cudaStream_t s);
// Router backward: dz = d(routing weights)/d(logits) applied to d_topk_w,
// per token from the saved fp32 logits; dz32 [T, E] fp32 and dz16 [T, E]
// bf16 are each optional.
// With lb_counts (the expert counts of the forward, [E]) every selected
// expert e's upstream gradient gets lb_scale * lb_counts[e] added (the
// load-balance loss's gradient: lb_scale = coef * E / (T * T k)).
cudaError_t launch_router_backward(const float* logits, const int32_t* topk_idx,
                                   const float* d_topk_w, int T, int E, int top_k, int sigmoid,
                                   int renorm, float scale, float* dz32, void* dz16,
                                   cudaStream_t s, const int32_t* lb_counts = nullptr,
                                   float lb_scale = 0.f);
// Capacity drop policy: for every expert with more than `capacity` routed
// copies, keep the `capacity` of them with the highest score (scores [T, k],
// the router's scores_out), equal scores to the lower token; the others get
// topk_idx = -1 and topk_w = 0.  thr is device scratch for E 64-bit keys;
// counts [E] (or null) receives the copies each expert keeps.
cudaError_t launch_capacity_drop(int32_t* topk_idx, float* topk_w, const float* scores, int T,
                                 int k, int E, int capacity, unsigned long long* thr,
                                 int32_t* counts, cudaStream_t s);
// counts [E] += histogram of idx [n] (counts cleared by the caller).
cudaError_t launch_expert_hist(const int32_t* idx, long long n, int E, int32_t* counts,
                               cudaStream_t s);
// Gradients of the gate x . w_router^T for dz16 [T, E] bf16: dw_router =
// dz^T x [E, d] and dx = dz w_router [T, d] (bf16, each optional); offsets2 is
// device scratch for two ints.
// dw_router is reduced over gate_splits(T, d, E) token segments into fp32
// partials [splits, E, d] (gpart), then summed in order; offsets holds
// splits + 1 ints (at most 64).
int gate_splits(int T, int d, int E);
cudaError_t launch_gate_backward_tc(const void* dz16, const void* x, const void* w_router, int T,
                                    int d, int E, void* dw_router, void* dx, int32_t* offsets,
                                    float* gpart, int* status, cudaStream_t s);
// offsets[i] = floor(i n / S), i = 0..S.
cudaError_t launch_uniform_segments(int32_t* offsets, int S, int n, cudaStream_t s);
// out [n] bf16 = sum over S fp32 partial arrays [S, n] (n a multiple of 4).
cudaError_t launch_sum_partials_bf16(const float* part, int S, size_t n, void* out,
                                     cudaStream_t s);
// Self-test of the bounded wait: sets MOE_DEV_TIMEOUT after kWaitLimitNs.
cudaError_t launch_selftest_timeout(int* status, cudaStream_t s);
// offsets[0] = 0, offsets[1] = n: the segmentation of a single expert.
cudaError_t launch_single_segment(int32_t* offsets, int n, cudaStream_t s);

// ---- grouped SwiGLU -----------------------------------------------------
// bf16 tcgen05 path: H (bf16 [N, h]) is scratch.
// rows_upto: offsets[E] may be below N (the rows past it are dropped copies
// and stay uncomputed).
cudaError_t launch_swiglu_tc(const void* x_perm, const int32_t* offsets, const void* w1,
                             const void* w3, const void* w2, const float* row_scale, int N,
                             int d, int h, int E, void* y, void* H, int* status,
                             cudaStream_t s, bool rows_upto = false);
// Same with GEMM1's rows read from x [T, d] through src_row [N] (TMA gather4).
cudaError_t launch_swiglu_tc_gather(const void* x, int T, const int32_t* src_row,
                                    const int32_t* offsets, const void* w1, const void* w3,
                                    const void* w2, const float* row_scale, int N, int d, int h,
                                    int E, void* y, void* H, int* status, cudaStream_t s);
// Training forward: also writes GU [N, 2h] bf16 (G = x w1^T | U = x w3^T),
// and H [N, h] is an output the backward reads.
cudaError_t launch_swiglu_tc_train(const void* x_perm, const int32_t* offsets, const void* w1,
                                   const void* w3, const void* w2, int N, int d, int h, int E,
                                   void* y, void* H, void* GU, int* status, cudaStream_t s);
// Whether the bf16 grouped SwiGLU of N rows over E experts runs on the
// CTA-pair kernel (segments averaging 64 rows or more).
bool swiglu_tc_uses_pairs(int N, int E);
// The grouped SwiGLU with the combine folded into GEMM2 (CTA-pair path only,
// cudaErrorInvalidValue otherwise): out32 [T, d] fp32 (zero before the
// call) += slot_w[s] * y[s] at row slot_tok[s] for every slot s; H [N, h]
// is scratch.
cudaError_t launch_swiglu_tc_combine(const void* x_perm, const int32_t* offsets, const void* w1,
                                     const void* w3, const void* w2, int N, int d, int h, int E,
                                     void* H, const int32_t* slot_tok, const float* slot_w,
                                     int T, float* out32, int* status, cudaStream_t s);
// slot_tok[dst_pos[t, j]] = t and slot_w[dst_pos[t, j]] = topk_w[t, j] (1
// when topk_w is null) for every position inside [0, N); slot_tok must be
// preset to -1.
cudaError_t launch_slot_map(const int32_t* dst_pos, const float* topk_w, int T, int top_k, int N,
                            int32_t* slot_tok, float* slot_w, cudaStream_t s);
// out [n] bf16 = in [n] fp32, rounded to nearest even (n a multiple of 8).
cudaError_t launch_f32_to_bf16(const float* in, size_t n, void* out, cudaStream_t s);
// Backward of the grouped SwiGLU (bf16, tcgen05): dX [N, d], dW1/dW3 [E, h, d],
// dW2 [E, d, h]; dGU [N, 2h] bf16 is scratch.
cudaError_t launch_swiglu_bwd_tc(const void* x_perm, const int32_t* offsets, const void* w1,
                                 const void* w3, const void* w2, const void* H, const void* GU,
                                 const void* dY, int N, int d, int h, int E, void* dX, void* dW1,
                                 void* dW3, void* dW2, void* dGU, int* status, cudaStream_t s);
// fp32 CUDA-core path: H (fp32 [N, h]) is scratch.
cudaError_t launch_swiglu_simt_f32(const float* x_perm, const int32_t* offsets,
                                   const float* w1, const float* w3, const float* w2,
                                   const float* row_scale, int N, int d, int h, int E, float* y,
                                   float* H, int* status, cudaStream_t s);
// fp32 training forward: also writes GU [N, 2h] fp32 (G | U), H is an output.
cudaError_t launch_swiglu_simt_f32_train(const float* x_perm, const int32_t* offsets,
                                         const float* w1, const float* w3, const float* w2,
                                         int N, int d, int h, int E, float* y, float* H,
                                         float* GU, int* status, cudaStream_t s);
// fp32 backward of the grouped SwiGLU on CUDA cores; dGU [N, 2h] fp32 scratch.
cudaError_t launch_swiglu_bwd_simt_f32(const float* x_perm, const int32_t* offsets,
                                       const float* w1, const float* w3, const float* w2,
                                       const float* H, const float* GU, const float* dY, int N,
                                       int d, int h, int E, float* dX, float* dW1, float* dW3,
                                       float* dW2, float* dGU, int* status, cudaStream_t s);
// fp32 gate gradients: dw_router = dz^T x [E, d], dx = dz w_router [T, d]
// (each optional) for dz [T, E] fp32.
cudaError_t launch_gate_backward_f32(const float* dz, const float* x, const float* w_router,
                                     int T, int d, int E, float* dw_router, float* dx,
                                     cudaStream_t s);
cudaError_t launch_swiglu_simt_f32_gather(const float* x, int x_rows, const int32_t* src_row,
                                          const int32_t* offsets, const float* w1,
                                          const float* w3, const float* w2,
                                          const float* row_scale, int N, int d, int h, int E,
                                          float* y, float* H, int* status, cudaStream_t s);

}  // namespace moe
