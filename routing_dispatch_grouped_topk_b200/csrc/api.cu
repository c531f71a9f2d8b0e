// C ABI of libmoe (include/moe.h): host-side argument checks, workspace
// layout and the launch sequence of every entry point.  Nothing here
// computes on the host: every step of the layer runs in the kernels.
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace moe {

static thread_local char g_err[512] = "";

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64) {
    if (!cache[dev]) {
      int n = 0;
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
      cache[dev] = n > 0 ? n : 1;
    }
    return cache[dev];
  }
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

namespace {

constexpr size_t kStatusBytes = 256;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t elt_bytes(moe_dtype_t dt) { return dt == MOE_BF16 ? 2 : 4; }

#define MOE_CHECK_ARG(cond, ...)            \
  do {                                      \
    if (!(cond)) {                          \
      set_last_error(__VA_ARGS__);          \
      return MOE_ERR_INVALID_ARG;           \
    }                                       \
  } while (0)

moe_status_t cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return MOE_OK;
  set_last_error("%s: %s", where, cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

moe_status_t check_dtype(moe_dtype_t dt) {
  MOE_CHECK_ARG(dt == MOE_F32 || dt == MOE_BF16, "dt must be MOE_F32 or MOE_BF16");
  return MOE_OK;
}

// Row length in bytes must be whole 16-byte vectors.
moe_status_t check_rows(int d, moe_dtype_t dt, const char* name) {
  MOE_CHECK_ARG(d >= 1 && (static_cast<size_t>(d) * elt_bytes(dt)) % 16 == 0,
                "%s: d=%d must be >= 1 and a multiple of %d for this dtype", name, d,
                static_cast<int>(16 / elt_bytes(dt)));
  return MOE_OK;
}

bool router_uses_tc(int E, moe_dtype_t dt) { return dt == MOE_BF16 && E <= 256; }

// Load-balance statistics (copies and weight sums per expert, 2E floats).
size_t lb_bytes(int E) { return align_up(2 * static_cast<size_t>(E) * sizeof(float), 256); }

// Per-count factor of the load-balance loss's gradient: a copy routed to
// expert e gets coef * E * f_e / T with f_e = counts_e / (T k).
float lb_grad_scale(float coef, int E, int T, int k) {
  return T > 0 ? static_cast<float>(static_cast<double>(coef) * E /
                                    (static_cast<double>(T) * T * k))
               : 0.f;
}

// Status word, the load-balance statistics, the fp32 logit scratch ([ksplit,
// T, E] partial logits of the tensor-core GEMM, or [T, E] logits of the
// CUDA-core path), then the capacity policy's scratch: the selected scores
// [T, kMaxTopK] and one 64-bit threshold per expert.
size_t logit_scratch_bytes(int T, int d, int E, moe_dtype_t dt) {
  const size_t planes = router_uses_tc(E, dt) ? router_plan(T, d).ksplit : 1;
  return align_up(planes * T * E * sizeof(float), 256);
}
size_t capacity_scratch_bytes(int T, int E) {
  return align_up(static_cast<size_t>(T) * kMaxTopK * sizeof(float), 256) +
         align_up(static_cast<size_t>(E) * 8, 256);
}
size_t router_ws(int T, int d, int E, moe_dtype_t dt) {
  return kStatusBytes + lb_bytes(E) + logit_scratch_bytes(T, d, E, dt) +
         capacity_scratch_bytes(T, E);
}

moe_router_options_t default_options() {
  moe_router_options_t o;
  o.score = MOE_SCORE_SOFTMAX;
  o.renormalize = 0;
  o.route_scale = 1.0f;
  o.expert_bias = nullptr;
  o.num_groups = 0;
  o.topk_groups = 0;
  o.tokens_per_expert = nullptr;
  o.score_before_experts = 0;
  o.aux_loss = nullptr;
  o.aux_loss_coef = 0.0f;
  o.capacity = 0;
  o.topk_scores = nullptr;
  return o;
}

moe_status_t check_router(const void* x, const void* w_router, const float* logits_in, int T,
                          int d, int E, int top_k, const moe_router_options_t& o, moe_dtype_t dt,
                          const int32_t* topk_idx, const float* topk_w) {
  if (moe_status_t s = check_dtype(dt)) return s;
  MOE_CHECK_ARG(o.score == MOE_SCORE_SOFTMAX || o.score == MOE_SCORE_SIGMOID,
                "score must be MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID");
  MOE_CHECK_ARG(T >= 0, "T=%d must be >= 0", T);
  MOE_CHECK_ARG(E >= 1 && E <= kMaxExperts, "E=%d must be in [1, %d]", E, kMaxExperts);
  MOE_CHECK_ARG(top_k >= 1 && top_k <= std::min(E, kMaxTopK), "top_k=%d must be in [1, min(E, %d)]",
                top_k, kMaxTopK);
  MOE_CHECK_ARG(std::isfinite(o.route_scale) && o.route_scale != 0.0f,
                "route_scale must be finite and non-zero");
  MOE_CHECK_ARG(o.capacity >= 0, "capacity=%d must be >= 0", o.capacity);
  if (o.num_groups != 0) {
    MOE_CHECK_ARG(o.num_groups >= 1 && o.num_groups <= 32 && E % o.num_groups == 0,
                  "num_groups=%d must be in [1, 32] and divide E=%d", o.num_groups, E);
    MOE_CHECK_ARG(o.topk_groups >= 1 && o.topk_groups <= o.num_groups &&
                      top_k <= o.topk_groups * (E / o.num_groups),
                  "topk_groups=%d must be in [1, num_groups] and keep >= top_k experts",
                  o.topk_groups);
  }
  if (T > 0) {
    MOE_CHECK_ARG(topk_idx && topk_w, "topk_idx and topk_w are required");
    if (!logits_in) {
      MOE_CHECK_ARG(x && w_router, "x and w_router are required without logits_in");
      MOE_CHECK_ARG(aligned16(x) && aligned16(w_router), "x / w_router must be 16-byte aligned");
      if (moe_status_t s = check_rows(d, dt, "router")) return s;
    }
  }
  return MOE_OK;
}

}  // namespace

// Argument rules of the dispatch entry points (moe_dispatch,
// moe_ep_dispatch_rank_major, moe_dispatch_noalloc): one copy, so that every
// entry point rejects the same arguments with the same status and text.
moe_status_t check_dispatch_args(const void* x, const int32_t* topk_idx, int T, int d, int E,
                                 int top_k, int R, moe_dtype_t dt, const int32_t* counts,
                                 const int32_t* offsets, const int32_t* src_row,
                                 const int32_t* dst_pos, const void* x_perm) {
  if (moe_status_t st = check_dtype(dt)) return st;
  MOE_CHECK_ARG(T >= 0, "T must be >= 0");
  MOE_CHECK_ARG(E >= 1 && E <= kMaxExperts, "E=%d must be in [1, %d]", E, kMaxExperts);
  MOE_CHECK_ARG(top_k >= 1 && top_k <= std::min(E, kMaxTopK), "top_k=%d out of range", top_k);
  MOE_CHECK_ARG(R >= 1 && E % R == 0 && E * R <= kMaxBins, "R=%d must divide E and E*R <= %d", R,
                kMaxBins);
  MOE_CHECK_ARG(counts && offsets, "counts and offsets are required");
  if (T > 0) {
    MOE_CHECK_ARG(topk_idx && src_row && dst_pos, "topk_idx, src_row, dst_pos are required");
    if (x_perm) {
      MOE_CHECK_ARG(x != nullptr, "x is required when x_perm is given");
      MOE_CHECK_ARG(aligned16(x) && aligned16(x_perm), "x / x_perm must be 16-byte aligned");
      if (moe_status_t st = check_rows(d, dt, "dispatch")) return st;
    }
  }
  return MOE_OK;
}

namespace {

RouterOptions kernel_options(const moe_router_options_t& o) {
  RouterOptions k;
  k.sigmoid = o.score == MOE_SCORE_SIGMOID;
  k.scale = o.route_scale;
  k.bias = o.expert_bias;
  k.groups = o.num_groups;
  k.topk_groups = o.num_groups ? o.topk_groups : 0;
  k.scores_out = o.topk_scores;
  return k;
}

// The fused tcgen05 router (bf16, E <= 256, no group limit, logits from
// the gate) serves this call.
bool router_is_fused(const float* logits_in, int T, int d, int E, const moe_router_options_t& o,
                     moe_dtype_t dt, const DispatchPlan* plan) {
  return T > 0 && !logits_in && router_uses_tc(E, dt) && o.num_groups == 0 &&
         router_fused_plan(T, d, E, plan).ok;
}

// Router launch sequence.  With `plan` and `blk` the top-k step also writes
// the dispatch histogram.  The fused router writes `counts` without atomics
// (a per-CTA table and a summing kernel) and, with own_status, clears the
// status word itself; on the other paths the caller has cleared the status
// word and `counts` is cleared here (they add into it with atomics).
cudaError_t run_router(const void* x, const void* w_router, const float* logits_in, int T, int d,
                       int E, int top_k, const moe_router_options_t& o, moe_dtype_t dt,
                       float* logits_out, int32_t* topk_idx, float* topk_w, int32_t* counts,
                       void* scratch, int* status, cudaStream_t s,
                       const DispatchPlan* plan = nullptr, int32_t* blk = nullptr,
                       bool own_status = false) {
  RouterOptions ko = kernel_options(o);
  const int renorm = o.renormalize;
  float* tpe = o.tokens_per_expert;
  float* lb = o.aux_loss ? static_cast<float*>(scratch) : nullptr;
  float* part = reinterpret_cast<float*>(static_cast<char*>(scratch) + lb_bytes(E));
  // The capacity policy ranks the copies by their scores, kept by the router
  // (the caller's topk_scores or the scratch), and changes the routing after
  // the router: the dispatch histogram is then the dispatch's own.
  const bool cap = o.capacity > 0 && T > 0;
  char* cap_scratch = static_cast<char*>(scratch) + lb_bytes(E) + logit_scratch_bytes(T, d, E, dt);
  if (cap && !ko.scores_out) ko.scores_out = reinterpret_cast<float*>(cap_scratch);
  if (cap) {
    plan = nullptr;
    blk = nullptr;
  }
  cudaError_t e = cudaSuccess;
  if (lb) e = cudaMemsetAsync(lb, 0, 2 * sizeof(float) * E, s);
  const bool fused = router_is_fused(logits_in, T, d, E, o, dt, plan);
  if (e == cudaSuccess && counts && !fused)
    e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
  if (e == cudaSuccess && T > 0) {
    if (logits_in) {
      e = launch_router_topk(logits_in, 1, T, E, top_k, renorm, ko, nullptr, topk_idx, topk_w,
                             counts, tpe, plan, blk, s, lb);
    } else if (fused) {
      e = launch_router_fused(x, w_router, T, d, E, top_k, renorm, ko, logits_out, topk_idx,
                              topk_w, counts, reinterpret_cast<int32_t*>(part), tpe, lb, plan,
                              blk, status, own_status, s);
    } else if (router_uses_tc(E, dt)) {
      e = launch_router_tc(x, w_router, T, d, E, part, status, s);
      if (e == cudaSuccess)
        e = launch_router_topk(part, router_plan(T, d).ksplit, T, E, top_k, renorm, ko,
                               logits_out, topk_idx, topk_w, counts, tpe, plan, blk, s, lb);
    } else {
      float* L = logits_out ? logits_out : part;
      e = launch_router_logits_simt(x, w_router, T, d, E, dt, L, s);
      if (e == cudaSuccess)
        e = launch_router_topk(L, 1, T, E, top_k, renorm, ko, nullptr, topk_idx, topk_w, counts,
                               tpe, plan, blk, s, lb);
    }
  }
  // [PF] PaddleFormers moe_gate _probs_drop_policy; the counts then count
  // the kept copies (tokens_per_expert and the load-balance statistics keep
  // the routed ones: they measure the router, which the capacity then caps)
  if (e == cudaSuccess && cap) {
    unsigned long long* thr = reinterpret_cast<unsigned long long*>(
        cap_scratch + align_up(static_cast<size_t>(T) * kMaxTopK * sizeof(float), 256));
    e = launch_capacity_drop(topk_idx, topk_w, ko.scores_out, T, top_k, E, o.capacity, thr,
                             counts, s);
  }
  // [HP] _compute_load_balance_loss of this call (0 for no tokens)
  if (e == cudaSuccess && lb) e = launch_lb_loss(lb, E, T, top_k, o.aux_loss, s);
  return e;
}

size_t swiglu_ws(int N, int h, moe_dtype_t dt) {
  return kStatusBytes + align_up(static_cast<size_t>(N) * h * elt_bytes(dt), 256);
}

moe_status_t check_swiglu_shape(int N, int d, int h, int E, moe_dtype_t dt) {
  if (moe_status_t s = check_dtype(dt)) return s;
  MOE_CHECK_ARG(N >= 0 && E >= 1 && E <= kMaxExperts && d >= 1 && h >= 1,
                "bad sizes N=%d d=%d h=%d E=%d", N, d, h, E);
  if (dt == MOE_BF16) {
    if (d % 64 != 0 || h % 64 != 0) {
      set_last_error("bf16 grouped SwiGLU needs d %% 64 == 0 and h %% 64 == 0 (d=%d h=%d)", d, h);
      return MOE_ERR_UNSUPPORTED;
    }
  } else {
    MOE_CHECK_ARG(d % 4 == 0 && h % 4 == 0, "fp32 grouped SwiGLU needs d, h multiples of 4");
  }
  return MOE_OK;
}

cudaError_t run_swiglu(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3,
                       const void* w2, const float* row_scale, int N, int d, int h, int E,
                       moe_dtype_t dt, void* y, void* H, int* status, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  if (dt == MOE_BF16)
    return launch_swiglu_tc(x_perm, offsets, w1, w3, w2, row_scale, N, d, h, E, y, H, status, s);
  return launch_swiglu_simt_f32(static_cast<const float*>(x_perm), offsets,
                                static_cast<const float*>(w1), static_cast<const float*>(w3),
                                static_cast<const float*>(w2), row_scale, N, d, h, E,
                                static_cast<float*>(y), static_cast<float*>(H), status, s);
}

cudaError_t run_swiglu_gather(const void* x, int T, const int32_t* src_row,
                              const int32_t* offsets, const void* w1, const void* w3,
                              const void* w2, const float* row_scale, int N, int d, int h, int E,
                              moe_dtype_t dt, void* y, void* H, int* status, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  if (dt == MOE_BF16)
    return launch_swiglu_tc_gather(x, T, src_row, offsets, w1, w3, w2, row_scale, N, d, h, E, y,
                                   H, status, s);
  return launch_swiglu_simt_f32_gather(static_cast<const float*>(x), T, src_row, offsets,
                                       static_cast<const float*>(w1),
                                       static_cast<const float*>(w3),
                                       static_cast<const float*>(w2), row_scale, N, d, h, E,
                                       static_cast<float*>(y), static_cast<float*>(H), status, s);
}

struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* p) : base(static_cast<char*>(p)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align_up(count * sizeof(T), 256);
    return p;
  }
};

// Workspace of moe_forward.  The same function sizes it (base = null) and
// carves it, so the two can never disagree.
struct ForwardWs {
  int* status;
  void* router_scratch;
  int32_t* idx;
  float* w;
  int32_t* counts_a;    // counts (R = 1) or counts_rm (R > 1)
  int32_t* offsets_a;   // offsets or offsets_rm
  int32_t* src_row;
  int32_t* dst_pos;
  void* disp_ws;
  void* x_a;            // x_perm (R = 1) or rank-major rows (R > 1)
  void* x_em;
  int32_t* counts_em;
  int32_t* offsets_em;
  int32_t* perm;
  int32_t* perm_inv;
  void* reg_ws;
  void* y;
  void* H;
  int32_t* offsets_s;   // shared expert (hs > 0): its one-segment offsets,
  void* H_s;            // hidden activation [T, hs]
  void* y_s;            // and output [T, d]
  size_t bytes;
};

ForwardWs carve_forward(void* ws, int T, int d, int E, int k, int h, int R, moe_dtype_t dt,
                        int hs = 0) {
  ForwardWs f{};
  Carve c(ws);
  const size_t N = static_cast<size_t>(T) * k;
  const size_t row = static_cast<size_t>(d) * elt_bytes(dt);
  f.status = c.take<int>(kStatusBytes / sizeof(int));
  f.router_scratch = c.take<char>(router_ws(T, d, E, dt) - kStatusBytes);
  f.idx = c.take<int32_t>(N);
  f.w = c.take<float>(N);
  const DispatchPlan p = layer_dispatch_plan(T, d, E, k, R, dt);
  f.counts_a = c.take<int32_t>(static_cast<size_t>(p.nbins));
  f.offsets_a = c.take<int32_t>(static_cast<size_t>(p.nbins) + 1);
  f.src_row = c.take<int32_t>(N);
  f.dst_pos = c.take<int32_t>(N);
  f.disp_ws = c.take<char>(dispatch_ws_bytes(p));
  f.x_a = c.take<char>(N * row);
  if (R > 1) {
    f.x_em = c.take<char>(N * row);
    f.counts_em = c.take<int32_t>(E);
    f.offsets_em = c.take<int32_t>(static_cast<size_t>(E) + 1);
    f.perm = c.take<int32_t>(N);
    f.perm_inv = c.take<int32_t>(N);
    f.reg_ws = c.take<char>(regroup_ws_bytes(R, R, E / R));
  }
  f.y = c.take<char>(N * row);
  f.H = c.take<char>(N * static_cast<size_t>(h) * elt_bytes(dt));
  if (hs > 0) {
    f.offsets_s = c.take<int32_t>(2);
    f.H_s = c.take<char>(static_cast<size_t>(T) * hs * elt_bytes(dt));
    f.y_s = c.take<char>(static_cast<size_t>(T) * row);
  }
  f.bytes = c.off;
  return f;
}

// State a training forward keeps for its backward (caller-owned, opaque).
struct TrainState {
  int* status;
  float* logits;       // [T, E] fp32
  int32_t* idx;        // [T, k]
  float* w;            // [T, k]
  int32_t* counts;     // [E]
  int32_t* offsets;    // [E + 1]
  int32_t* src_row;    // [N]
  int32_t* dst_pos;    // [T, k]
  void* router_scratch;
  void* disp_ws;
  void* x_perm;        // [N, d]
  void* y;             // [N, d]
  void* H;             // [N, h]
  void* GU;            // [N, 2h]
  // shared expert (h_shared > 0): its one-segment offsets, output and the
  // training forward's H and G | U over every token
  int32_t* offsets_s;  // [2]
  void* ys;            // [T, d]
  void* Hs;            // [T, hs]
  void* GUs;           // [T, 2hs]
  size_t bytes;
};

TrainState carve_train(void* base, int T, int d, int E, int k, int h, int hs = 0) {
  TrainState t{};
  Carve c(base);
  const size_t N = static_cast<size_t>(T) * k;
  t.status = c.take<int>(kStatusBytes / sizeof(int));
  t.logits = c.take<float>(static_cast<size_t>(T) * E);
  t.idx = c.take<int32_t>(N);
  t.w = c.take<float>(N);
  const DispatchPlan p = layer_dispatch_plan(T, d, E, k, 1, MOE_BF16);
  t.counts = c.take<int32_t>(E);
  t.offsets = c.take<int32_t>(static_cast<size_t>(E) + 1);
  t.src_row = c.take<int32_t>(N);
  t.dst_pos = c.take<int32_t>(N);
  t.router_scratch = c.take<char>(router_ws(T, d, E, MOE_BF16) - kStatusBytes);
  t.disp_ws = c.take<char>(dispatch_ws_bytes(p));
  t.x_perm = c.take<char>(N * d * 2);
  t.y = c.take<char>(N * d * 2);
  t.H = c.take<char>(N * h * 2);
  t.GU = c.take<char>(N * 2 * h * 2);
  if (hs > 0) {
    t.offsets_s = c.take<int32_t>(2);
    t.ys = c.take<char>(static_cast<size_t>(T) * d * 2);
    t.Hs = c.take<char>(static_cast<size_t>(T) * hs * 2);
    t.GUs = c.take<char>(static_cast<size_t>(T) * 2 * hs * 2);
  }
  t.bytes = c.off;
  return t;
}

// Backward workspace of moe_backward.
struct BackwardWs {
  int* status;
  int32_t* off2;       // segment offsets of the gate's products (256 B)
  void* dY;            // [N, d]
  float* dtw;          // [T, k]
  void* dXp;           // [N, d]
  void* dGU;           // [N, 2h]
  void* dz16;          // [T, E]
  void* dxr;           // [T, d] the router's share of dx
  float* gpart;        // [splits, E, d] fp32 partials of dw_router
  void* dXs;           // [T, d] the shared expert's share of dx
  void* dGUs;          // [T, 2hs]
  size_t bytes;
};

BackwardWs carve_backward(void* base, int T, int d, int E, int k, int h, int hs = 0) {
  BackwardWs b{};
  Carve c(base);
  const size_t N = static_cast<size_t>(T) * k;
  b.status = c.take<int>(kStatusBytes / sizeof(int));
  b.off2 = c.take<int32_t>(64);
  b.dY = c.take<char>(N * d * 2);
  b.dtw = c.take<float>(N);
  b.dXp = c.take<char>(N * d * 2);
  b.dGU = c.take<char>(N * 2 * h * 2);
  b.dz16 = c.take<char>(static_cast<size_t>(T) * E * 2);
  b.dxr = c.take<char>(static_cast<size_t>(T) * d * 2);
  b.gpart = c.take<float>(static_cast<size_t>(gate_splits(T, d, E)) * E * d);
  if (hs > 0) {
    b.dXs = c.take<char>(static_cast<size_t>(T) * d * 2);
    b.dGUs = c.take<char>(static_cast<size_t>(T) * 2 * hs * 2);
  }
  b.bytes = c.off;
  return b;
}

// Shape and option rules of the whole-layer training entry points.
moe_status_t check_train(int T, int d, int E, int top_k, int h, const moe_router_options_t& o,
                         moe_dtype_t dt) {
  if (dt != MOE_BF16) {
    set_last_error("training entry points: bf16 only");
    return MOE_ERR_UNSUPPORTED;
  }
  if (o.capacity != 0) {
    set_last_error("training entry points: no capacity policy");
    return MOE_ERR_UNSUPPORTED;
  }
  MOE_CHECK_ARG(T >= 0 && E >= 1 && E <= kMaxExperts && top_k >= 1 && top_k <= kMaxTopK &&
                    top_k <= E,
                "bad sizes T=%d E=%d top_k=%d", T, E, top_k);
  if (moe_status_t st = check_swiglu_shape(T * top_k, d, h, E, dt)) return st;
  if (E % 8 != 0) {
    set_last_error("training entry points need E %% 8 == 0 (E=%d)", E);
    return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

// Shared expert of the training entry points: a dense SwiGLU FFN on every
// token, with the tensor-core rules of the grouped SwiGLU.
moe_status_t check_shared(const moe_shared_expert_t* sh, int T, int d, moe_dtype_t dt) {
  if (!sh) return MOE_OK;
  MOE_CHECK_ARG(sh->h >= 1, "shared->h=%d must be >= 1", sh->h);
  if (moe_status_t st = check_swiglu_shape(T, d, sh->h, 1, dt)) return st;
  MOE_CHECK_ARG(sh->w1 && sh->w3 && sh->w2, "shared expert w1, w3, w2 are required");
  MOE_CHECK_ARG(aligned16(sh->w1) && aligned16(sh->w3) && aligned16(sh->w2),
                "shared expert weights must be 16-byte aligned");
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return 1 * 10000 + 0 * 100 + 0; }

const char* moe_last_error(void) { return g_err; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or option";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

moe_status_t moe_selftest_timeout(void* ws, size_t ws_bytes, void* stream) {
  MOE_CHECK_ARG(ws != nullptr && ws_bytes >= kStatusBytes, "ws of at least %zu bytes is required",
                kStatusBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess) e = launch_selftest_timeout(status, s);
  return cuda_status(e, "moe_selftest_timeout");
}

moe_status_t moe_get_device_status(const void* ws, int* code, void* stream) {
  if (!ws || !code) {
    set_last_error("ws and code are required");
    return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "moe_get_device_status");
  *code = v;
  return MOE_OK;
}

// ------------------------------------------------------------------ router
size_t moe_router_workspace_size(int T, int d, int E, moe_dtype_t dt) {
  (void)d;
  if (T < 0 || E < 1) return kStatusBytes;
  return router_ws(T, d, E, dt);
}

void moe_router_options_init(moe_router_options_t* opts) {
  if (opts) *opts = default_options();
}

moe_status_t moe_router_topk_ex(const void* x, const void* w_router, const float* logits_in,
                                int T, int d, int E, int top_k, const moe_router_options_t* opts,
                                moe_dtype_t dt, float* logits_out, int32_t* topk_idx,
                                float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                void* stream) {
  const moe_router_options_t o = opts ? *opts : default_options();
  if (moe_status_t st = check_router(x, w_router, logits_in, T, d, E, top_k, o, dt, topk_idx,
                                     topk_w))
    return st;
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  if (ws_bytes < router_ws(T, d, E, dt)) {
    set_last_error("router workspace %zu < %zu", ws_bytes, router_ws(T, d, E, dt));
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  // the fused router clears the status word itself (it is the only kernel
  // that can write it); the other paths start from a cleared word
  const bool fused = router_is_fused(logits_in, T, d, E, o, dt, nullptr);
  cudaError_t e = fused ? cudaSuccess : cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = run_router(x, w_router, logits_in, T, d, E, top_k, o, dt, logits_out, topk_idx, topk_w,
                   counts, static_cast<char*>(ws) + kStatusBytes, status, s, nullptr, nullptr,
                   fused);
  return cuda_status(e, "moe_router_topk");
}

moe_status_t moe_router_topk(const void* x, const void* w_router, const float* logits_in, int T,
                             int d, int E, int top_k, moe_score_t score, int renormalize,
                             moe_dtype_t dt, float* logits_out, int32_t* topk_idx, float* topk_w,
                             int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  moe_router_options_t o = default_options();
  o.score = score;
  o.renormalize = renormalize;
  return moe_router_topk_ex(x, w_router, logits_in, T, d, E, top_k, &o, dt, logits_out, topk_idx,
                            topk_w, counts, ws, ws_bytes, stream);
}

// ----------------------------------------------------------------- dispatch
static moe_status_t dispatch_common(const void* x, const int32_t* topk_idx, int T, int d, int E,
                                    int top_k, int R, moe_dtype_t dt, int32_t* counts,
                                    int32_t* offsets, int32_t* src_row, int32_t* dst_pos,
                                    void* x_perm, void* ws, size_t ws_bytes, void* stream) {
  if (moe_status_t st = check_dispatch_args(x, topk_idx, T, d, E, top_k, R, dt, counts, offsets,
                                            src_row, dst_pos, x_perm))
    return st;
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const DispatchPlan p = make_dispatch_plan(T, E, top_k, R);
  const size_t need = kStatusBytes + dispatch_ws_bytes(p);
  if (ws_bytes < need) {
    set_last_error("dispatch workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  // the column scan writes the whole status word: nothing to clear first
  cudaError_t e = launch_dispatch(p, x, topk_idx, d, dt, counts, offsets, src_row, dst_pos,
                                  x ? x_perm : nullptr, static_cast<char*>(ws) + kStatusBytes,
                                  status, s, false, nullptr, /*own_status=*/true);
  return cuda_status(e, "moe_dispatch");
}

size_t moe_dispatch_workspace_size(int T, int E, int top_k) {
  if (T < 0 || E < 1 || top_k < 1) return kStatusBytes;
  return kStatusBytes + dispatch_ws_bytes(make_dispatch_plan(T, E, top_k, 1));
}

moe_status_t moe_dispatch(const void* x, const int32_t* topk_idx, int T, int d, int E, int top_k,
                          moe_dtype_t dt, int32_t* counts, int32_t* offsets, int32_t* src_row,
                          int32_t* dst_pos, void* x_perm, void* ws, size_t ws_bytes,
                          void* stream) {
  return dispatch_common(x, topk_idx, T, d, E, top_k, 1, dt, counts, offsets, src_row, dst_pos,
                         x_perm, ws, ws_bytes, stream);
}

size_t moe_ep_dispatch_workspace_size(int T, int E, int top_k, int R) {
  if (T < 0 || E < 1 || top_k < 1 || R < 1 || E % R) return kStatusBytes;
  return kStatusBytes + dispatch_ws_bytes(make_dispatch_plan(T, E, top_k, R));
}

moe_status_t moe_ep_dispatch_rank_major(const void* x, const int32_t* topk_idx, int T, int d,
                                        int E, int top_k, int R, moe_dtype_t dt,
                                        int32_t* counts_rm, int32_t* offsets_rm,
                                        int32_t* src_row, int32_t* dst_pos, void* x_rm, void* ws,
                                        size_t ws_bytes, void* stream) {
  return dispatch_common(x, topk_idx, T, d, E, top_k, R, dt, counts_rm, offsets_rm, src_row,
                         dst_pos, x_rm, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ regroup
size_t moe_regroup_workspace_size(int G, int R, int L) {
  if (G < 1 || R < 1 || L < 1) return kStatusBytes;
  return kStatusBytes + regroup_ws_bytes(G, R, L);
}

moe_status_t moe_ep_local_regroup(const void* in, const int32_t* counts_rm, int G, int R, int L,
                                  int rows, int d, moe_dtype_t dt, void* out,
                                  int32_t* counts_em, int32_t* offsets_em, int32_t* perm,
                                  int32_t* perm_inv, void* ws, size_t ws_bytes, void* stream) {
  if (moe_status_t st = check_dtype(dt)) return st;
  MOE_CHECK_ARG(G >= 1 && R >= 1 && L >= 1 && 1LL * G * R * L <= kMaxSegments,
                "G*R*L must be in [1, %d]", kMaxSegments);
  MOE_CHECK_ARG(rows >= 0, "rows must be >= 0");
  MOE_CHECK_ARG(counts_rm && counts_em && offsets_em, "counts_rm, counts_em, offsets_em required");
  if (rows > 0) {
    MOE_CHECK_ARG(in && out && perm, "in, out, perm are required");
    MOE_CHECK_ARG(aligned16(in) && aligned16(out), "in / out must be 16-byte aligned");
    if (moe_status_t st = check_rows(d, dt, "regroup")) return st;
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const size_t need = kStatusBytes + regroup_ws_bytes(G, R, L);
  if (ws_bytes < need) {
    set_last_error("regroup workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  // one kernel, which writes the whole status word itself
  cudaError_t e = launch_regroup(in, counts_rm, G, R, L, rows, d, dt, out, counts_em, offsets_em,
                                 perm, perm_inv, static_cast<char*>(ws) + kStatusBytes, status, s,
                                 /*own_status=*/true);
  return cuda_status(e, "moe_ep_local_regroup");
}

// ----------------------------------------------------------- grouped SwiGLU
size_t moe_grouped_swiglu_workspace_size(int N, int d, int h, int E, moe_dtype_t dt) {
  (void)d;
  (void)E;
  if (N < 0 || h < 1) return kStatusBytes;
  return swiglu_ws(N, h, dt);
}

moe_status_t moe_grouped_swiglu(const void* x_perm, const int32_t* offsets, const void* w1,
                                const void* w3, const void* w2, const float* row_scale, int N,
                                int d, int h, int E, moe_dtype_t dt, void* y, void* ws,
                                size_t ws_bytes, void* stream) {
  if (moe_status_t st = check_swiglu_shape(N, d, h, E, dt)) return st;
  if (N > 0) {
    MOE_CHECK_ARG(x_perm && offsets && w1 && w3 && w2 && y, "x_perm, offsets, w1, w3, w2, y required");
    MOE_CHECK_ARG(aligned16(x_perm) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                      aligned16(y),
                  "x_perm, w1, w3, w2, y must be 16-byte aligned");
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const size_t need = swiglu_ws(N, h, dt);
  if (ws_bytes < need) {
    set_last_error("grouped_swiglu workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = run_swiglu(x_perm, offsets, w1, w3, w2, row_scale, N, d, h, E, dt, y,
                   static_cast<char*>(ws) + kStatusBytes, status, s);
  return cuda_status(e, "moe_grouped_swiglu");
}

moe_status_t moe_grouped_swiglu_gather(const void* x, int T, const int32_t* src_row,
                                       const int32_t* offsets, const void* w1, const void* w3,
                                       const void* w2, const float* row_scale, int N, int d,
                                       int h, int E, moe_dtype_t dt, void* y, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (moe_status_t st = check_swiglu_shape(N, d, h, E, dt)) return st;
  MOE_CHECK_ARG(T >= 0, "T must be >= 0");
  if (N > 0) {
    MOE_CHECK_ARG(T > 0 && x && src_row && offsets && w1 && w3 && w2 && y,
                  "x (T > 0), src_row, offsets, w1, w3, w2, y required");
    MOE_CHECK_ARG(aligned16(x) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                      aligned16(y),
                  "x, w1, w3, w2, y must be 16-byte aligned");
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const size_t need = swiglu_ws(N, h, dt);
  if (ws_bytes < need) {
    set_last_error("grouped_swiglu workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = run_swiglu_gather(x, T, src_row, offsets, w1, w3, w2, row_scale, N, d, h, E, dt, y,
                          static_cast<char*>(ws) + kStatusBytes, status, s);
  return cuda_status(e, "moe_grouped_swiglu_gather");
}

// ------------------------------------------ grouped SwiGLU + folded combine
namespace {
// status, H [N, h] bf16, the fp32 output [T, d], slot tokens and weights [N]
struct FoldWs {
  int* status;
  void* H;
  float* out32;
  int32_t* slot_tok;
  float* slot_w;
  size_t bytes;
};
FoldWs carve_fold(void* base, int T, int k, int d, int h) {
  FoldWs f{};
  Carve c(base);
  const size_t N = static_cast<size_t>(T) * k;
  f.status = c.take<int>(kStatusBytes / sizeof(int));
  f.H = c.take<char>(N * h * 2);
  f.out32 = c.take<float>(static_cast<size_t>(T) * d);
  f.slot_tok = c.take<int32_t>(N);
  f.slot_w = c.take<float>(N);
  f.bytes = c.off;
  return f;
}
}  // namespace

size_t moe_grouped_swiglu_combine_workspace_size(int T, int top_k, int d, int h, int E,
                                                 moe_dtype_t dt) {
  (void)E;
  (void)dt;
  if (T < 0 || top_k < 1 || d < 1 || h < 1) return kStatusBytes;
  return carve_fold(nullptr, T, top_k, d, h).bytes;
}

moe_status_t moe_grouped_swiglu_combine(const void* x_perm, const int32_t* offsets,
                                        const void* w1, const void* w3, const void* w2,
                                        const int32_t* dst_pos, const float* topk_w, int T,
                                        int top_k, int d, int h, int E, moe_dtype_t dt, void* out,
                                        void* ws, size_t ws_bytes, void* stream) {
  MOE_CHECK_ARG(T >= 0 && top_k >= 1 && top_k <= kMaxTopK, "bad sizes T=%d top_k=%d", T, top_k);
  const int N = T * top_k;
  if (moe_status_t st = check_swiglu_shape(N, d, h, E, dt)) return st;
  if (dt != MOE_BF16 || (N > 0 && !swiglu_tc_uses_pairs(N, E))) {
    set_last_error("moe_grouped_swiglu_combine: bf16 layers whose segments average 64 rows or "
                   "more (the CTA-pair GEMM path); N=%d E=%d",
                   N, E);
    return MOE_ERR_UNSUPPORTED;
  }
  if (T > 0) {
    MOE_CHECK_ARG(x_perm && offsets && w1 && w3 && w2 && dst_pos && out,
                  "x_perm, offsets, w1, w3, w2, dst_pos, out are required");
    MOE_CHECK_ARG(aligned16(x_perm) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                      aligned16(out),
                  "x_perm, w1, w3, w2, out must be 16-byte aligned");
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const size_t need = moe_grouped_swiglu_combine_workspace_size(T, top_k, d, h, E, dt);
  if (ws_bytes < need) {
    set_last_error("grouped_swiglu_combine workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  const FoldWs f = carve_fold(ws, T, top_k, d, h);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(f.status, 0, sizeof(int), s);
  if (e == cudaSuccess && T > 0) {
    // slots no (t, j) points to keep token -1 and add nothing
    e = cudaMemsetAsync(f.slot_tok, 0xff, static_cast<size_t>(N) * sizeof(int32_t), s);
    if (e == cudaSuccess) e = launch_slot_map(dst_pos, topk_w, T, top_k, N, f.slot_tok, f.slot_w, s);
    if (e == cudaSuccess)
      e = cudaMemsetAsync(f.out32, 0, static_cast<size_t>(T) * d * sizeof(float), s);
    if (e == cudaSuccess)
      e = launch_swiglu_tc_combine(x_perm, offsets, w1, w3, w2, N, d, h, E, f.H, f.slot_tok,
                                   f.slot_w, T, f.out32, f.status, s);
    if (e == cudaSuccess) e = launch_f32_to_bf16(f.out32, static_cast<size_t>(T) * d, out, s);
  }
  return cuda_status(e, "moe_grouped_swiglu_combine");
}

// ------------------------------------------------------------------ combine
moe_status_t moe_combine(const void* y, const int32_t* dst_pos, const int32_t* row_map,
                         const float* topk_w, int T, int d, int N, int top_k, moe_dtype_t dt,
                         void* out, void* stream) {
  if (moe_status_t st = check_dtype(dt)) return st;
  MOE_CHECK_ARG(T >= 0 && N >= 0, "T, N must be >= 0");
  MOE_CHECK_ARG(top_k >= 1 && top_k <= kMaxTopK, "top_k=%d out of range", top_k);
  if (T > 0) {
    MOE_CHECK_ARG(out && dst_pos, "out and dst_pos are required");
    MOE_CHECK_ARG(N == 0 || y, "y is required");
    MOE_CHECK_ARG(aligned16(out) && aligned16(y), "y / out must be 16-byte aligned");
    if (moe_status_t st = check_rows(d, dt, "combine")) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_combine(y, dst_pos, row_map, topk_w, T, d, N, top_k, dt, out, s),
                     "moe_combine");
}

// ------------------------------------------------------------ training path
moe_status_t moe_grouped_swiglu_train(const void* x_perm, const int32_t* offsets, const void* w1,
                                      const void* w3, const void* w2, int N, int d, int h, int E,
                                      moe_dtype_t dt, void* y, void* h_act, void* gu, void* ws,
                                      size_t ws_bytes, void* stream) {
  if (moe_status_t st = check_swiglu_shape(N, d, h, E, dt)) return st;
  if (N > 0) {
    MOE_CHECK_ARG(x_perm && offsets && w1 && w3 && w2 && y && h_act && gu,
                  "x_perm, offsets, w1, w3, w2, y, h_act, gu required");
    MOE_CHECK_ARG(aligned16(x_perm) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                      aligned16(y) && aligned16(h_act) && aligned16(gu),
                  "x_perm, w1, w3, w2, y, h_act, gu must be 16-byte aligned");
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  if (ws_bytes < kStatusBytes) {
    set_last_error("grouped_swiglu_train workspace %zu < %zu", ws_bytes, kStatusBytes);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess && N > 0) {
    if (dt == MOE_BF16)
      e = launch_swiglu_tc_train(x_perm, offsets, w1, w3, w2, N, d, h, E, y, h_act, gu, status,
                                 s);
    else
      e = launch_swiglu_simt_f32_train(
          static_cast<const float*>(x_perm), offsets, static_cast<const float*>(w1),
          static_cast<const float*>(w3), static_cast<const float*>(w2), N, d, h, E,
          static_cast<float*>(y), static_cast<float*>(h_act), static_cast<float*>(gu), status, s);
  }
  return cuda_status(e, "moe_grouped_swiglu_train");
}

size_t moe_grouped_swiglu_backward_workspace_size(int N, int d, int h, int E, moe_dtype_t dt) {
  (void)d;
  (void)E;
  if (N < 0 || h < 1) return kStatusBytes;
  return kStatusBytes + align_up(static_cast<size_t>(N) * 2 * h * elt_bytes(dt), 256);
}

moe_status_t moe_grouped_swiglu_backward(const void* x_perm, const int32_t* offsets,
                                         const void* w1, const void* w3, const void* w2,
                                         const void* h_act, const void* gu, const void* dy, int N,
                                         int d, int h, int E, moe_dtype_t dt, void* dx_perm,
                                         void* dw1, void* dw3, void* dw2, void* ws,
                                         size_t ws_bytes, void* stream) {
  if (moe_status_t st = check_swiglu_shape(N, d, h, E, dt)) return st;
  MOE_CHECK_ARG(offsets && w1 && w3 && w2 && dw1 && dw3 && dw2,
                "offsets, w1, w3, w2, dw1, dw3, dw2 required");
  if (N > 0) {
    MOE_CHECK_ARG(x_perm && h_act && gu && dy && dx_perm,
                  "x_perm, h_act, gu, dy, dx_perm required");
    MOE_CHECK_ARG(aligned16(x_perm) && aligned16(h_act) && aligned16(gu) && aligned16(dy) &&
                      aligned16(dx_perm),
                  "x_perm, h_act, gu, dy, dx_perm must be 16-byte aligned");
  }
  MOE_CHECK_ARG(aligned16(w1) && aligned16(w3) && aligned16(w2) && aligned16(dw1) &&
                    aligned16(dw3) && aligned16(dw2),
                "w1, w3, w2, dw1, dw3, dw2 must be 16-byte aligned");
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const size_t need = moe_grouped_swiglu_backward_workspace_size(N, d, h, E, dt);
  if (ws_bytes < need) {
    set_last_error("grouped_swiglu_backward workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess && N == 0) {
    // no rows: every weight gradient is zero
    const size_t wbytes = static_cast<size_t>(E) * h * d * elt_bytes(dt);
    e = cudaMemsetAsync(dw1, 0, wbytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw3, 0, wbytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw2, 0, wbytes, s);
  } else if (e == cudaSuccess && dt == MOE_F32) {
    e = launch_swiglu_bwd_simt_f32(
        static_cast<const float*>(x_perm), offsets, static_cast<const float*>(w1),
        static_cast<const float*>(w3), static_cast<const float*>(w2),
        static_cast<const float*>(h_act), static_cast<const float*>(gu),
        static_cast<const float*>(dy), N, d, h, E, static_cast<float*>(dx_perm),
        static_cast<float*>(dw1), static_cast<float*>(dw3), static_cast<float*>(dw2),
        reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes), status, s);
  } else if (e == cudaSuccess) {
    e = launch_swiglu_bwd_tc(x_perm, offsets, w1, w3, w2, h_act, gu, dy, N, d, h, E, dx_perm, dw1,
                             dw3, dw2, static_cast<char*>(ws) + kStatusBytes, status, s);
  }
  return cuda_status(e, "moe_grouped_swiglu_backward");
}

moe_status_t moe_combine_backward(const void* dout, const void* y, const int32_t* dst_pos,
                                  const float* topk_w, int T, int d, int N, int top_k,
                                  moe_dtype_t dt, void* dy, float* d_topk_w, void* stream) {
  if (moe_status_t st = check_dtype(dt)) return st;
  MOE_CHECK_ARG(T >= 0 && N >= 0, "T, N must be >= 0");
  MOE_CHECK_ARG(top_k >= 1 && top_k <= kMaxTopK, "top_k=%d out of range", top_k);
  if (T > 0) {
    MOE_CHECK_ARG(dout && dst_pos && dy, "dout, dst_pos and dy are required");
    MOE_CHECK_ARG(!d_topk_w || y, "y is required for d_topk_w");
    MOE_CHECK_ARG(aligned16(dout) && aligned16(dy) && aligned16(y),
                  "dout / dy / y must be 16-byte aligned");
    if (moe_status_t st = check_rows(d, dt, "combine_backward")) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_combine_backward(dout, y, dst_pos, topk_w, T, d, N, top_k, dt, dy,
                                             d_topk_w, s),
                     "moe_combine_backward");
}

moe_status_t moe_dispatch_backward(const void* dx_perm, const int32_t* dst_pos,
                                   const void* dx_add, int T, int d, int N, int top_k,
                                   moe_dtype_t dt, void* dx, void* stream) {
  if (moe_status_t st = check_dtype(dt)) return st;
  MOE_CHECK_ARG(T >= 0 && N >= 0, "T, N must be >= 0");
  MOE_CHECK_ARG(top_k >= 1 && top_k <= kMaxTopK, "top_k=%d out of range", top_k);
  if (T > 0) {
    MOE_CHECK_ARG(dx && dst_pos, "dx and dst_pos are required");
    MOE_CHECK_ARG(N == 0 || dx_perm, "dx_perm is required");
    MOE_CHECK_ARG(aligned16(dx) && aligned16(dx_perm) && aligned16(dx_add),
                  "dx_perm / dx_add / dx must be 16-byte aligned");
    if (moe_status_t st = check_rows(d, dt, "dispatch_backward")) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_combine(dx_perm, dst_pos, nullptr, nullptr, T, d, N, top_k, dt, dx, s,
                                    dx_add),
                     "moe_dispatch_backward");
}

// status, segment offsets (256 B), dz in bf16 [T, E], fp32 partials of
// dw_router [splits, E, d]
size_t moe_router_backward_workspace_size(int T, int d, int E) {
  if (T < 0 || E < 1 || d < 1) return kStatusBytes;
  // status, gate segment offsets, dz (bf16 for the tcgen05 gate products,
  // fp32 for the fp32 ones), the gate's fp32 partials, then the expert
  // counts of the load-balance gradient
  return kStatusBytes + 256 + align_up(static_cast<size_t>(T) * E * 4, 256) +
         align_up(static_cast<size_t>(gate_splits(T, d, E)) * E * d * 4, 256) +
         align_up(static_cast<size_t>(E) * 4, 256);
}

moe_status_t moe_router_backward(const float* logits, const int32_t* topk_idx,
                                 const float* d_topk_w, const void* x, const void* w_router,
                                 int T, int d, int E, int top_k,
                                 const moe_router_options_t* opts, moe_dtype_t dt,
                                 float* d_logits, void* dw_router, void* dx, void* ws,
                                 size_t ws_bytes, void* stream) {
  const moe_router_options_t o = opts ? *opts : default_options();
  if (moe_status_t st = check_dtype(dt)) return st;
  MOE_CHECK_ARG(T >= 0 && d >= 1 && E >= 1 && E <= kMaxExperts, "bad sizes T=%d d=%d E=%d", T,
                d, E);
  MOE_CHECK_ARG(top_k >= 1 && top_k <= kMaxTopK && top_k <= E, "top_k=%d out of range", top_k);
  MOE_CHECK_ARG(o.score == MOE_SCORE_SOFTMAX || o.score == MOE_SCORE_SIGMOID, "bad score");
  MOE_CHECK_ARG(std::isfinite(o.route_scale) && o.route_scale != 0.0f, "bad route_scale");
  const bool gemm = dw_router || dx;
  if (gemm && dt == MOE_BF16 && (E % 8 != 0 || d % 64 != 0)) {
    set_last_error("bf16 router backward gate gradients need E %% 8 == 0 and d %% 64 == 0");
    return MOE_ERR_UNSUPPORTED;
  }
  if (T > 0) {
    MOE_CHECK_ARG(logits && topk_idx && d_topk_w, "logits, topk_idx, d_topk_w required");
    MOE_CHECK_ARG(!dw_router || x, "x is required for dw_router");
    MOE_CHECK_ARG(!dx || w_router, "w_router is required for dx");
    MOE_CHECK_ARG(aligned16(x) && aligned16(w_router) && aligned16(dw_router) && aligned16(dx),
                  "x, w_router, dw_router, dx must be 16-byte aligned");
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const size_t need = moe_router_backward_workspace_size(T, d, E);
  if (ws_bytes < need) {
    set_last_error("router_backward workspace %zu < %zu", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  int32_t* off2 = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + kStatusBytes);
  void* dz16 = static_cast<char*>(ws) + kStatusBytes + 256;
  float* gpart = reinterpret_cast<float*>(static_cast<char*>(dz16) +
                                          align_up(static_cast<size_t>(T) * E * 4, 256));
  int32_t* lbc = reinterpret_cast<int32_t*>(
      reinterpret_cast<char*>(gpart) +
      align_up(static_cast<size_t>(gate_splits(T, d, E)) * E * d * 4, 256));
  const bool lb = o.aux_loss_coef != 0.0f && T > 0;
  MOE_CHECK_ARG(std::isfinite(o.aux_loss_coef), "aux_loss_coef must be finite");
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess && T == 0 && dw_router)
    e = cudaMemsetAsync(dw_router, 0, static_cast<size_t>(E) * d * elt_bytes(dt), s);
  // fp32 gate products read dz in fp32: the caller's d_logits, else the
  // workspace
  const bool f32 = dt == MOE_F32;
  float* dz32 = f32 && gemm && !d_logits ? static_cast<float*>(dz16) : d_logits;
  // the load-balance gradient needs the forward's expert counts: recounted
  // from topk_idx
  if (e == cudaSuccess && lb) e = cudaMemsetAsync(lbc, 0, static_cast<size_t>(E) * 4, s);
  if (e == cudaSuccess && lb) e = launch_expert_hist(topk_idx, 1LL * T * top_k, E, lbc, s);
  if (e == cudaSuccess && T > 0)
    e = launch_router_backward(logits, topk_idx, d_topk_w, T, E, top_k,
                               o.score == MOE_SCORE_SIGMOID, o.renormalize, o.route_scale,
                               dz32, gemm && !f32 ? dz16 : nullptr, s, lb ? lbc : nullptr,
                               lb ? lb_grad_scale(o.aux_loss_coef, E, T, top_k) : 0.f);
  if (e == cudaSuccess && T > 0 && gemm && f32)
    e = launch_gate_backward_f32(dz32, static_cast<const float*>(x),
                                 static_cast<const float*>(w_router), T, d, E,
                                 static_cast<float*>(dw_router), static_cast<float*>(dx), s);
  else if (e == cudaSuccess && T > 0 && gemm)
    e = launch_gate_backward_tc(dz16, x, w_router, T, d, E, dw_router, dx, off2, gpart, status,
                                s);
  return cuda_status(e, "moe_router_backward");
}

// ---------------------------------------------------- whole-layer training
size_t moe_train_state_size(int T, int d, int E, int top_k, int h) {
  return moe_train_state_size_ex(T, d, E, top_k, h, 0);
}

size_t moe_train_state_size_ex(int T, int d, int E, int top_k, int h, int h_shared) {
  if (T < 0 || d < 1 || E < 1 || top_k < 1 || h < 1 || h_shared < 0) return kStatusBytes;
  return carve_train(nullptr, T, d, E, top_k, h, h_shared).bytes;
}

size_t moe_backward_workspace_size(int T, int d, int E, int top_k, int h) {
  return moe_backward_workspace_size_ex(T, d, E, top_k, h, 0);
}

size_t moe_backward_workspace_size_ex(int T, int d, int E, int top_k, int h, int h_shared) {
  if (T < 0 || d < 1 || E < 1 || top_k < 1 || h < 1 || h_shared < 0) return kStatusBytes;
  return carve_backward(nullptr, T, d, E, top_k, h, h_shared).bytes;
}

moe_status_t moe_forward_train_ex(const void* x, const void* w_router, const float* logits_in,
                                  const void* w1, const void* w3, const void* w2, int T, int d,
                                  int E, int top_k, int h, const moe_router_options_t* opts,
                                  const moe_shared_expert_t* shared, moe_dtype_t dt, void* out,
                                  void* state, size_t state_bytes, void* stream) {
  const moe_router_options_t o = opts ? *opts : default_options();
  if (moe_status_t st = check_train(T, d, E, top_k, h, o, dt)) return st;
  if (moe_status_t st = check_router(x, w_router, logits_in, T, d, E, top_k, o, dt,
                                     reinterpret_cast<int32_t*>(1), reinterpret_cast<float*>(1)))
    return st;
  if (moe_status_t st = check_shared(shared, T, d, dt)) return st;
  const int hs = shared ? shared->h : 0;
  if (T > 0) {
    MOE_CHECK_ARG(x && w1 && w3 && w2 && out, "x, w1, w3, w2, out are required");
    MOE_CHECK_ARG(aligned16(x) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                      aligned16(out),
                  "x, w1, w3, w2, out must be 16-byte aligned");
  }
  MOE_CHECK_ARG(state != nullptr, "state is required");
  const TrainState need = carve_train(nullptr, T, d, E, top_k, h, hs);
  if (state_bytes < need.bytes) {
    set_last_error("training state %zu < %zu", state_bytes, need.bytes);
    return MOE_ERR_WORKSPACE;
  }
  const TrainState t = carve_train(state, T, d, E, top_k, h, hs);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int N = T * top_k;
  const bool before = o.score_before_experts != 0;
  const DispatchPlan p = layer_dispatch_plan(T, d, E, top_k, 1, dt);
  cudaError_t e = cudaMemsetAsync(t.status, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = run_router(x, w_router, logits_in, T, d, E, top_k, o, dt, t.logits, t.idx, t.w, nullptr,
                   t.router_scratch, t.status, s, &p, static_cast<int32_t*>(t.disp_ws));
  if (e == cudaSuccess && logits_in && T > 0)   // the backward reads the logits from the state
    e = cudaMemcpyAsync(t.logits, logits_in, static_cast<size_t>(T) * E * sizeof(float),
                        cudaMemcpyDeviceToDevice, s);
  // [HP] MoE.forward with score_before_experts: the routed rows are scaled by
  // their weights (the state's x_perm holds the scaled rows)
  if (e == cudaSuccess)
    e = launch_dispatch(p, x, t.idx, d, dt, t.counts, t.offsets, t.src_row, t.dst_pos, t.x_perm,
                        t.disp_ws, t.status, s, /*hist_done=*/T > 0, before ? t.w : nullptr);
  if (e == cudaSuccess && N > 0)
    e = launch_swiglu_tc_train(t.x_perm, t.offsets, w1, w3, w2, N, d, h, E, t.y, t.H, t.GU,
                               t.status, s);
  // [HP] MoE.forward: shared_expert(x_flat), kept for its backward
  if (e == cudaSuccess && hs > 0 && T > 0) {
    e = launch_single_segment(t.offsets_s, T, s);
    if (e == cudaSuccess)
      e = launch_swiglu_tc_train(x, t.offsets_s, shared->w1, shared->w3, shared->w2, T, d, hs, 1,
                                 t.ys, t.Hs, t.GUs, t.status, s);
  }
  if (e == cudaSuccess)
    e = launch_combine(t.y, t.dst_pos, nullptr, before ? nullptr : t.w, T, d, N, top_k, dt, out,
                       s, hs > 0 ? t.ys : nullptr);
  return cuda_status(e, "moe_forward_train");
}

moe_status_t moe_forward_train(const void* x, const void* w_router, const float* logits_in,
                               const void* w1, const void* w3, const void* w2, int T, int d,
                               int E, int top_k, int h, const moe_router_options_t* opts,
                               moe_dtype_t dt, void* out, void* state, size_t state_bytes,
                               void* stream) {
  return moe_forward_train_ex(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, opts,
                              nullptr, dt, out, state, state_bytes, stream);
}

moe_status_t moe_backward_ex(const void* dout, const void* x, const void* w_router,
                             const void* w1, const void* w3, const void* w2, int T, int d, int E,
                             int top_k, int h, const moe_router_options_t* opts,
                             const moe_shared_expert_t* shared, moe_dtype_t dt,
                             const void* state, void* dx, float* d_logits, void* dw_router,
                             void* dw1, void* dw3, void* dw2, void* dws1, void* dws3, void* dws2,
                             void* ws, size_t ws_bytes, void* stream) {
  const moe_router_options_t o = opts ? *opts : default_options();
  if (moe_status_t st = check_train(T, d, E, top_k, h, o, dt)) return st;
  MOE_CHECK_ARG(std::isfinite(o.route_scale) && o.route_scale != 0.0f, "bad route_scale");
  MOE_CHECK_ARG(std::isfinite(o.aux_loss_coef), "aux_loss_coef must be finite");
  if (moe_status_t st = check_shared(shared, T, d, dt)) return st;
  const int hs = shared ? shared->h : 0;
  const bool before = o.score_before_experts != 0;
  MOE_CHECK_ARG(w1 && w3 && w2 && dw1 && dw3 && dw2, "w1, w3, w2, dw1, dw3, dw2 are required");
  MOE_CHECK_ARG(!dw_router || (x && w_router), "dw_router needs x and w_router");
  MOE_CHECK_ARG(!shared || (dws1 && dws3 && dws2 && x), "a shared expert needs x, dws1, dws3, dws2");
  MOE_CHECK_ARG(!before || x, "score_before_experts needs x");
  MOE_CHECK_ARG(aligned16(w1) && aligned16(w3) && aligned16(w2) && aligned16(dw1) &&
                    aligned16(dw3) && aligned16(dw2) && aligned16(dw_router) &&
                    aligned16(x) && aligned16(w_router) && aligned16(dws1) && aligned16(dws3) &&
                    aligned16(dws2),
                "weights, gradients and x must be 16-byte aligned");
  if (T > 0) {
    MOE_CHECK_ARG(dout && dx, "dout and dx are required");
    MOE_CHECK_ARG(aligned16(dout) && aligned16(dx), "dout, dx must be 16-byte aligned");
  }
  MOE_CHECK_ARG(state != nullptr && ws != nullptr, "state and ws are required");
  const BackwardWs need = carve_backward(nullptr, T, d, E, top_k, h, hs);
  if (ws_bytes < need.bytes) {
    set_last_error("backward workspace %zu < %zu", ws_bytes, need.bytes);
    return MOE_ERR_WORKSPACE;
  }
  const TrainState t = carve_train(const_cast<void*>(state), T, d, E, top_k, h, hs);
  const BackwardWs b = carve_backward(ws, T, d, E, top_k, h, hs);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int N = T * top_k;
  const bool gate = dw_router != nullptr;
  cudaError_t e = cudaMemsetAsync(b.status, 0, sizeof(int), s);
  if (N == 0) {
    const size_t wbytes = static_cast<size_t>(E) * h * d * 2;
    if (e == cudaSuccess) e = cudaMemsetAsync(dw1, 0, wbytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw3, 0, wbytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw2, 0, wbytes, s);
    if (e == cudaSuccess && gate) e = cudaMemsetAsync(dw_router, 0, static_cast<size_t>(E) * d * 2, s);
    if (shared) {
      const size_t sbytes = static_cast<size_t>(hs) * d * 2;
      if (e == cudaSuccess) e = cudaMemsetAsync(dws1, 0, sbytes, s);
      if (e == cudaSuccess) e = cudaMemsetAsync(dws3, 0, sbytes, s);
      if (e == cudaSuccess) e = cudaMemsetAsync(dws2, 0, sbytes, s);
    }
    return cuda_status(e, "moe_backward");
  }
  // combine -> experts -> (scaled dispatch) -> router -> shared expert ->
  // dispatch, all on `s`.  With score_before_experts the combine was
  // unweighted (its backward has no weight gradient) and the weights' gradient
  // comes from the scaled rows: d topk_w[t, j] = <dx_perm[p(t, j)], x[t]>.
  if (e == cudaSuccess)
    e = launch_combine_backward(dout, t.y, t.dst_pos, before ? nullptr : t.w, T, d, N, top_k, dt,
                                b.dY, before ? nullptr : b.dtw, s);
  if (e == cudaSuccess)
    e = launch_swiglu_bwd_tc(t.x_perm, t.offsets, w1, w3, w2, t.H, t.GU, b.dY, N, d, h, E, b.dXp,
                             dw1, dw3, dw2, b.dGU, b.status, s);
  if (e == cudaSuccess && before)
    e = launch_combine_backward(x, b.dXp, t.dst_pos, nullptr, T, d, N, top_k, dt, nullptr, b.dtw,
                                s);
  if (e == cudaSuccess)
    e = launch_router_backward(t.logits, t.idx, b.dtw, T, E, top_k,
                               o.score == MOE_SCORE_SIGMOID, o.renormalize, o.route_scale,
                               d_logits, gate ? b.dz16 : nullptr, s,
                               o.aux_loss_coef != 0.0f ? t.counts : nullptr,
                               lb_grad_scale(o.aux_loss_coef, E, T, top_k));
  if (e == cudaSuccess && gate)
    e = launch_gate_backward_tc(b.dz16, x, w_router, T, d, E, dw_router, b.dxr, b.off2, b.gpart,
                                b.status, s);
  // the shared expert: a one-segment grouped SwiGLU backward over every token
  // with the layer's upstream gradient
  if (e == cudaSuccess && hs > 0)
    e = launch_swiglu_bwd_tc(x, t.offsets_s, shared->w1, shared->w3, shared->w2, t.Hs, t.GUs,
                             dout, T, d, hs, 1, b.dXs, dws1, dws3, dws2, b.dGUs, b.status, s);
  // dx[t] = sum_j (w[t, j] with score_before_experts) dx_perm[p(t, j)] + the
  // router's share + the shared expert's share
  const void* add1 = gate ? b.dxr : (hs > 0 ? b.dXs : nullptr);
  const void* add2 = (gate && hs > 0) ? b.dXs : nullptr;
  if (e == cudaSuccess)
    e = launch_combine(b.dXp, t.dst_pos, nullptr, before ? t.w : nullptr, T, d, N, top_k, dt, dx,
                       s, add1, add2);
  return cuda_status(e, "moe_backward");
}

moe_status_t moe_backward(const void* dout, const void* x, const void* w_router, const void* w1,
                          const void* w3, const void* w2, int T, int d, int E, int top_k, int h,
                          const moe_router_options_t* opts, moe_dtype_t dt, const void* state,
                          void* dx, float* d_logits, void* dw_router, void* dw1, void* dw3,
                          void* dw2, void* ws, size_t ws_bytes, void* stream) {
  return moe_backward_ex(dout, x, w_router, w1, w3, w2, T, d, E, top_k, h, opts, nullptr, dt,
                         state, dx, d_logits, dw_router, dw1, dw3, dw2, nullptr, nullptr, nullptr,
                         ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ forward
size_t moe_forward_ex_workspace_size(int T, int d, int E, int top_k, int h, int ep_ranks,
                                     moe_dtype_t dt, int h_shared) {
  if (T < 0 || d < 1 || E < 1 || top_k < 1 || h < 1 || ep_ranks < 1 || E % ep_ranks ||
      h_shared < 0)
    return kStatusBytes;
  return carve_forward(nullptr, T, d, E, top_k, h, ep_ranks, dt, h_shared).bytes;
}

size_t moe_forward_workspace_size(int T, int d, int E, int top_k, int h, int ep_ranks,
                                  moe_dtype_t dt) {
  if (T < 0 || d < 1 || E < 1 || top_k < 1 || h < 1 || ep_ranks < 1 || E % ep_ranks)
    return kStatusBytes;
  return carve_forward(nullptr, T, d, E, top_k, h, ep_ranks, dt).bytes;
}

moe_status_t moe_forward_ex(const void* x, const void* w_router, const float* logits_in,
                            const void* w1, const void* w3, const void* w2, int T, int d, int E,
                            int top_k, int h, const moe_router_options_t* opts,
                            const moe_shared_expert_t* shared, int ep_ranks, moe_dtype_t dt,
                            void* out, float* logits_out, int32_t* topk_idx, float* topk_w,
                            int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  const moe_router_options_t o = opts ? *opts : default_options();
  const int hs = shared ? shared->h : 0;
  if (shared) {
    MOE_CHECK_ARG(hs >= 1, "shared->h=%d must be >= 1", hs);
    if (moe_status_t st = check_swiglu_shape(T, d, hs, 1, dt)) return st;
    if (T > 0) {
      MOE_CHECK_ARG(shared->w1 && shared->w3 && shared->w2,
                    "shared expert w1, w3, w2 are required");
      MOE_CHECK_ARG(aligned16(shared->w1) && aligned16(shared->w3) && aligned16(shared->w2),
                    "shared expert weights must be 16-byte aligned");
    }
  }
  if (moe_status_t st = check_router(x, w_router, logits_in, T, d, E, top_k, o, dt,
                                     reinterpret_cast<int32_t*>(1), reinterpret_cast<float*>(1)))
    return st;
  const int N = T * top_k;
  if (moe_status_t st = check_swiglu_shape(N, d, h, E, dt)) return st;
  if (o.capacity > 0 && (ep_ranks != 1 || dt != MOE_BF16)) {
    set_last_error("moe_forward_ex: the capacity policy needs ep_ranks = 1 and bf16");
    return MOE_ERR_UNSUPPORTED;
  }
  MOE_CHECK_ARG(ep_ranks >= 1 && E % ep_ranks == 0 && E * ep_ranks <= kMaxBins &&
                    1LL * ep_ranks * E <= kMaxSegments,
                "ep_ranks=%d must divide E with E*ep_ranks <= %d", ep_ranks, kMaxBins);
  if (T > 0) {
    MOE_CHECK_ARG(x && w1 && w3 && w2 && out, "x, w1, w3, w2, out are required");
    MOE_CHECK_ARG(aligned16(x) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                      aligned16(out),
                  "x, w1, w3, w2, out must be 16-byte aligned");
    if (moe_status_t st = check_rows(d, dt, "forward")) return st;
  }
  MOE_CHECK_ARG(ws != nullptr, "ws is required");
  const ForwardWs need = carve_forward(nullptr, T, d, E, top_k, h, ep_ranks, dt, hs);
  if (ws_bytes < need.bytes) {
    set_last_error("forward workspace %zu < %zu", ws_bytes, need.bytes);
    return MOE_ERR_WORKSPACE;
  }
  const ForwardWs f = carve_forward(ws, T, d, E, top_k, h, ep_ranks, dt, hs);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* idx = topk_idx ? topk_idx : f.idx;
  float* w = topk_w ? topk_w : f.w;
  const int R = ep_ranks;
  cudaError_t e = cudaMemsetAsync(f.status, 0, sizeof(int), s);
  const DispatchPlan p = layer_dispatch_plan(T, d, E, top_k, R, dt);
  // The router's top-k kernel also writes the dispatch histogram table,
  // unless the capacity policy changes the routing after it.
  const bool cap = o.capacity > 0;
  if (e == cudaSuccess)
    e = run_router(x, w_router, logits_in, T, d, E, top_k, o, dt, logits_out, idx, w, nullptr,
                   f.router_scratch, f.status, s, &p, static_cast<int32_t*>(f.disp_ws));
  if (e != cudaSuccess) return cuda_status(e, "moe_forward/router");
  int32_t* cnt_a = (R == 1 && counts) ? counts : f.counts_a;
  // The routed rows are materialised expert-major (single device) or
  // rank-major (simulated EP: what an all-to-all would deliver), then
  // regrouped.  Materialising costs one 16-byte-vector copy pass; measured
  // on B200 it is faster than gathering GEMM1's rows with TMA gather4
  // (moe_grouped_swiglu_gather), whose 512-byte requests limit the loads.
  // With score_before_experts the copy also scales each routed row by its
  // weight and the combine below is unweighted.
  const bool before = o.score_before_experts != 0;
  e = launch_dispatch(p, x, idx, d, dt, cnt_a, f.offsets_a, f.src_row, f.dst_pos, f.x_a,
                      f.disp_ws, f.status, s, /*hist_done=*/T > 0 && !cap, before ? w : nullptr);
  if (e != cudaSuccess) return cuda_status(e, "moe_forward/dispatch");
  const void* xe = f.x_a;
  const int32_t* off = f.offsets_a;
  const int32_t* row_map = nullptr;
  if (R > 1) {
    int32_t* cem = counts ? counts : f.counts_em;
    e = launch_regroup(f.x_a, f.counts_a, R, R, E / R, N, d, dt, f.x_em, cem, f.offsets_em,
                       f.perm, f.perm_inv, f.reg_ws, f.status, s);
    if (e != cudaSuccess) return cuda_status(e, "moe_forward/regroup");
    xe = f.x_em;
    off = f.offsets_em;
    row_map = f.perm_inv;
  }
  // with the capacity policy the kept copies fill the first offsets[E] < N
  // slots
  e = N == 0 ? cudaSuccess
             : cap ? launch_swiglu_tc(xe, off, w1, w3, w2, nullptr, N, d, h, E, f.y, f.H,
                                      f.status, s, /*rows_upto=*/true)
                   : run_swiglu(xe, off, w1, w3, w2, nullptr, N, d, h, E, dt, f.y, f.H, f.status,
                                s);
  if (e != cudaSuccess) return cuda_status(e, "moe_forward/grouped_swiglu");
  // [HP] MoE.forward: shared_expert(x_flat), added to the routed output in
  // the combine.
  if (hs > 0 && T > 0) {
    e = launch_single_segment(f.offsets_s, T, s);
    if (e == cudaSuccess)
      e = run_swiglu(x, f.offsets_s, shared->w1, shared->w3, shared->w2, nullptr, T, d, hs, 1,
                     dt, f.y_s, f.H_s, f.status, s);
    if (e != cudaSuccess) return cuda_status(e, "moe_forward/shared_expert");
  }
  e = launch_combine(f.y, f.dst_pos, row_map, before ? nullptr : w, T, d, N, top_k, dt, out, s,
                     hs > 0 ? f.y_s : nullptr);
  return cuda_status(e, "moe_forward/combine");
}

moe_status_t moe_forward(const void* x, const void* w_router, const float* logits_in,
                         const void* w1, const void* w3, const void* w2, int T, int d, int E,
                         int top_k, int h, moe_score_t score, int renormalize, int ep_ranks,
                         moe_dtype_t dt, void* out, float* logits_out, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                         void* stream) {
  moe_router_options_t o = default_options();
  o.score = score;
  o.renormalize = renormalize;
  return moe_forward_ex(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, &o, nullptr,
                        ep_ranks, dt, out, logits_out, topk_idx, topk_w, counts, ws, ws_bytes,
                        stream);
}

}  // extern "C"
