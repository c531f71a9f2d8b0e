// Fused tcgen05 router of libmoe: the gate contraction, the scores, the top-k
// selection and the routing weights in one kernel ([HP]
// TokenChoiceTopKRouter.forward: the gate in fp32, softmax or sigmoid,
// topk, gather, optional renormalisation, route_scale, expert_bias).
//
// A tile of 128 tokens is computed by a cluster of C CTAs (C = 1, 2, 4 or 8,
// chosen so that tiles x C come close to the SM count): CTA r of the cluster
// accumulates the r-th K range of d into TMEM (tcgen05.mma, operands staged
// by TMA).  The C partial logit tiles are reduced through distributed shared
// memory, not HBM: CTA r owns token rows [r 128 / C, (r + 1) 128 / C) of the
// tile, every CTA stores its partial rows into their owner's shared memory
// (st.shared::cluster), and the owner adds the C partials in rank order (a
// fixed order: the logits do not depend on timing or on the grid; each
// warp stages its rows so that the remote stores write whole 128-byte row
// pieces).  The owner's 128 epilogue threads, C per token, then select the
// k winners (sorted register lists of each thread's experts merged by k
// shuffle arg-max rounds: descending key, ties to the lower expert index)
// and write the indices and weights; in the
// layer forward the CTA also writes the dispatch histogram of its token
// blocks.  The expert counts of the entry
// point go through a per-CTA table that a second small kernel sums.  The
// stage memory is sized so that two CTAs fit on an SM (for E <= 128): twice
// the loads in flight and twice the scoring threads per SM.
//
// Every mbarrier wait is bounded (2 s) and unwinds by setting
// MOE_DEV_TIMEOUT; the control flow after the K loop is the same in every
// CTA (no early exit), so the cluster and named barriers are always met.
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace rtc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;          // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
// Pipeline stages: 96 KB for E <= 128 (two CTAs per SM), 192 KB for the
// 256-column accumulator (whose exchange buffer needs 133 KB).  After the K
// loop the same memory (at least `region` bytes, see Args) holds the partial
// logits of the cluster, the dispatch bins and the expert bins.
template <int BN>
struct Layout {
  static constexpr int kStageBytes = BM * BK * 2 + BN * BK * 2;
  static constexpr int kStages = BN <= 64 ? 4 : BN == 128 ? 3 : 4;
  static constexpr int kStageRegion = kStages * kStageBytes;
  static constexpr uint32_t kTmemCols = BN < 32 ? 32u : static_cast<uint32_t>(BN);
  static constexpr int kNumBars = 2 * kStages + 1;
  static constexpr int kTailBytes = kNumBars * 8 + 16;   // barriers, TMEM slot, abort flag
};

struct Args {
  int T, d, E, k, renorm;
  int C;                 // CTAs per tile (cluster size)
  int kb_total;          // 64-wide K blocks of d
  int kb_per_cta;        // K blocks of each CTA of a cluster
  int pitch;             // fp32 pitch of a row of partial logits in shared memory
  int region;            // bytes before the barriers: max(stages, exchange + bins)
  RouterOptions opt;
  float* logits_out;     // [T, E] or null
  int32_t* topk_idx;     // [T, k]
  float* topk_w;         // [T, k]
  int32_t* counts_part;  // [grid, E] per-CTA expert histograms, or null
  int clear_status;      // the kernel is its call's only status writer: clear it
  float* tpe;            // tokens_per_expert [E] (+=) or null
  float* lb;             // [2E] copies and weight sums per expert (+=) or null
  int32_t* blk;          // dispatch histogram table [nbins, nblk] or null
  int nbins, tb, nblk, R, L, S;
  int* status;
};

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void bar_epi() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// floats of one epilogue warp's 32 x 32 staging tile of the exchange (padded rows)
constexpr int kXchgTile = 32 * 33;

// Sorted list of the KM largest (key, expert) pairs a thread has seen, key
// descending; a thread meets its experts in ascending order, so an equal key
// never displaces an entry (ties go to the lower expert).
template <int KM>
__device__ __forceinline__ void topk_insert(int (&kk)[KM], int (&ee)[KM], float (&vv)[KM], int key,
                                            int e, float v) {
  if (key <= kk[KM - 1]) return;
#pragma unroll
  for (int j = KM - 1; j >= 0; --j) {
    if (kk[j] < key) {
      if (j > 0 && kk[j - 1] < key) {
        kk[j] = kk[j - 1];
        ee[j] = ee[j - 1];
        vv[j] = vv[j - 1];
      } else {
        kk[j] = key;
        ee[j] = e;
        vv[j] = v;
      }
    }
  }
}

// Logits of experts 4j .. 4j+3 of a token: its C partial rows (rank r at
// row + r rstride) added in rank order.
__device__ __forceinline__ float4 partial_sum4(const float* row, size_t rstride, int C, int j) {
  float4 z = *reinterpret_cast<const float4*>(row + 4 * j);
  for (int r = 1; r < C; ++r) {
    const float4 q = *reinterpret_cast<const float4*>(row + r * rstride + 4 * j);
    z.x += q.x;
    z.y += q.y;
    z.z += q.z;
    z.w += q.w;
  }
  return z;
}

__device__ __forceinline__ float f4_at(const float4& v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// Scores, top-k and weights of the tokens a CTA owns, on its 128 epilogue
// threads: G = 128 / own threads per token (G = C), thread g taking the
// expert quads g, g + G, ... of the token's row.  Each thread keeps the KM
// best (key, expert) pairs of its experts; k rounds of a G-way arg-max
// (xor shuffles on (key descending, expert ascending)) merge them.  The
// partial-logit rows are read as 16-byte vectors; the row pitch
// (4 G mod 32 floats) puts the eight threads of each load phase on distinct
// banks.  Arithmetic: z = partials in rank order; max and denominator over
// the experts of a thread in ascending order, then across the G threads by
// the xor butterfly; the renormalising sum over the winners in rank order.
template <int KM>
__device__ __forceinline__ void score_owned(const Args& a, const float* recv, int own, int C,
                                            int t_own0, int* tok_e, float* tok_w, int* ebins,
                                            float* wsum) {
  const int i = static_cast<int>(threadIdx.x) - 64;
  const int G = BM / own;
  const int it = i / G, g = i - it * G;
  const int t = t_own0 + it;
  const bool live = t < a.T;   // the G threads of a token agree; every thread takes part
  const int E = a.E, k = a.k;
  const RouterOptions& opt = a.opt;
  const bool on_logits = opt.bias == nullptr && opt.scale > 0.f;
  const size_t rstride = static_cast<size_t>(own) * a.pitch;
  const float* row = recv + static_cast<size_t>(it) * a.pitch;
  const int nq = (E + 3) >> 2;

  // Softmax scores as keys (bias or a non-positive scale): the maximum and
  // the denominator first.
  float mx = -INFINITY, den = 1.f;
  if (!on_logits && !opt.sigmoid) {
    for (int j = g; j < nq; j += G) {
      const float4 z4 = partial_sum4(row, rstride, C, j);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float z = f4_at(z4, c);
        if (4 * j + c < E && z == z) mx = fmaxf(mx, z);
      }
    }
    for (int sh = 1; sh < G; sh <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
    float dn = 0.f;
    for (int j = g; j < nq; j += G) {
      const float4 z4 = partial_sum4(row, rstride, C, j);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float z = f4_at(z4, c);
        if (z != z) z = -INFINITY;
        if (4 * j + c < E) dn += expf(z - mx);
      }
    }
    for (int sh = 1; sh < G; sh <<= 1) dn += __shfl_xor_sync(0xffffffffu, dn, sh);
    den = dn;
  }

  // selection: every expert of the thread into its sorted list; a winner
  // carries its logit (keys on the logits) or its score
  int kk[KM], ee[KM];
  float vv[KM];
#pragma unroll
  for (int q = 0; q < KM; ++q) {
    kk[q] = INT_MIN;
    ee[q] = INT_MAX;
    vv[q] = 0.f;
  }
  for (int j = g; j < nq; j += G) {
    const float4 z4 = partial_sum4(row, rstride, C, j);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      const int e = 4 * j + c;
      if (e >= E) break;
      float z = f4_at(z4, c);
      if (a.logits_out && live) a.logits_out[static_cast<size_t>(t) * E + e] = z;
      if (z != z) z = -INFINITY;
      float kv = z, v = z;
      if (!on_logits) {
        v = opt.sigmoid ? 1.0f / (1.0f + expf(-z)) : expf(z - mx);
        kv = v / den * opt.scale;
        if (opt.bias) {
          kv += opt.bias[e];
          if (kv != kv) kv = -INFINITY;
        }
      }
      topk_insert<KM>(kk, ee, vv, score_key(kv), e, v);
    }
  }

  // merge: round r takes the best head of the G lists and pops it; the
  // winner's expert goes to tok_e and its unbiased score to tok_w (with keys
  // on the logits: the softmax numerator exp(z - max z), max z being the
  // first winner's logit, or sigmoid(z)); sel sums them in round order
  float sel = 0.f;
  for (int r = 0; r < k; ++r) {
    int bk = kk[0], be = ee[0];
    float bv = vv[0];
    for (int sh = 1; sh < G; sh <<= 1) {
      const int ok = __shfl_xor_sync(0xffffffffu, bk, sh);
      const int oe = __shfl_xor_sync(0xffffffffu, be, sh);
      const float ov = __shfl_xor_sync(0xffffffffu, bv, sh);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
        bv = ov;
      }
    }
    if (ee[0] == be) {
#pragma unroll
      for (int q = 0; q + 1 < KM; ++q) {
        kk[q] = kk[q + 1];
        ee[q] = ee[q + 1];
        vv[q] = vv[q + 1];
      }
      kk[KM - 1] = INT_MIN;
      ee[KM - 1] = INT_MAX;
    }
    if (on_logits) {
      if (r == 0) mx = bv;
      bv = opt.sigmoid ? 1.0f / (1.0f + expf(-bv)) : expf(bv - mx);
    }
    sel += bv;
    if (g == 0) {
      tok_e[it * k + r] = be;
      tok_w[it * k + r] = bv;
    }
  }
  // softmax with keys on the logits: the denominator when it is asked for
  if (on_logits && !opt.sigmoid && (!a.renorm || opt.scores_out)) {
    float dn = 0.f;
    for (int j = g; j < nq; j += G) {
      const float4 z4 = partial_sum4(row, rstride, C, j);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float z = f4_at(z4, c);
        if (z != z) z = -INFINITY;
        if (4 * j + c < E) dn += expf(z - mx);
      }
    }
    for (int sh = 1; sh < G; sh <<= 1) dn += __shfl_xor_sync(0xffffffffu, dn, sh);
    den = dn;
  }
  __syncwarp();
  // weights: the winners' scores (renormalised), times the scale; thread g
  // writes the winners r = g, g + G, ...
  if (live) {
    for (int r = g; r < k; r += G) {
      const size_t o = static_cast<size_t>(t) * k + r;
      const int e = tok_e[it * k + r];
      const float wx = tok_w[it * k + r];
      const float wv = wx / (a.renorm ? sel : den) * opt.scale;
      a.topk_idx[o] = e;
      a.topk_w[o] = wv;
      if (opt.scores_out) opt.scores_out[o] = wx / den;
      atomicAdd(&ebins[e], 1);
      if (a.lb) atomicAdd(&wsum[e], wv);
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmW, const Args a) {
  using Lay = Layout<BN>;
  constexpr int STAGES = Lay::kStages;
  constexpr int kABytes = BM * BK * 2;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.region);
  uint64_t* empty = full + STAGES;
  uint64_t* mma_done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = a.C;
  const int rank = static_cast<int>(cluster_ctarank());
  const int tile = blockIdx.x / C;
  const int own = BM / C;                       // token rows this CTA owns
  const int kb0 = rank * a.kb_per_cta;
  const int kb1 = min(a.kb_total, kb0 + a.kb_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  pdl_wait();   // x may be written by the previous kernel
  // When this kernel is its call's only writer of the status word, CTA 0
  // clears it here (a wait can give up only 2 s after its CTA started).
  if (a.clear_status && blockIdx.x == 0 && threadIdx.x == 0) *a.status = 0;
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ------------------------------------------------------------ K loop
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, a.status)) break;
        uint8_t* sa = smem + stage * Lay::kStageBytes;
        mbar_arrive_expect_tx(full + stage, Lay::kStageBytes);
        tma_load_2d(sa, &tmX, full + stage, kb * BK, tile * BM, pol);
        tma_load_2d(sa + kABytes, &tmW, full + stage, kb * BK, 0, pol);
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // drain: every issued load has landed before the stage memory is reused
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < min(issued, STAGES); ++i) {
        if (s == 0) {
          s = STAGES - 1;
          ph ^= 1u;
        } else {
          --s;
        }
        mbar_wait(full + s, ph, nullptr, a.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full + stage, phase, abort_flag, a.status)) break;
        tc_fence_after();
        const uint8_t* sa = smem + stage * Lay::kStageBytes;
        const uint64_t ad = sw128_kmajor_desc(sa);
        const uint64_t bd = sw128_kmajor_desc(sa + kABytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma_bf16(tmem_base, ad + 2u * kk, bd + 2u * kk, IDESC, (kb != kb0 || kk != 0) ? 1u : 0u);
        tc_commit(empty + stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, a.status);
    }
  } else {
    if (lane == 0) mbar_wait(mma_done, 0, nullptr, a.status);
    __syncwarp();
    tc_fence_after();
  }
  __syncwarp();
  pdl_trigger();
  // #1: every CTA of the cluster is done with its MMAs and loads, so the
  // stage memory may now receive the partial logits of the peers.
  cluster_sync_all();

  // ------------------------------------------------- partial-logit exchange
  // Each epilogue warp moves its 32 rows in 32 x 32 chunks: TMEM -> its
  // staging tile in local shared memory (lane = row) -> read back so that 8
  // lanes hold one row's 32 columns -> 16-byte remote stores that write 4
  // whole 128-byte row pieces per instruction.
  float* recv = reinterpret_cast<float*>(smem);   // [C][own][pitch]
  const int pitch = a.pitch;
  if (warp >= 2) {
    const int q = warp & 3;
    float* stg = reinterpret_cast<float*>(smem + align_up(static_cast<size_t>(BM) * pitch * 4, 16)) +
                 (warp - 2) * kXchgTile;        // [32][33]
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int sub = lane >> 3, c4 = (lane & 7) * 4;
    uint32_t dst_row[8];                          // remote address of the row each pass writes
#pragma unroll
    for (int pss = 0; pss < 8; ++pss) {
      const int row = q * 32 + 4 * pss + sub;
      const int o = row / own, lr = row - o * own;
      dst_row[pss] = cluster_map(recv, static_cast<uint32_t>(o)) +
                     static_cast<uint32_t>((rank * own + lr) * pitch + c4) * 4u;
    }
    for (int c = 0; c * 32 < a.E; ++c) {
      uint32_t v[32];
      tmem_ld32(taddr + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) stg[lane * 33 + j] = __uint_as_float(v[j]);
      __syncwarp();
#pragma unroll
      for (int pss = 0; pss < 8; ++pss) {
        const float* src = stg + (4 * pss + sub) * 33 + c4;
        st_cluster_v4(dst_row[pss] + static_cast<uint32_t>(c * 32 * 4), __float_as_uint(src[0]),
                      __float_as_uint(src[1]), __float_as_uint(src[2]), __float_as_uint(src[3]));
      }
      __syncwarp();
    }
    tc_fence_before();
  }
  __syncwarp();
  // #2: the partials of every CTA are in their owners' shared memory
  cluster_sync_all();

  // --------------------------------------------------- scores and top-k
  // The 128 epilogue threads score the owned tokens (score_owned); warps 0
  // and 1 wait at the barrier below.
  const int i = threadIdx.x - 64;                 // epilogue threads: 0..127
  const int E = a.E, k = a.k;
  int* dbins = reinterpret_cast<int*>(smem + align_up(static_cast<size_t>(BM) * pitch * 4, 16));
  int* ebins = dbins + (a.blk ? a.nbins : 0);
  float* wsum = reinterpret_cast<float*>(ebins + E);
  int* tok_e = reinterpret_cast<int*>(wsum + E);   // [own][k] winners, for the histograms
  float* tok_w = reinterpret_cast<float*>(tok_e + BM * kMaxTopK);   // [own][k] their scores
  const int t_own0 = tile * BM + rank * own;
  for (int e = threadIdx.x; e < E; e += kThreads) {
    ebins[e] = 0;
    wsum[e] = 0.f;
  }
  __syncthreads();
  if (warp >= 2) {
    if (a.k <= 4)
      score_owned<4>(a, recv, own, C, t_own0, tok_e, tok_w, ebins, wsum);
    else if (a.k <= 8)
      score_owned<8>(a, recv, own, C, t_own0, tok_e, tok_w, ebins, wsum);
    else
      score_owned<16>(a, recv, own, C, t_own0, tok_e, tok_w, ebins, wsum);
  }
  __syncthreads();   // the winners of every owned token are in tok_e
  if (warp >= 2) {
    // dispatch histogram of every token block of tb rows this CTA owns
    if (a.blk) {
      if (blockIdx.x == 0 && i == 0)   // the dispatch column scan's ticket
        a.blk[static_cast<size_t>(a.nbins) * a.nblk] = 0;
      const int nb = own / a.tb;
      for (int jb = 0; jb < nb; ++jb) {
        const int b = t_own0 / a.tb + jb;
        for (int x = i; x < a.nbins; x += 128) dbins[x] = 0;
        bar_epi();
        // the copies of the block's tb tokens, one per thread
        for (int c = i; c < a.tb * k; c += 128) {
          const int it = jb * a.tb + c / k;
          const int t = t_own0 + it;
          if (t < a.T) atomicAdd(&dbins[dispatch_key(tok_e[it * k + c % k], t, a.R, a.L, a.S)], 1);
        }
        bar_epi();
        if (b < a.nblk)
          for (int x = i; x < a.nbins; x += 128)
            a.blk[static_cast<size_t>(x) * a.nblk + b] = dbins[x];
        bar_epi();
      }
    }
    bar_epi();
    for (int e = i; e < E; e += 128) {
      const int c = ebins[e];
      if (a.counts_part) a.counts_part[static_cast<size_t>(blockIdx.x) * E + e] = c;
      if (c) {
        if (a.tpe) atomicAdd(&a.tpe[e], static_cast<float>(c));
        if (a.lb) {
          atomicAdd(&a.lb[e], static_cast<float>(c));
          atomicAdd(&a.lb[E + e], wsum[e]);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

// counts[e] = sum over the CTAs of the fused router of their histograms
// (plain stores: counts needs no clearing).
__global__ void router_counts_kernel(const int32_t* __restrict__ part, int G, int E,
                                     int32_t* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
    int c = 0;
    for (int g = 0; g < G; ++g) c += part[static_cast<size_t>(g) * E + e];
    counts[e] = c;
  }
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& tx, const CUtensorMap& tw, const Args& a, int grid,
                      size_t smem, cudaStream_t s) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, router_tc_kernel<BN>, tx, tw, a);
}

}  // namespace rtc

RouterFusedPlan router_fused_plan(int T, int d, int E, const DispatchPlan* plan) {
  // (the plan only adds its bins to the shared memory; C does not depend on it)
  RouterFusedPlan p{};
  p.bn = E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
  p.tiles = std::max(1, cdiv(T, rtc::BM));
  p.kb_total = std::max(1, cdiv(d, rtc::BK));
  // the row pitch is (E rounded up to 32) + 4 C mod 32 floats (conflict-free
  // 16-byte reads in score_owned); the memory is sized for the widest one
  const int pitch_max = (E + 31) / 32 * 32 + 16;
  // shared memory: the stages, or after the K loop the partial logits of the
  // cluster, the dispatch bins and the expert bins, whichever is larger
  int stages = 0, tail = 0;
  switch (p.bn) {
    case 32: stages = rtc::Layout<32>::kStageRegion; tail = rtc::Layout<32>::kTailBytes; break;
    case 64: stages = rtc::Layout<64>::kStageRegion; tail = rtc::Layout<64>::kTailBytes; break;
    case 128: stages = rtc::Layout<128>::kStageRegion; tail = rtc::Layout<128>::kTailBytes; break;
    default: stages = rtc::Layout<256>::kStageRegion; tail = rtc::Layout<256>::kTailBytes; break;
  }
  // (during the exchange the four epilogue warps' staging tiles sit where
  // the bins go afterwards)
  const size_t recv = align_up(static_cast<size_t>(rtc::BM) * pitch_max * 4, 16);
  const size_t exch = recv + std::max<size_t>(
                                 4 * rtc::kXchgTile * 4,
                                 (plan ? static_cast<size_t>(plan->nbins) * 4 : 0) +
                                     8 * static_cast<size_t>(E) +
                                     static_cast<size_t>(rtc::BM) * kMaxTopK * 8);
  p.region = static_cast<int>(align_up(std::max<size_t>(stages, exch), 1024));
  p.smem = p.region + tail + 1024;   // + slack for the 1 KB alignment
  // two CTAs per SM when they fit (228 KB per SM, 1 KB reserved per CTA)
  const int per_sm = p.smem + 1024 <= 114 * 1024 ? 2 : 1;
  // clusters of C CTAs per tile: tiles x C close to what the SMs hold at
  // once and every CTA with at least one K block.  C depends on the sizes
  // only, so the logits (summed over the C partials in rank order) are the
  // same with and without the EP layout; the layer's dispatch plan is made
  // with blocks of at most 128 / C tokens (layer_dispatch_plan).
  int C = 1;
  while (C < 8 && p.tiles * C * 2 <= per_sm * kRouterTargetTiles && 2 * C <= p.kb_total) C *= 2;
  while (C > 1 && (C - 1) * cdiv(p.kb_total, C) >= p.kb_total) C /= 2;
  p.C = C;
  p.pitch = (E + 31) / 32 * 32 + (4 * C) % 32;
  p.kb_per_cta = cdiv(p.kb_total, C);
  p.grid = p.tiles * C;
  p.ok = p.smem <= 227 * 1024 && (!plan || rtc::BM / C >= plan->tb);
  return p;
}

cudaError_t launch_router_fused(const void* x, const void* w_router, int T, int d, int E,
                                int top_k, int renorm, const RouterOptions& o, float* logits_out,
                                int32_t* topk_idx, float* topk_w, int32_t* counts,
                                int32_t* counts_part, float* tokens_per_expert, float* lb,
                                const DispatchPlan* plan, int32_t* blk, int* status,
                                bool clear_status, cudaStream_t s) {
  const RouterFusedPlan p = router_fused_plan(T, d, E, plan);
  if (!p.ok) return cudaErrorInvalidValue;
  CUtensorMap tx, tw;
  if (!tc::make_tmap(&tx, x, d, T, rtc::BM)) return cudaErrorInvalidValue;
  if (!tc::make_tmap(&tw, w_router, d, E, p.bn)) return cudaErrorInvalidValue;
  rtc::Args a{};
  a.T = T;
  a.d = d;
  a.E = E;
  a.k = top_k;
  a.renorm = renorm;
  a.C = p.C;
  a.kb_total = p.kb_total;
  a.kb_per_cta = p.kb_per_cta;
  a.pitch = p.pitch;
  a.region = p.region;
  a.opt = o;
  a.logits_out = logits_out;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts_part = counts ? counts_part : nullptr;
  a.clear_status = clear_status ? 1 : 0;
  a.tpe = tokens_per_expert;
  a.lb = lb;
  a.blk = plan ? blk : nullptr;
  if (plan) {
    a.nbins = plan->nbins;
    a.tb = plan->tb;
    a.nblk = plan->nblk;
    a.R = plan->R;
    a.L = plan->L;
    a.S = plan->S;
  } else {
    a.nbins = 0;
    a.tb = 1;
    a.nblk = 0;
    a.R = 1;
    a.L = E;
    a.S = T;
  }
  a.status = status;
  cudaError_t e;
  switch (p.bn) {
    case 32: e = rtc::launch_bn<32>(tx, tw, a, p.grid, p.smem, s); break;
    case 64: e = rtc::launch_bn<64>(tx, tw, a, p.grid, p.smem, s); break;
    case 128: e = rtc::launch_bn<128>(tx, tw, a, p.grid, p.smem, s); break;
    default: e = rtc::launch_bn<256>(tx, tw, a, p.grid, p.smem, s); break;
  }
  if (e == cudaSuccess && counts) {
    launch_k(rtc::router_counts_kernel, dim3(cdiv(E, 256)), dim3(256), 0, s, counts_part, p.grid,
             E, counts);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace moe

namespace moe {

DispatchPlan layer_dispatch_plan(int T, int d, int E, int top_k, int R, moe_dtype_t dt) {
  int max_tb = 128;
  if (dt == MOE_BF16 && E <= 256 && T > 0) max_tb = rtc::BM / router_fused_plan(T, d, E, nullptr).C;
  return make_dispatch_plan(T, E, top_k, R, max_tb);
}

}  // namespace moe
