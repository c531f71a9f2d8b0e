// tcgen05 (5th-generation tensor core) GEMMs of the MoE layer on sm_100a.
//
// One warp-specialised, persistent kernel skeleton serves three problems:
//   * the router        fp32 partial logits of x[T, d] . w_router[E, d]^T,
//                       split over d so that the (token tile, K split) tiles
//                       fill the SMs; router_topk_kernel adds the splits
//                       ([HP] TokenChoiceTopKRouter.forward, the gate);
//   * GEMM1 (up)        for every expert segment, one 128 x 256 accumulator
//                       holds x . w1^T (columns 0..127) and x . w3^T
//                       (columns 128..255) for the same 128 hidden units; the
//                       epilogue writes H = silu(G) * U in bf16
//                       ([HP] _run_experts_for_loop, silu(x w1^T) * (x w3^T));
//   * GEMM2 (down)      y = H . w2^T (times an optional row scale).
//
// Roles (192 threads): warp 0 issues TMA loads into a STAGES-deep ring of
// shared-memory stages, warp 1 allocates TMEM and issues tcgen05.mma from one
// thread, warps 2..5 drain the accumulator (tcgen05.ld) and write results
// (the gathered GEMM1 adds four cp.async gather warps).  Two TMEM
// accumulators let the epilogue of tile i overlap the MMAs of tile i + 1.
// Tiles are 128 rows (BM) x BN columns, K in steps of 64 bf16 (one 128-byte
// swizzle row).  The expert tile schedule is built on the device from the
// offsets array: no host synchronisation, no per-expert launches.  Tiles of
// one expert that share a weight tile are adjacent in the schedule, so the
// CTAs that read the same weight tile run at the same time and the second
// read hits L2.
//
// On B200 these kernels are bound by the delivery of operand tiles from L2
// to shared memory (about 100 GB/s per SM), not by DRAM or the tensor pipe:
// each 64-wide K block of a 128 x 256 tile moves 48 KB for 512 MMA cycles.
//
// Every mbarrier wait is bounded (2 s), sets MOE_DEV_TIMEOUT and unwinds;
// the kernel then waits (bounded) for its own loads and MMAs and frees TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kATileBytes = BM * BK * 2;   // 16 KB
constexpr int kSmemBudget = 200 * 1024;    // stages; the rest is barriers + schedule

struct TileInfo {
  int a_row;     // first A row (token or routed copy)
  int b_row;     // first B row in the [E * n, K] view of the weights
  int m_valid;   // rows of this tile that belong to the problem / expert
  int n0;        // first output column (router: the K split)
  int kb0, kb1;  // K blocks [kb0, kb1) of this tile
  int m0;        // weight-gradient tiles: first output row (A column)
};

// A grouped tile with few valid rows (an expert's last rows, or decode) is
// a plain 128-row tile.  (Swap-AB tiles -- the weight halves of the B stage
// as the MMA's M = 128 operand, the tile's tokens as N -- were measured on
// B200: no faster for decode, whose grouped GEMMs stream every weight once
// at the HBM copy rate either way, and 2-6 % slower for segment tails at the
// gpt-oss EP8 sizes: small-N MMAs do not run proportionally faster.)

struct Args {
  int M;                     // rows of A: T (router) or N (grouped)
  int K;                     // reduction length
  int E;
  int n_out;                 // output columns: E (router), h (up), d (down)
  const int32_t* offsets;    // [E+1] expert segments (grouped)
  int* status;
  // router
  float* logits_part;        // [ksplit, T, E] fp32 partial logits
  int ksplit;                // number of K splits
  int kb_per_split;          // K blocks per split
  // grouped
  __nv_bfloat16* out;        // H [N, h] (up) or y [N, d] (down)
  const int32_t* src_row;    // gathered GEMM1: token of every expert-major slot
  int src_rows;              // gathered GEMM1: rows of x (T)
  const void* gather_src;    // gathered GEMM1: x [T, K]
  const float* row_scale;    // down only, may be null
  // training forward: GEMM1 also keeps its two products for the backward
  __nv_bfloat16* gu_out;     // [N, 2h]: G = x w1^T in columns [0, h), U = x w3^T in [h, 2h)
  // backward
  const __nv_bfloat16* gu_in;  // [N, 2h] the saved G | U (data gradient of GEMM2)
  __nv_bfloat16* out1;       // weight gradient: output rows >= split of each expert
  int split;                 // weight gradient: rows of each expert that go to `out`
  int Ma;                    // weight gradient: output rows per expert
  float* out_f32;            // weight gradient: fp32 output [E, Ma, n_out] instead of bf16
  // Which rows of each expert segment a grouped launch covers (see
  // pair_head): 0 all of them, 1 the head (CTA-pair launch), 2 the tail
  // (single-CTA launch).
  int seg_part;
  // Grouped launches: offsets[E] may be below M (rows past it are copies the
  // capacity policy dropped, left uncomputed); else it must equal M.
  int rows_upto;
  // GEMM2 with the combine folded in (CTA-pair kernel): output row s is
  // scaled by comb_w[s] and added into comb_out[comb_tok[s]] with fp32
  // reductions instead of being stored
  float* comb_out;           // [comb_T, n_out] fp32, zero before the launch
  const int32_t* comb_tok;   // [M] token of every slot (outside [0, comb_T): skipped)
  const float* comb_w;       // [M] routing weight of every slot
  int comb_T;
};

__host__ __device__ constexpr int stages_for(int bn) {
  return (kSmemBudget / (kATileBytes + bn * BK * 2)) > 8 ? 8
                                                          : (kSmemBudget / (kATileBytes + bn * BK * 2));
}
__host__ __device__ constexpr uint32_t tmem_cols_for(int bn) {
  return (2 * bn <= 32) ? 32u : (2 * bn <= 64) ? 64u : (2 * bn <= 128) ? 128u
                                                     : (2 * bn <= 256) ? 256u : 512u;
}

// ---------------------------------------------------------------- policies
// Router: A = x [T, d], B = w_router [E, d] (rows >= E are zero-filled by
// TMA).  A tile is 128 tokens x one slice of the reduction: d is split into
// `ksplit` ranges so that there are about as many tiles as SMs even for a
// few hundred tokens, and each tile writes its fp32 partial logits to
// logits_part[split][t][0..E).  router_topk_kernel adds the splits in a fixed
// order and does softmax / top-k, one warp per token.
template <int BN_>
struct RouterPolicy {
  static constexpr int BN = BN_;
  static constexpr int NUM_B = 1;
  static constexpr bool GATHER_A = false;
  static constexpr bool A_MN = false, B_MN = false, MASK_K = false, CUSTOM_LOADS = false;
  static constexpr int EPI_STAGE_BYTES = 0;   // shared staging of the epilogue warps
  static constexpr int EPI_WARPS = 4;         // one per TMEM lane quadrant
  static __device__ int k_rows(const TileInfo&, int) { return BK; }
  static constexpr int THREADS = kThreads;
  static constexpr int SCHED_INTS = 8;

  static __device__ void prologue(const Args&, int*) {}
  static __device__ int num_tiles(const Args& a, const int*) { return cdiv(a.M, BM) * a.ksplit; }
  static __device__ TileInfo tile_info(const Args& a, const int*, int tile) {
    const int mt = tile / a.ksplit;
    const int sp = tile - mt * a.ksplit;
    TileInfo t;
    t.a_row = mt * BM;
    t.b_row = 0;
    t.m_valid = min(BM, a.M - t.a_row);
    t.n0 = sp;
    t.kb0 = sp * a.kb_per_split;
    t.kb1 = min(cdiv(a.K, BK), t.kb0 + a.kb_per_split);
    return t;
  }
  static __device__ void epilogue(const Args& a, int*, const TileInfo& ti, uint32_t taddr,
                                  int row) {
    const int E = a.E;
    const bool valid = row < ti.m_valid;
    float* dst = a.logits_part + (static_cast<size_t>(ti.n0) * a.M + ti.a_row + row) * E;
    const bool vec = (E % 4) == 0;
    const int nch = cdiv(E, 32);
    for (int c = 0; c < nch; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      if (!valid) continue;
      if (vec && c * 32 + 32 <= E) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<float4*>(dst + c * 32)[q] =
              make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                          __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (c * 32 + q < E) dst[c * 32 + q] = __uint_as_float(r[q]);
      }
    }
  }
  static __device__ void finish(const Args&, int*) {}
};

// The forward's grouped GEMMs split each expert segment of cnt rows between
// the CTA-pair kernel (256-row pair tiles) and the single-CTA kernel
// (128-row tiles): a last block of at most 128 rows after at least one full
// pair tile, or a whole segment of at most 128 rows, goes to the single-CTA
// kernel, which spends one SM on it where a pair tile would spend two.  The
// head is the rows the pair kernel covers.
// Measured on B200: with K = 2880 (64-wide K blocks: 45 per tile) the split
// took the two GEMMs from 1924 to 1847 us; with K = 2048 and 768 it made
// them 13 % slower (the second launch waits for the first to finish, and
// short tiles do not win that back).
constexpr int kSplitMinK = 2560;
__host__ __device__ __forceinline__ int pair_head(int cnt) {
  if (cnt <= 128) return 0;
  const int mt = cdiv(cnt, 256);
  return (mt >= 2 && cnt - (mt - 1) * 256 <= 128) ? (mt - 1) * 256 : cnt;
}
// First row and length of the part of a segment of cnt rows that a launch
// with the given seg_part covers.
__device__ __forceinline__ void split_rows(int part, int cnt, int& start, int& len) {
  const int head = part ? pair_head(max(cnt, 0)) : 0;
  start = part == 2 ? head : 0;
  len = part == 0 ? cnt : part == 1 ? head : cnt - head;
}

// Grouped problems: schedule over expert segments.  sched layout:
//   [0] total tiles  [1] n-tiles per m-tile row  [8 .. 8+E]  offsets
//   [8+E+1 .. 8+2E+1] cumulative tile counts
template <int BN_, int NUM_B_, int NCOLS_PER_TILE, int MR = BM>
struct GroupedSched {
  static constexpr int BN = BN_;
  static constexpr int MROWS = MR;   // rows of one m-tile (256: a CTA pair)
  static constexpr int NUM_B = NUM_B_;
  static constexpr bool GATHER_A = false;
  static constexpr bool A_MN = false, B_MN = false, MASK_K = false, CUSTOM_LOADS = false;
  static constexpr int EPI_STAGE_BYTES = 0;   // shared staging of the epilogue warps
  static constexpr int EPI_WARPS = 4;         // one per TMEM lane quadrant
  static __device__ int k_rows(const TileInfo&, int) { return BK; }
  static constexpr int THREADS = kThreads;
  static constexpr int SCHED_INTS = 8 + 2 * (kMaxExperts + 1);

  static __device__ void prologue(const Args& a, int* sched) {
    const int E = a.E;
    int* off = sched + 8;
    int* cum = off + E + 1;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = a.offsets[i];
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const int nt = cdiv(a.n_out, NCOLS_PER_TILE);
      const int per = cdiv(E, 32);
      const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
      int local = 0;
      int bad = 0;
      for (int e = e0; e < e1; ++e) {
        const int cnt = off[e + 1] - off[e];
        bad |= cnt < 0;
        int start, len;
        split_rows(a.seg_part, cnt, start, len);
        local += cdiv(max(len, 0), MR) * nt;
      }
      int incl = local;
#pragma unroll
      for (int sh = 1; sh < 32; sh <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, sh);
        if (lane >= sh) incl += v;
      }
      int run = incl - local;
      for (int e = e0; e < e1; ++e) {
        cum[e] = run;
        int start, len;
        split_rows(a.seg_part, off[e + 1] - off[e], start, len);
        run += cdiv(max(len, 0), MR) * nt;
      }
      bad = __any_sync(0xffffffffu, bad);
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) {
        bad |= (off[0] != 0) || (a.rows_upto ? off[E] > a.M : off[E] != a.M);
        cum[E] = total;
        sched[0] = bad ? 0 : total;
        sched[1] = nt;
        if (bad && blockIdx.x == 0) set_status(a.status, MOE_DEV_BAD_OFFSETS);
      }
    }
  }
  static __device__ int num_tiles(const Args&, const int* sched) { return sched[0]; }
  // tile -> (expert e, n-tile, m-tile); m-tiles of one (e, n-tile) are adjacent.
  static __device__ void locate(const Args& a, const int* sched, int tile, int& e, int& nt,
                                int& mt, int& cnt, int& seg0) {
    const int E = a.E;
    const int* off = sched + 8;
    const int* cum = off + E + 1;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cum[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    int start;
    split_rows(a.seg_part, off[e + 1] - off[e], start, cnt);
    seg0 = off[e] + start;
    const int mtiles = cdiv(cnt, MR);
    const int local = tile - cum[e];
    nt = local / mtiles;
    mt = local - nt * mtiles;
  }
};

// GEMM1: B0 = w1 rows [e*h + n0, +128), B1 = w3 rows (same), accumulator
// columns [0,128) = G, [128,256) = U.
template <bool GATHER>
struct UpPolicyT : GroupedSched<256, 2, 128> {
  // With GATHER the A operand is not an expert-major copy of the tokens: four
  // extra warps copy the 128 rows of a tile straight from x through src_row
  // (16-byte cp.async, one warp per pipeline stage).
  static constexpr bool GATHER_A = GATHER;
  static constexpr int THREADS = GATHER ? kThreads + 128 : kThreads;
  static __device__ TileInfo tile_info(const Args& a, const int* sched, int tile) {
    int e, nt, mt, cnt, seg0;
    locate(a, sched, tile, e, nt, mt, cnt, seg0);
    TileInfo t;
    t.a_row = seg0 + mt * BM;
    t.m_valid = min(BM, cnt - mt * BM);
    t.n0 = nt * 128;
    t.b_row = e * a.n_out + t.n0;
    t.kb0 = 0;
    t.kb1 = cdiv(a.K, BK);
    return t;
  }
  static __device__ void epilogue(const Args& a, int*, const TileInfo& ti, uint32_t taddr,
                                  int row) {
    const bool valid = row < ti.m_valid;
    __nv_bfloat16* dst_row = a.out + static_cast<size_t>(ti.a_row + row) * a.n_out + ti.n0;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t g[32], u[32];
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tmem_ld_wait();
      if (valid && ti.n0 + c * 32 < a.n_out) {
        uint32_t p[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float g0 = __uint_as_float(g[2 * q]), g1 = __uint_as_float(g[2 * q + 1]);
          const float u0 = __uint_as_float(u[2 * q]), u1 = __uint_as_float(u[2 * q + 1]);
          const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
          const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
          p[q] = pack_bf16x2(h0, h1);
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) d4[q] = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
        if (a.gu_out) {
          // the bf16 G and U of these 32 hidden units, for the backward
          uint4* g4 = reinterpret_cast<uint4*>(
              a.gu_out + static_cast<size_t>(ti.a_row + row) * (2 * a.n_out) + ti.n0 + c * 32);
          uint4* u4 = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(g4) + a.n_out);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            g4[q] = make_uint4(pack_bf16x2(__uint_as_float(g[8 * q]), __uint_as_float(g[8 * q + 1])),
                               pack_bf16x2(__uint_as_float(g[8 * q + 2]), __uint_as_float(g[8 * q + 3])),
                               pack_bf16x2(__uint_as_float(g[8 * q + 4]), __uint_as_float(g[8 * q + 5])),
                               pack_bf16x2(__uint_as_float(g[8 * q + 6]), __uint_as_float(g[8 * q + 7])));
            u4[q] = make_uint4(pack_bf16x2(__uint_as_float(u[8 * q]), __uint_as_float(u[8 * q + 1])),
                               pack_bf16x2(__uint_as_float(u[8 * q + 2]), __uint_as_float(u[8 * q + 3])),
                               pack_bf16x2(__uint_as_float(u[8 * q + 4]), __uint_as_float(u[8 * q + 5])),
                               pack_bf16x2(__uint_as_float(u[8 * q + 6]), __uint_as_float(u[8 * q + 7])));
          }
        }
      }
    }
  }
  static __device__ void finish(const Args&, int*) {}
};
using UpPolicy = UpPolicyT<false>;
using UpGatherPolicy = UpPolicyT<true>;

// GEMM2: B = w2 rows [e*d + n0, +256).
struct DownPolicy : GroupedSched<256, 1, 256> {
  static __device__ TileInfo tile_info(const Args& a, const int* sched, int tile) {
    int e, nt, mt, cnt, seg0;
    locate(a, sched, tile, e, nt, mt, cnt, seg0);
    TileInfo t;
    t.a_row = seg0 + mt * BM;
    t.m_valid = min(BM, cnt - mt * BM);
    t.n0 = nt * 256;
    t.b_row = e * a.n_out + t.n0;
    t.kb0 = 0;
    t.kb1 = cdiv(a.K, BK);
    return t;
  }
  static __device__ void epilogue(const Args& a, int*, const TileInfo& ti, uint32_t taddr,
                                  int row) {
    const bool valid = row < ti.m_valid;
    const size_t grow = static_cast<size_t>(ti.a_row + row);
    const float scale = (valid && a.row_scale) ? a.row_scale[grow] : 1.0f;
    __nv_bfloat16* dst_row = a.out + grow * a.n_out + ti.n0;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      if (valid && ti.n0 + c * 32 < a.n_out) {
        uint32_t p[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          p[q] = pack_bf16x2(__uint_as_float(r[2 * q]) * scale,
                             __uint_as_float(r[2 * q + 1]) * scale);
        uint4* d4 = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) d4[q] = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
      }
    }
  }
  static __device__ void finish(const Args&, int*) {}
};

// ------------------------------------------------------- backward policies
// The backward of the grouped SwiGLU (the derivative of the forward above,
// one expert segment at a time; G = S w1^T, U = S w3^T, A = silu(G) * U,
// Y = A w2^T):
//   dA = dY w2,  dU = dA * silu(G),  dG = dA * U * silu'(G)   (DownBwdPolicy)
//   dS = dG w1 + dU w3                                          (UpBwdPolicy)
//   dw2 = dY^T A,  dw1 = dG^T S,  dw3 = dU^T S                  (WgradPolicy)
// The weights enter the data gradients untransposed, so their tiles are
// MN-major: a stage holds BN/64 TMA boxes of 64 K rows x 64 columns (one
// 128-byte swizzled line per K row), 8 KB apart.  The weight gradients
// reduce over an expert's rows: both operands are MN-major and the K loop
// runs over the segment, 64 rows per stage; rows of the last stage that
// belong to the next segment are zeroed in shared memory before the MMA.
constexpr int kMnBoxBytes = 64 * BK * 2;   // one 64 x 64 MN-major box: 8 KB

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Epilogue staging: a warp's 32 rows x 32 bf16 columns (64 bytes per row)
// pass through 2 KB of shared memory so that global loads and stores move
// whole 64-byte row segments (4 lanes per row, 8 rows per instruction)
// instead of one 16-byte piece of 32 different rows.  The 16-byte part j of
// row r sits at r * 64 + (j ^ ((r >> 1) & 3)) * 16: conflict-free both for
// "one row per lane" and for "four lanes per row".
__device__ __forceinline__ uint32_t stg_off(int r, int j) {
  return static_cast<uint32_t>(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// Data gradient of GEMM2 with the SwiGLU backward in the epilogue:
// A = dY [N, d] (K-major, K = d), B = w2[e] [d, h] as K rows x h columns.
// The accumulator holds dA for 256 hidden units; the epilogue reads G and U
// from gu_in and writes dG | dU into `out` ([N, 2h], the layout of gu).
struct DownBwdPolicy : GroupedSched<256, 1, 256> {
  static constexpr bool B_MN = true, CUSTOM_LOADS = true;
  static constexpr int EPI_WARPS = 8;   // two per lane quadrant, 128 columns each
  static constexpr int THREADS = kThreads + 128;
  static __device__ TileInfo tile_info(const Args& a, const int* sched, int tile) {
    int e, nt, mt, cnt, seg0;
    locate(a, sched, tile, e, nt, mt, cnt, seg0);
    TileInfo t;
    t.a_row = seg0 + mt * BM;
    t.m_valid = min(BM, cnt - mt * BM);
    t.n0 = nt * 256;
    t.b_row = e * a.K;
    t.kb0 = 0;
    t.kb1 = cdiv(a.K, BK);
    t.m0 = 0;
    return t;
  }
  static __device__ void issue_loads(const Args&, const CUtensorMap* tmA, const CUtensorMap* tmB0,
                                     const CUtensorMap*, const TileInfo& ti, int kb, uint8_t* sa,
                                     uint8_t* sb, uint64_t* bar, uint64_t pa, uint64_t pb) {
    tma_load_2d(sa, tmA, bar, kb * BK, ti.a_row, pa);
#pragma unroll
    for (int c = 0; c < BN / 64; ++c)
      tma_load_2d(sb + c * kMnBoxBytes, tmB0, bar, ti.n0 + 64 * c, ti.b_row + kb * BK, pb);
  }
  static constexpr int EPI_STAGE_BYTES = 8 * 2048;   // per warp: 32 rows x 64 bytes
  static __device__ void epilogue(const Args&, int*, const TileInfo&, uint32_t, int) {}
  // Per 32-column chunk in [c0, c1): the warp loads G and U of its 32 rows
  // (coalesced; the next chunk's loads are in flight while this one is
  // computed), each lane takes its own row through shared memory, forms dG
  // and dU with the accumulator's dA, and the warp stores them coalesced.
  static __device__ void epilogue_staged(const Args& a, int*, const TileInfo& ti, uint32_t taddr,
                                         int row, uint8_t* stg, int c0, int c1) {
    const int h = a.n_out;
    const int lane = threadIdx.x & 31;
    const int wrow0 = row - lane;
    const int j = lane & 3;
    auto load_chunk = [&](int c, uint4 (&buf)[8]) {
      const bool live = ti.n0 + c * 32 < h;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = 8 * q + (lane >> 2);
        if (live && wrow0 + rr < ti.m_valid) {
          const __nv_bfloat16* src =
              a.gu_in + static_cast<size_t>(ti.a_row + wrow0 + rr) * (2 * h) + ti.n0 + c * 32 + j * 8;
          buf[q] = *reinterpret_cast<const uint4*>(src);
          buf[4 + q] = *reinterpret_cast<const uint4*>(src + h);
        } else {
          buf[q] = make_uint4(0u, 0u, 0u, 0u);
          buf[4 + q] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    };
    // coalesced rows -> staging -> this lane's row (16 words)
    auto to_row = [&](const uint4* part, uint32_t (&w)[16]) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(stg + stg_off(8 * q + (lane >> 2), j)) = part[q];
      __syncwarp();
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint4 v = *reinterpret_cast<const uint4*>(stg + stg_off(lane, p));
        w[4 * p] = v.x;
        w[4 * p + 1] = v.y;
        w[4 * p + 2] = v.z;
        w[4 * p + 3] = v.w;
      }
      __syncwarp();
    };
    // this lane's row (16 words) -> staging -> coalesced stores at column offset
    auto from_row = [&](const uint32_t (&w)[16], int c, int col_off) {
#pragma unroll
      for (int p = 0; p < 4; ++p)
        *reinterpret_cast<uint4*>(stg + stg_off(lane, p)) =
            make_uint4(w[4 * p], w[4 * p + 1], w[4 * p + 2], w[4 * p + 3]);
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = 8 * q + (lane >> 2);
        if (wrow0 + rr < ti.m_valid)
          *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(ti.a_row + wrow0 + rr) * (2 * h) +
                                    col_off + ti.n0 + c * 32 + j * 8) =
              *reinterpret_cast<const uint4*>(stg + stg_off(rr, j));
      }
      __syncwarp();
    };
    uint4 cur[8], nxt[8];
    load_chunk(c0, cur);
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      const bool live = ti.n0 + c * 32 < h;
      if (c + 1 < c1) load_chunk(c + 1, nxt);
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      if (live) {
        uint32_t gw[16], uw[16];
        to_row(cur, gw);
        to_row(cur + 4, uw);
        uint32_t pg[16], pu[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float dg[2], du[2];
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            const float g = hlf ? bf16_hi(gw[q]) : bf16_lo(gw[q]);
            const float u = hlf ? bf16_hi(uw[q]) : bf16_lo(uw[q]);
            const float da = __uint_as_float(r[2 * q + hlf]);
            const float sgm = __fdividef(1.0f, 1.0f + __expf(-g));
            du[hlf] = da * (g * sgm);
            dg[hlf] = da * u * (sgm * (1.0f + g * (1.0f - sgm)));
          }
          pg[q] = pack_bf16x2(dg[0], dg[1]);
          pu[q] = pack_bf16x2(du[0], du[1]);
        }
        from_row(pg, c, 0);
        from_row(pu, c, h);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) cur[q] = nxt[q];
    }
  }
  static __device__ void finish(const Args&, int*) {}
};

// Data gradient of GEMM1: A = dG | dU [N, 2h] (K-major, K = 2h), B = the
// K rows of w1[e] (K blocks [0, h/64)) then of w3[e] ([h/64, 2h/64)), each
// [h, d] as K rows x d columns.  Output dS [N, d].
struct UpBwdPolicy : GroupedSched<256, 2, 256> {
  static constexpr bool B_MN = true, CUSTOM_LOADS = true;
  static __device__ TileInfo tile_info(const Args& a, const int* sched, int tile) {
    int e, nt, mt, cnt, seg0;
    locate(a, sched, tile, e, nt, mt, cnt, seg0);
    TileInfo t;
    t.a_row = seg0 + mt * BM;
    t.m_valid = min(BM, cnt - mt * BM);
    t.n0 = nt * 256;
    t.b_row = e * (a.K / 2);
    t.kb0 = 0;
    t.kb1 = cdiv(a.K, BK);
    t.m0 = 0;
    return t;
  }
  static __device__ void issue_loads(const Args& a, const CUtensorMap* tmA,
                                     const CUtensorMap* tmB0, const CUtensorMap* tmB1,
                                     const TileInfo& ti, int kb, uint8_t* sa, uint8_t* sb,
                                     uint64_t* bar, uint64_t pa, uint64_t pb) {
    tma_load_2d(sa, tmA, bar, kb * BK, ti.a_row, pa);
    const int hb = (a.K / 2) / BK;   // K blocks of w1
    const CUtensorMap* m = kb < hb ? tmB0 : tmB1;
    const int y = ti.b_row + (kb < hb ? kb : kb - hb) * BK;
#pragma unroll
    for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * kMnBoxBytes, m, bar, ti.n0 + 64 * c, y, pb);
  }
  static __device__ void epilogue(const Args& a, int* s, const TileInfo& ti, uint32_t taddr,
                                  int row) {
    DownPolicy::epilogue(a, s, ti, taddr, row);   // plain bf16 rows (row_scale is null)
  }
  static __device__ void finish(const Args&, int*) {}
};

// GEMM1 with the staged epilogue: H (and, in the training forward, G and U)
// of 32 hidden units per chunk, 8 epilogue warps (two per lane quadrant, two
// chunks each), every store staged through shared memory so that a warp
// writes whole 64-byte row segments (per-row stores write 16 bytes of 32
// rows per instruction; with G and U added they cost ~15 % of GEMM1).
struct UpStagedPolicy : UpPolicyT<false> {
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = kThreads + 128;
  static constexpr int EPI_STAGE_BYTES = 8 * 2048;
  static __device__ void epilogue_staged(const Args& a, int* s, const TileInfo& ti,
                                         uint32_t taddr, int row, uint8_t* stg, int c0, int c1) {
    const int lane = threadIdx.x & 31;
    const int wrow0 = row - lane;
    const int h = a.n_out;
    const int j = lane & 3;
    // chunk range over the 4 chunks of 32 hidden units (c0, c1 index 8 halves)
    const int q0 = c0 / 2, q1 = c1 / 2;
    auto store = [&](const uint32_t (&w)[16], __nv_bfloat16* base, size_t stride, int col) {
#pragma unroll
      for (int p = 0; p < 4; ++p)
        *reinterpret_cast<uint4*>(stg + stg_off(lane, p)) =
            make_uint4(w[4 * p], w[4 * p + 1], w[4 * p + 2], w[4 * p + 3]);
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = 8 * q + (lane >> 2);
        if (wrow0 + rr < ti.m_valid)
          *reinterpret_cast<uint4*>(base + static_cast<size_t>(ti.a_row + wrow0 + rr) * stride +
                                    col + j * 8) =
              *reinterpret_cast<const uint4*>(stg + stg_off(rr, j));
      }
      __syncwarp();
    };
#pragma unroll 1
    for (int c = q0; c < q1; ++c) {
      uint32_t g[32], u[32];
      tmem_ld32(taddr + c * 32, g);
      tmem_ld32(taddr + 128 + c * 32, u);
      tmem_ld_wait();
      if (ti.n0 + c * 32 >= h) continue;   // warp-uniform
      uint32_t ph[16], pg[16], pu[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float g0 = __uint_as_float(g[2 * q]), g1 = __uint_as_float(g[2 * q + 1]);
        const float u0 = __uint_as_float(u[2 * q]), u1 = __uint_as_float(u[2 * q + 1]);
        ph[q] = pack_bf16x2(silu_f(g0) * u0, silu_f(g1) * u1);
        pg[q] = pack_bf16x2(g0, g1);
        pu[q] = pack_bf16x2(u0, u1);
      }
      const int col = ti.n0 + c * 32;
      store(ph, a.out, static_cast<size_t>(h), col);
      if (a.gu_out) {
        store(pg, a.gu_out, 2 * static_cast<size_t>(h), col);
        store(pu, a.gu_out, 2 * static_cast<size_t>(h), h + col);
      }
    }
  }
};

// GEMM2 with the staged epilogue: 8 warps (two per lane quadrant, four
// 32-column chunks each), each chunk scaled per row, converted, staged and
// stored as whole 64-byte row segments.  Swap-AB tiles keep the per-row
// epilogue (the first warp of each quadrant).
struct DownStagedPolicy : DownPolicy {
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = kThreads + 128;
  static constexpr int EPI_STAGE_BYTES = 8 * 2048;
  static __device__ void epilogue_staged(const Args& a, int* s, const TileInfo& ti,
                                         uint32_t taddr, int row, uint8_t* stg, int c0, int c1) {
    const int lane = threadIdx.x & 31;
    const int wrow0 = row - lane;
    const int j = lane & 3;
    const bool valid = row < ti.m_valid;
    const float scale = (valid && a.row_scale) ? a.row_scale[ti.a_row + row] : 1.0f;
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      if (ti.n0 + c * 32 >= a.n_out) continue;   // warp-uniform
#pragma unroll
      for (int p = 0; p < 4; ++p)
        *reinterpret_cast<uint4*>(stg + stg_off(lane, p)) = make_uint4(
            pack_bf16x2(__uint_as_float(r[8 * p]) * scale, __uint_as_float(r[8 * p + 1]) * scale),
            pack_bf16x2(__uint_as_float(r[8 * p + 2]) * scale,
                        __uint_as_float(r[8 * p + 3]) * scale),
            pack_bf16x2(__uint_as_float(r[8 * p + 4]) * scale,
                        __uint_as_float(r[8 * p + 5]) * scale),
            pack_bf16x2(__uint_as_float(r[8 * p + 6]) * scale,
                        __uint_as_float(r[8 * p + 7]) * scale));
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int rr = 8 * q + (lane >> 2);
        if (wrow0 + rr < ti.m_valid)
          *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(ti.a_row + wrow0 + rr) * a.n_out +
                                    ti.n0 + c * 32 + j * 8) =
              *reinterpret_cast<const uint4*>(stg + stg_off(rr, j));
      }
      __syncwarp();
    }
  }
};

// ------------------------------------------------------ CTA-pair tile schedule
// The forward GEMMs on CTA pairs (cta_group::2).  Every expert segment is
// covered by 256-row pair tiles: CTA rank r owns rows [256 mt + 128 r, +128)
// (its A operand and its accumulator lanes) and loads half of the B tile,
// so a pair moves 64 KB per K block for the work that two single-CTA
// 128 x 256 tiles do with 96 KB.  A segment's last tile may be mostly
// padding; it is still a plain pair tile.  (Swap-AB pair tiles for tails of
// at most 128 rows -- weights as the M = 256 operand, the tail's tokens as
// N -- were built for both GEMMs and measured slower on B200: with them in
// GEMM2, GEMM1 + GEMM2 took 7 % longer at the Qwen3-30B-A3B sizes, 10 % on
// the Zipf layer and 19 % at the gpt-oss EP8 sizes (in both GEMMs: 5 %, 12 %
// and 21 %).  A swap tile streams the whole weight tile for
// a fraction of the MMA work, its small-N MMAs do not run proportionally
// faster, and GEMM2's tail, run right after its normal tile, re-read the
// weight tile from DRAM.)
//   GEMM1: rank 0 loads w1 rows [e h + n0, +128), rank 1 the w3 rows of the
//     same hidden units; accumulator columns 0..127 hold G and 128..255 U.
//   GEMM2: rank r loads w2 rows [e d + n0 + 128 r, +128).
//
// Tiles, taken round-robin by the pairs, are ordered (expert, n-tile,
// m-tile), so the tiles that run at the same time share weight tiles and
// token rows in L2.  (Handing tiles out from a global counter instead was
// measured slower: claimed tiles stay in lock-step, and the pairs working on
// one expert then read the same lines at the same moment.)  sched layout:
// [0] tiles, [1] n-tiles per expert, [8 .. 8+E] offsets, [8+E+1 .. 8+2E+1]
// cumulative tiles per expert.
template <int NCOLS, int NUM_B_, bool UP_>
struct PairSched : GroupedSched<256, NUM_B_, NCOLS, 256> {
  static constexpr bool UP = UP_;

  static __device__ void prologue(const Args& a, int* sched) {
    const int E = a.E;
    int* off = sched + 8;
    int* cum = off + E + 1;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = a.offsets[i];
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const int nt = cdiv(a.n_out, NCOLS);
      const int per = cdiv(E, 32);
      const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
      int local = 0, bad = 0;
      for (int e = e0; e < e1; ++e) {
        const int cnt = off[e + 1] - off[e];
        bad |= cnt < 0;
        int start, len;
        split_rows(a.seg_part, cnt, start, len);
        local += cdiv(max(len, 0), 256) * nt;
      }
      int incl = local;
#pragma unroll
      for (int sh = 1; sh < 32; sh <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, sh);
        if (lane >= sh) incl += v;
      }
      int run = incl - local;
      for (int e = e0; e < e1; ++e) {
        cum[e] = run;
        int start, len;
        split_rows(a.seg_part, off[e + 1] - off[e], start, len);
        run += cdiv(max(len, 0), 256) * nt;
      }
      bad = __any_sync(0xffffffffu, bad);
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) {
        bad |= (off[0] != 0) || (a.rows_upto ? off[E] > a.M : off[E] != a.M);
        cum[E] = total;
        sched[0] = bad ? 0 : total;
        sched[1] = nt;
        if (bad && blockIdx.x == 0) set_status(a.status, MOE_DEV_BAD_OFFSETS);
      }
    }
  }
  static __device__ int num_tiles(const Args&, const int* sched) { return sched[0]; }

  // tile -> its half for CTA `rank` of the pair
  static __device__ TileInfo tile_info(const Args& a, const int* sched, int tile, int rank) {
    const int E = a.E;
    const int* off = sched + 8;
    const int* cum = off + E + 1;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cum[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    int start, cnt;
    split_rows(a.seg_part, off[e + 1] - off[e], start, cnt);
    const int seg0 = off[e] + start;
    const int mtiles = cdiv(cnt, 256);
    const int local = tile - cum[e];
    const int nt = local / mtiles, mt = local - nt * mtiles;
    const int r0 = mt * 256 + rank * 128;
    TileInfo t;
    t.n0 = nt * NCOLS;
    t.kb0 = 0;
    t.kb1 = cdiv(a.K, BK);
    t.m0 = 0;
    t.a_row = seg0 + r0;
    t.m_valid = max(0, min(BM, cnt - r0));
    t.b_row = UP ? e * a.n_out + t.n0 : e * a.n_out + t.n0 + 128 * rank;
    return t;
  }
};

struct UpPairPolicy : PairSched<128, 2, true> {
  static __device__ void epilogue_staged(const Args& a, int* s, const TileInfo& ti,
                                         uint32_t taddr, int row, uint8_t* stg, int c0, int c1) {
    UpStagedPolicy::epilogue_staged(a, s, ti, taddr, row, stg, c0, c1);
  }
};

struct DownPairPolicy : PairSched<256, 1, false> {
  static __device__ void epilogue_staged(const Args& a, int* s, const TileInfo& ti,
                                         uint32_t taddr, int row, uint8_t* stg, int c0, int c1) {
    if (a.comb_out) {
      combine_rows(a, ti, taddr, row, c0, c1);
      return;
    }
    DownStagedPolicy::epilogue_staged(a, s, ti, taddr, row, stg, c0, c1);
  }
  // With the combine folded in: the thread of row s adds its 32 columns of a
  // chunk, times the slot's weight, into the token's fp32 row as eight
  // 16-byte reductions.
  static __device__ void combine_rows(const Args& a, const TileInfo& ti, uint32_t taddr, int row,
                                      int c0, int c1) {
    int tok = -1;
    float w = 0.f;
    if (row < ti.m_valid) {
      const size_t r = static_cast<size_t>(ti.a_row + row);
      tok = a.comb_tok[r];
      w = a.comb_w[r];
    }
    const bool live = static_cast<unsigned>(tok) < static_cast<unsigned>(a.comb_T);
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      if (ti.n0 + c * 32 >= a.n_out || !live) continue;
      float* dst = a.comb_out + static_cast<size_t>(tok) * a.n_out + ti.n0 + c * 32;
#pragma unroll
      for (int g = 0; g < 8; ++g)
        red_add_f32x4(dst + 4 * g, __uint_as_float(r[4 * g]) * w,
                      __uint_as_float(r[4 * g + 1]) * w, __uint_as_float(r[4 * g + 2]) * w,
                      __uint_as_float(r[4 * g + 3]) * w);
    }
  }
};

// Data gradient through one untransposed weight: out [M, n_out] = A B with
// A [M, K] K-major and B [K, n_out] (K rows, MN-major), one segment.  Used
// for the gate: dx = dz . w_router (K = E).
struct DgradPolicy : GroupedSched<256, 1, 256> {
  static constexpr bool B_MN = true, CUSTOM_LOADS = true;
  static __device__ TileInfo tile_info(const Args& a, const int* sched, int tile) {
    int e, nt, mt, cnt, seg0;
    locate(a, sched, tile, e, nt, mt, cnt, seg0);
    TileInfo t;
    t.a_row = seg0 + mt * BM;
    t.m_valid = min(BM, cnt - mt * BM);
    t.n0 = nt * 256;
    t.b_row = e * a.K;
    t.kb0 = 0;
    t.kb1 = cdiv(a.K, BK);
    t.m0 = 0;
    return t;
  }
  static __device__ void issue_loads(const Args& a, const CUtensorMap* tmA,
                                     const CUtensorMap* tmB0, const CUtensorMap* tmB1,
                                     const TileInfo& ti, int kb, uint8_t* sa, uint8_t* sb,
                                     uint64_t* bar, uint64_t pa, uint64_t pb) {
    DownBwdPolicy::issue_loads(a, tmA, tmB0, tmB1, ti, kb, sa, sb, bar, pa, pb);
  }
  static __device__ void epilogue(const Args& a, int* s, const TileInfo& ti, uint32_t taddr,
                                  int row) {
    DownPolicy::epilogue(a, s, ti, taddr, row);   // plain bf16 rows (row_scale is null)
  }
  static __device__ void finish(const Args&, int*) {}
};

// Weight gradients: out[e] = A_e^T B_e over the rows of segment e, with
// A [N, Ma] and B [N, n_out] both MN-major (their columns are the output's
// rows and columns).  Tiles are (expert, 128 output rows, 256 output
// columns), expert-major; an expert with no rows gets zeros.  Output rows
// [0, split) of expert e go to out[e], rows [split, Ma) to out1[e].
struct WgradPolicy {
  static constexpr int BN = 256;
  static constexpr int NUM_B = 1;
  static constexpr bool GATHER_A = false;
  static constexpr bool A_MN = true, B_MN = true, MASK_K = true, CUSTOM_LOADS = true;
  static constexpr int EPI_WARPS = 8;   // two per lane quadrant, 128 columns each
  static constexpr int THREADS = kThreads + 128 + 32;   // + the tail-clearing warp
  static constexpr int SCHED_INTS = 8 + kMaxExperts + 1;   // [0] tiles [1] m-tiles [2] n-tiles, offsets

  static __device__ void prologue(const Args& a, int* sched) {
    const int E = a.E;
    int* off = sched + 8;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = a.offsets[i];
    __syncthreads();
    if (threadIdx.x < 32) {
      int bad = 0;
      for (int e = threadIdx.x; e < E; e += 32) bad |= off[e + 1] < off[e];
      bad = __any_sync(0xffffffffu, bad);
      if (threadIdx.x == 0) {
        bad |= (off[0] != 0) || (a.rows_upto ? off[E] > a.M : off[E] != a.M);
        const int mt = cdiv(a.Ma, BM), nt = cdiv(a.n_out, BN);
        sched[0] = bad ? 0 : E * mt * nt;
        sched[1] = mt;
        sched[2] = nt;
        if (bad && blockIdx.x == 0) set_status(a.status, MOE_DEV_BAD_OFFSETS);
      }
    }
  }
  static __device__ int num_tiles(const Args&, const int* sched) { return sched[0]; }
  static __device__ TileInfo tile_info(const Args&, const int* sched, int tile) {
    const int mt = sched[1], nt = sched[2];
    const int per = mt * nt;
    const int e = tile / per;
    const int r = tile - e * per;
    const int m = r / nt;
    const int* off = sched + 8;
    TileInfo t;
    t.a_row = off[e];
    t.m_valid = off[e + 1] - off[e];
    t.b_row = e;
    t.m0 = m * BM;
    t.n0 = (r - m * nt) * BN;
    t.kb0 = 0;
    t.kb1 = cdiv(t.m_valid, BK);
    return t;
  }
  // rows of K block kb that belong to the segment (the rest are zeroed)
  static __device__ int k_rows(const TileInfo& ti, int kb) { return min(BK, ti.m_valid - kb * BK); }
  static __device__ void issue_loads(const Args&, const CUtensorMap* tmA, const CUtensorMap* tmB0,
                                     const CUtensorMap*, const TileInfo& ti, int kb, uint8_t* sa,
                                     uint8_t* sb, uint64_t* bar, uint64_t pa, uint64_t pb) {
    const int y = ti.a_row + kb * BK;
#pragma unroll
    for (int c = 0; c < BM / 64; ++c) tma_load_2d(sa + c * kMnBoxBytes, tmA, bar, ti.m0 + 64 * c, y, pa);
#pragma unroll
    for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * kMnBoxBytes, tmB0, bar, ti.n0 + 64 * c, y, pb);
  }
  static constexpr int EPI_STAGE_BYTES = 8 * 2048;   // per warp: 32 rows x 64 bytes
  static __device__ void epilogue(const Args&, int*, const TileInfo&, uint32_t, int) {}
  // Each lane converts its row's 32 accumulator columns of a chunk to bf16
  // into the warp's staging rows; the warp then stores 8 rows x 64 bytes per
  // instruction.
  static __device__ void epilogue_staged(const Args& a, int*, const TileInfo& ti, uint32_t taddr,
                                         int row, uint8_t* stg, int c0, int c1) {
    const int lane = threadIdx.x & 31;
    const int wrow0 = row - lane;
    const int Nb = a.n_out;
    const int e = ti.b_row;
    const int j = lane & 3;
    const bool empty = ti.kb1 == ti.kb0;
    if (a.out_f32) {
      // fp32 partials (split reductions): each lane stores its own row
      const int m = ti.m0 + row;
      float* drow = a.out_f32 + (static_cast<size_t>(e) * a.Ma + m) * Nb + ti.n0;
#pragma unroll 1
      for (int c = c0; c < c1; ++c) {
        if (ti.n0 + c * 32 >= Nb) break;   // warp-uniform
        uint32_t r[32];
        if (!empty) {
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) r[q] = 0u;
        }
        if (m < a.Ma) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<uint4*>(drow + c * 32)[q] =
                make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        }
      }
      return;
    }
    __nv_bfloat16* dst[4];
    bool rvalid[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int m = ti.m0 + wrow0 + 8 * q + (lane >> 2);
      rvalid[q] = m < a.Ma;
      dst[q] = m < a.split
                   ? a.out + (static_cast<size_t>(e) * a.split + m) * Nb + ti.n0 + j * 8
                   : a.out1 + (static_cast<size_t>(e) * (a.Ma - a.split) + (m - a.split)) * Nb +
                         ti.n0 + j * 8;
    }
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      if (ti.n0 + c * 32 >= Nb) break;   // warp-uniform
      uint32_t r[32];
      if (!empty) {
        tmem_ld32(taddr + c * 32, r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) r[q] = 0u;
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
        *reinterpret_cast<uint4*>(stg + stg_off(lane, p)) =
            make_uint4(pack_bf16x2(__uint_as_float(r[8 * p]), __uint_as_float(r[8 * p + 1])),
                       pack_bf16x2(__uint_as_float(r[8 * p + 2]), __uint_as_float(r[8 * p + 3])),
                       pack_bf16x2(__uint_as_float(r[8 * p + 4]), __uint_as_float(r[8 * p + 5])),
                       pack_bf16x2(__uint_as_float(r[8 * p + 6]), __uint_as_float(r[8 * p + 7])));
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (rvalid[q])
          *reinterpret_cast<uint4*>(dst[q] + c * 32) =
              *reinterpret_cast<const uint4*>(stg + stg_off(8 * q + (lane >> 2), j));
      __syncwarp();
    }
  }
  static __device__ void finish(const Args&, int*) {}
};

// ------------------------------------------------------------- the kernel

template <class P>
struct Layout {
  static constexpr int BN = P::BN;
  static constexpr int kBTileBytes = BN * BK * 2;
  static constexpr int kStageBytes = kATileBytes + kBTileBytes;
  static constexpr int kStages = stages_for(BN);
  static constexpr uint32_t kTmemCols = tmem_cols_for(BN);
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kNumBars = 3 * kStages + 5;   // full, empty, tail-cleared; 5 more
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSchedOff = (kMiscOff + 16 + 15) / 16 * 16;
  static constexpr int kEpiOff = (kSchedOff + P::SCHED_INTS * 4 + 15) / 16 * 16;
  static constexpr int kBytes = kEpiOff + P::EPI_STAGE_BYTES;
  static constexpr int kLaunchBytes = kBytes + 1024;   // slack for 1 KB alignment
  static_assert(kLaunchBytes <= 227 * 1024, "shared memory budget");
  static_assert(kStages >= 2, "pipeline depth");
  static_assert(!P::GATHER_A || kStages == 4, "one gather warp per stage (warps 6..9)");
  static_assert(!P::GATHER_A || P::EPI_WARPS == 4, "warps 6..9 are either gather or epilogue");
  static_assert(P::THREADS == 64 + 32 * P::EPI_WARPS + (P::GATHER_A ? 128 : 0) +
                                  (P::MASK_K ? 32 : 0),
                "warp roles");
};

template <class P>
__global__ void __launch_bounds__(P::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const Args args) {
  using L = Layout<P>;
  constexpr int BN = P::BN;
  constexpr int STAGES = L::kStages;
  constexpr uint32_t IDESC = idesc_bf16_f32_major(BM, BN, P::A_MN, P::B_MN);
  // descriptor advance per 16-wide K step, in 16-byte units: 32 bytes along
  // a K-major line, or two 128-byte K rows of an MN-major box
  constexpr uint32_t A_KSTEP = P::A_MN ? 128u : 2u;
  constexpr uint32_t B_KSTEP = P::B_MN ? 128u : 2u;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* cleared = mma_done + 1;   // [STAGES] MASK_K: tail rows of the stage zeroed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  int* sched = reinterpret_cast<int*>(smem + L::kSchedOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, P::GATHER_A ? 2 : 1);   // TMA producer (+ gather warp)
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, P::EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    if (P::MASK_K)
      for (int st = 0; st < STAGES; ++st) mbar_init(cleared + st, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (P::NUM_B == 2) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  pdl_wait();   // offsets, A and B may be written by the previous kernel
  P::prologue(args, sched);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = P::num_tiles(args, sched);

  if (warp == 0 && P::GATHER_A) {
    // ------------------------------ TMA producer of the weights (gathered A)
    // The A rows of each stage are copied by the gather warps below; this
    // thread loads the B tile and arms the barrier for its bytes only.
    if (lane == 0) {
      const uint64_t pol_b = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = P::tile_info(args, sched, tile);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          uint8_t* sb = tiles + stage * L::kStageBytes + kATileBytes;
          mbar_arrive_expect_tx(full + stage, L::kBTileBytes);
          tma_load_2d(sb, &tmB0, full + stage, kb * BK, ti.b_row, pol_b);
          if (P::NUM_B == 2)
            tma_load_2d(sb + L::kBTileBytes / 2, &tmB1, full + stage, kb * BK, ti.b_row, pol_b);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < min(issued, STAGES); ++i) {
        if (s == 0) {
          s = STAGES - 1;
          ph ^= 1u;
        } else {
          --s;
        }
        mbar_wait(full + s, ph, nullptr, args.status);
      }
    }
  } else if (P::GATHER_A && warp >= 6) {
    // ------------------------------------ gather warps (A rows from x)
    // Gather warp g owns stage g (STAGES gather warps): for every K block
    // that lands in its stage it copies the tile's 128 rows x 64 columns
    // from x[src_row[.]] with 16-byte cp.async into the 128-byte-swizzled
    // K-major layout the MMA descriptor expects (chunk c of row r at
    // (c ^ (r & 7)) * 16), waits for its copies, fences them into the async
    // proxy and arrives on the stage's "full" barrier.  Rows outside the
    // segment are zero-filled.
    const int g = warp - 6;
    int it = 0;
    bool ok = true;
    const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(args.gather_src);
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileInfo ti = P::tile_info(args, sched, tile);
      const int nkb = ti.kb1 - ti.kb0;
      // this warp's K blocks of the tile: global index it + j with (it + j) % STAGES == g
      int j0 = (g - it % STAGES + STAGES) % STAGES;
      if (j0 < nkb) {
        int rows[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = 4 * lane + q;
          int t = -1;
          if (r < ti.m_valid) {
            const int v = args.src_row[ti.a_row + r];
            if (static_cast<unsigned>(v) < static_cast<unsigned>(args.src_rows)) t = v;
          }
          rows[q] = t;
        }
        for (int j = j0; j < nkb; j += STAGES) {
          const int gi = it + j;                 // global K-block counter
          const uint32_t phase = static_cast<uint32_t>(gi / STAGES) & 1u;
          int go = 1;
          if (lane == 0) go = mbar_wait(empty + g, phase ^ 1u, abort_flag, args.status) ? 1 : 0;
          go = __shfl_sync(0xffffffffu, go, 0);
          if (!go) {
            ok = false;
            break;
          }
          uint8_t* sa = tiles + g * L::kStageBytes;
          const int col0 = (ti.kb0 + j) * BK;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int r = 4 * lane + q;
            const __nv_bfloat16* src =
                xg + static_cast<size_t>(rows[q] < 0 ? 0 : rows[q]) * args.K + col0;
            const uint32_t nbytes = rows[q] < 0 ? 0u : 16u;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              cp_async16(sa + r * 128 + ((c ^ (r & 7)) << 4), src + c * 8, nbytes);
          }
          cp_async_wait_all();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(full + g);
        }
      }
      it += nkb;
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint64_t pol_b = l2_policy_evict_last();
      const uint64_t pol_a = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = P::tile_info(args, sched, tile);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = tiles + stage * L::kStageBytes;
          uint8_t* sb = sa + kATileBytes;
          mbar_arrive_expect_tx(full + stage, L::kStageBytes);
          if constexpr (P::CUSTOM_LOADS) {
            P::issue_loads(args, &tmA, &tmB0, &tmB1, ti, kb, sa, sb, full + stage, pol_a, pol_b);
          } else {
            tma_load_2d(sa, &tmA, full + stage, kb * BK, ti.a_row, pol_a);
            if (P::NUM_B == 1) {
              tma_load_2d(sb, &tmB0, full + stage, kb * BK, ti.b_row, pol_b);
            } else {
              tma_load_2d(sb, &tmB0, full + stage, kb * BK, ti.b_row, pol_b);
              tma_load_2d(sb + L::kBTileBytes / 2, &tmB1, full + stage, kb * BK, ti.b_row, pol_b);
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the last loads land before the CTA may exit.
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < min(issued, STAGES); ++i) {
        if (s == 0) {
          s = STAGES - 1;
          ph ^= 1u;
        } else {
          --s;
        }
        mbar_wait(full + s, ph, nullptr, args.status);
      }
    }
  } else if (P::MASK_K && warp == 2 + P::EPI_WARPS) {
    // ------------------------------------------ tail-clearing warp
    // The last K block of a segment also holds rows of the next segment.
    // Only the 16-row MMA steps that hold segment rows are issued; the rows
    // of the last of them past the segment's end (fewer than 16) are zeroed
    // here in both operands as soon as the stage lands (a K row is one
    // 128-byte line of every 8 KB box, whatever the swizzle).  The warp is a
    // stage of the pipeline: it waits for every fill in order and hands every
    // stage to the MMA thread through its "cleared" barrier, so it can
    // neither run a ring cycle ahead of the fills nor fall behind them (a
    // parity wait cannot tell phases two apart).  Off the MMA thread's path:
    // the pipeline runs ahead, so a stage is usually cleared before the MMAs
    // reach it.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileInfo ti = P::tile_info(args, sched, tile);
      for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
        const int rows = P::k_rows(ti, kb);
        const int zr = ((rows + 15) & ~15) - rows;   // rows [rows, ceil16(rows)) to clear
        const bool landed = mbar_wait(full + stage, phase, abort_flag, args.status);
        if (!__all_sync(0xffffffffu, landed)) {
          ok = false;
          break;
        }
        if (zr > 0) {
          uint8_t* sa = tiles + stage * L::kStageBytes;
          const int per_box = zr * 8;   // 16-byte chunks per box (< 128)
          constexpr int kBoxes = L::kStageBytes / kMnBoxBytes;
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            for (int i = lane; i < per_box; i += 32)
              *reinterpret_cast<uint4*>(sa + bx * kMnBoxBytes + rows * 128 + i * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cleared + stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1 && P::MASK_K) {
    if (lane == 0) {
      // ------------------------------------- MMA issuer, K tails masked
      // Every stage comes through the tail-clearing warp; a segment's last K
      // block issues only the 16-row steps holding its rows.
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(tempty + acc, aph ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const TileInfo ti = P::tile_info(args, sched, tile);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          const int ksteps = (P::k_rows(ti, kb) + 15) >> 4;
          if (!mbar_wait(cleared + stage, phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sa = tiles + stage * L::kStageBytes;
          const uint64_t ad = sw128_mnmajor_desc(sa, kMnBoxBytes);
          const uint64_t bd = sw128_mnmajor_desc(sa + kATileBytes, kMnBoxBytes);
          for (int kk = 0; kk < ksteps; ++kk)
            tc_mma_bf16(d_tmem, ad + A_KSTEP * kk, bd + B_KSTEP * kk, IDESC,
                        (kb != ti.kb0 || kk != 0) ? 1u : 0u);
          tc_commit(empty + stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull + acc);
      }
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, args.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(tempty + acc, aph ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const TileInfo ti = P::tile_info(args, sched, tile);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(full + stage, phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sa = tiles + stage * L::kStageBytes;
          const uint64_t ad =
              P::A_MN ? sw128_mnmajor_desc(sa, kMnBoxBytes) : sw128_kmajor_desc(sa);
          const uint64_t bd = P::B_MN ? sw128_mnmajor_desc(sa + kATileBytes, kMnBoxBytes)
                                      : sw128_kmajor_desc(sa + kATileBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16(d_tmem, ad + A_KSTEP * kk, bd + B_KSTEP * kk, IDESC,
                        (kb != ti.kb0 || kk != 0) ? 1u : 0u);
          tc_commit(empty + stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull + acc);
      }
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, args.status);
    }
  } else if (warp < 2 + P::EPI_WARPS) {
    // -------------------------------------------------- epilogue warps
    // Warp w reads TMEM lanes 32 (w % 4) .. +32 (its quadrant); with 8
    // epilogue warps the two warps of a quadrant split the 8 column chunks.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int half = (warp - 2) >> 2;
    const int c0 = P::EPI_WARPS == 8 ? 4 * half : 0;
    const int c1 = P::EPI_WARPS == 8 ? c0 + 4 : 8;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(tfull + acc, aph, abort_flag, args.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const TileInfo ti = P::tile_info(args, sched, tile);
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if constexpr (P::EPI_STAGE_BYTES > 0)
        P::epilogue_staged(args, sched, ti, taddr, row,
                           smem + L::kEpiOff + (warp - 2) * (P::EPI_STAGE_BYTES / P::EPI_WARPS),
                           c0, c1);
      else
        P::epilogue(args, sched, ti, taddr, row);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
    }
  }
  pdl_trigger();   // the next kernel may start its prologue
  __syncthreads();
  P::finish(args, sched);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------- the CTA-pair kernel
// Two CTAs (a cluster of 2 on neighbouring SMs) share each tile of the
// hybrid schedule through tcgen05.mma.cta_group::2.  Rank 0 (leader) issues
// the MMAs and commits to the barriers of both CTAs; both CTAs' TMA loads
// count on the leader's "full" barrier; both CTAs' epilogue warps arrive on
// the leader's "tmem empty" barrier.  Roles per CTA (320 threads): warp 0
// TMA producer, warp 1 TMEM owner and (leader) MMA issuer, warps 2..9 the
// epilogue (two per TMEM lane quadrant, each taking half of the columns).
// Maps: tmA the token rows, tmB0 / tmB1 the weight halves (128-row boxes;
// tmB1 only for GEMM1).
template <class P>
struct PairLayout {
  static constexpr int kBHalfBytes = 128 * BK * 2;                  // 16 KB
  static constexpr int kStageBytes = kATileBytes + kBHalfBytes;    // 32 KB per CTA
  static constexpr int kStages = 6;
  static constexpr uint32_t kTmemCols = 512;                       // 2 x 256 columns
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 5;   // + tfull[2], tempty[2], mma_done
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSchedOff = (kMiscOff + 16 + 15) / 16 * 16;
  static constexpr int kEpiOff = (kSchedOff + P::SCHED_INTS * 4 + 15) / 16 * 16;
  static constexpr int kBytes = kEpiOff + kEpiWarps * 2048;   // the staged epilogue
  static constexpr int kLaunchBytes = kBytes + 1024;
  static_assert(kLaunchBytes <= 227 * 1024, "shared memory budget");
};

template <class P>
__global__ void __launch_bounds__(PairLayout<P>::kThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const Args args) {
  using L = PairLayout<P>;
  constexpr int STAGES = L::kStages;
  constexpr uint32_t IDESC = idesc_bf16_f32(256, 256);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  int* sched = reinterpret_cast<int*>(smem + L::kSchedOff);
  uint8_t* epi = smem + L::kEpiOff;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, 2 * L::kEpiWarps);   // every epilogue warp of both CTAs
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (P::UP) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  pdl_wait();   // offsets, A and B may be written by the previous kernel
  P::prologue(args, sched);
  __syncthreads();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = P::num_tiles(args, sched);
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      const uint64_t pol = l2_policy_evict_last();
      const CUtensorMap* tb = (P::NUM_B == 2 && rank == 1) ? &tmB1 : &tmB0;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo ti = P::tile_info(args, sched, tile, rank);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = tiles + stage * L::kStageBytes;
          uint8_t* sb = sa + kATileBytes;
          const uint32_t bar = cluster_map(full + stage, 0);
          if (leader) mbar_arrive_expect_tx(full + stage, 2 * L::kStageBytes);
          tma_load_2d_pair(sa, &tmA, bar, kb * BK, ti.a_row, pol);
          tma_load_2d_pair(sb, tb, bar, kb * BK, ti.b_row, pol);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: a stage's loads have landed once the MMAs that read it are
      // done, which the leader commits to this CTA's "empty" barrier.
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < min(issued, STAGES); ++i) {
        if (s == 0) {
          s = STAGES - 1;
          ph ^= 1u;
        } else {
          --s;
        }
        mbar_wait(empty + s, ph, nullptr, args.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_cluster(tempty + acc, aph ^ 1u, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        const TileInfo ti = P::tile_info(args, sched, tile, 0);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(full + stage, phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sa = tiles + stage * L::kStageBytes;
          const uint64_t ad = sw128_kmajor_desc(sa);
          const uint64_t bd = sw128_kmajor_desc(sa + kATileBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16_pair(d_tmem, ad + 2u * kk, bd + 2u * kk, IDESC,
                             (kb != ti.kb0 || kk != 0) ? 1u : 0u);
          tc_commit_pair_mc(empty + stage, 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(tfull + acc, 0x3);
      }
      tc_commit_pair(mma_done);
      mbar_wait(mma_done, 0, nullptr, args.status);
    }
  } else {
    // -------------------------------------------------- epilogue warps (both CTAs)
    // Warp w reads TMEM lanes 32 (w % 4) .. +32; the two warps of a quadrant
    // (half 0: warps 2..5, half 1: warps 6..9) split the columns.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int half = (warp - 2) >> 2;
    uint32_t tempty_leader[2];
    tempty_leader[0] = cluster_map(tempty + 0, 0);
    tempty_leader[1] = cluster_map(tempty + 1, 0);
    int it = 0;
    bool run = true;
    for (int tile = pair; tile < total && run; tile += npairs, ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(tfull + acc, aph, abort_flag, args.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        run = false;
        break;
      }
      tc_fence_after();
      const TileInfo ti = P::tile_info(args, sched, tile, rank);
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 256);
      P::epilogue_staged(args, sched, ti, taddr, row, epi + (warp - 2) * 2048, 4 * half,
                         4 * half + 4);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
    }
  }
  pdl_trigger();   // the next kernel may start its prologue
  __syncthreads();
  cluster_sync_all();   // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, inner] array, box [box_rows, 64],
// 128-byte swizzle, zero fill outside the array.
bool make_tmap(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled failed (%d) for rows=%llu inner=%llu", (int)r,
                   (unsigned long long)rows, (unsigned long long)inner);
    return false;
  }
  return true;
}

template <class P>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                   const Args& args, int grid, cudaStream_t s) {
  using L = Layout<P>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<P>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kLaunchBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  launch_k(tc_gemm_kernel<P>, dim3(grid), dim3(P::THREADS), L::kLaunchBytes, s, a, b0, b1, args);
  return cudaGetLastError();
}

// Launch of the CTA-pair kernel: clusters of 2 CTAs, an even grid.
template <class P>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const Args& args, int pairs, cudaStream_t s) {
  using L = PairLayout<P>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_pair_kernel<P>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kLaunchBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(L::kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kLaunchBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<P>, a, b0, b1, args);
}

}  // namespace tc

RouterPlan router_plan(int T, int d) {
  RouterPlan p{};
  const int mt = std::max(1, cdiv(T, tc::BM));
  const int kb = std::max(1, cdiv(d, tc::BK));
  // at most one wave of tiles: mt * ksplit <= kRouterTargetTiles when mt allows
  int split = std::max(1, std::min(kb, kRouterTargetTiles / mt));
  p.kb_per_split = cdiv(kb, split);
  p.ksplit = cdiv(kb, p.kb_per_split);   // every split has at least one K block
  return p;
}

cudaError_t launch_router_tc(const void* x, const void* w_router, int T, int d, int E,
                             float* logits_part, int* status, cudaStream_t s) {
  using namespace tc;
  const int bn = E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, x, d, T, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, w_router, d, E, bn)) return cudaErrorInvalidValue;
  const RouterPlan p = router_plan(T, d);
  Args a{};
  a.M = T;
  a.K = d;
  a.E = E;
  a.n_out = E;
  a.status = status;
  a.logits_part = logits_part;
  a.ksplit = p.ksplit;
  a.kb_per_split = p.kb_per_split;
  const int grid = std::min(num_sms(), cdiv(T, BM) * p.ksplit);
  switch (bn) {
    case 32: return launch<RouterPolicy<32>>(ta, tb, tb, a, grid, s);
    case 64: return launch<RouterPolicy<64>>(ta, tb, tb, a, grid, s);
    case 128: return launch<RouterPolicy<128>>(ta, tb, tb, a, grid, s);
    default: return launch<RouterPolicy<256>>(ta, tb, tb, a, grid, s);
  }
}

// Grouped SwiGLU with GEMM1's A operand gathered from x [T, d] through
// src_row (no expert-major copy of the tokens in memory).
// Folded combine of GEMM2 (CTA-pair path only): see Args::comb_out.
struct FoldedCombine {
  float* out;           // [T, d] fp32, zero before the call
  const int32_t* tok;   // [N]
  const float* w;       // [N]
  int T;
};

static cudaError_t swiglu_tc_impl(const void* a_src, int a_rows, const int32_t* src_row,
                                  const int32_t* offsets, const void* w1, const void* w3,
                                  const void* w2, const float* row_scale, int N, int d, int h,
                                  int E, void* y, void* H, int* status, cudaStream_t s,
                                  void* gu = nullptr, const FoldedCombine* fold = nullptr,
                                  bool rows_upto = false);

cudaError_t launch_swiglu_tc(const void* x_perm, const int32_t* offsets, const void* w1,
                             const void* w3, const void* w2, const float* row_scale, int N,
                             int d, int h, int E, void* y, void* H, int* status,
                             cudaStream_t s, bool rows_upto) {
  return swiglu_tc_impl(x_perm, N, nullptr, offsets, w1, w3, w2, row_scale, N, d, h, E, y, H,
                        status, s, nullptr, nullptr, rows_upto);
}

cudaError_t launch_swiglu_tc_gather(const void* x, int T, const int32_t* src_row,
                                    const int32_t* offsets, const void* w1, const void* w3,
                                    const void* w2, const float* row_scale, int N, int d, int h,
                                    int E, void* y, void* H, int* status, cudaStream_t s) {
  return swiglu_tc_impl(x, T, src_row, offsets, w1, w3, w2, row_scale, N, d, h, E, y, H, status,
                        s);
}

bool swiglu_tc_uses_pairs(int N, int E) { return N >= 64LL * E; }

cudaError_t launch_swiglu_tc_combine(const void* x_perm, const int32_t* offsets, const void* w1,
                                     const void* w3, const void* w2, int N, int d, int h, int E,
                                     void* H, const int32_t* slot_tok, const float* slot_w,
                                     int T, float* out32, int* status, cudaStream_t s) {
  if (!swiglu_tc_uses_pairs(N, E)) return cudaErrorInvalidValue;
  const FoldedCombine fold{out32, slot_tok, slot_w, T};
  return swiglu_tc_impl(x_perm, N, nullptr, offsets, w1, w3, w2, nullptr, N, d, h, E, nullptr,
                        H, status, s, nullptr, &fold);
}

static cudaError_t swiglu_tc_impl(const void* a_src, int a_rows, const int32_t* src_row,
                                  const int32_t* offsets, const void* w1, const void* w3,
                                  const void* w2, const float* row_scale, int N, int d, int h,
                                  int E, void* y, void* H, int* status, cudaStream_t s,
                                  void* gu, const FoldedCombine* fold, bool rows_upto) {
  using namespace tc;
  CUtensorMap tx, t1, t3, th, t2;
  const bool gather = src_row != nullptr;
  if (!make_tmap(&tx, a_src, d, a_rows, gather ? 1 : BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&t1, w1, d, static_cast<uint64_t>(E) * h, 128)) return cudaErrorInvalidValue;
  if (!make_tmap(&t3, w3, d, static_cast<uint64_t>(E) * h, 128)) return cudaErrorInvalidValue;
  if (!make_tmap(&th, H, h, N, BM)) return cudaErrorInvalidValue;
  // The CTA-pair kernel (256-row pair tiles) serves every layer whose
  // segments average 64 rows or more; shorter segments (decode) stay on the
  // single-CTA kernel, whose 128-row tiles stream each weight tile once.
  const bool pairs = !gather && swiglu_tc_uses_pairs(N, E);
  if (fold && !pairs) return cudaErrorInvalidValue;
  if (!make_tmap(&t2, w2, h, static_cast<uint64_t>(E) * d, pairs ? 128 : 256))
    return cudaErrorInvalidValue;
  const int max_mt = cdiv(N, BM) + E;   // upper bound on m-tiles over all segments
  Args a{};
  a.M = N;
  a.E = E;
  a.offsets = offsets;
  a.status = status;
  a.rows_upto = rows_upto ? 1 : 0;
  // GEMM1: H = silu(x w1^T) * (x w3^T)
  a.K = d;
  a.n_out = h;
  a.out = static_cast<__nv_bfloat16*>(H);
  a.src_row = src_row;
  a.src_rows = a_rows;
  a.gather_src = a_src;
  a.gu_out = static_cast<__nv_bfloat16*>(gu);
  if (pairs) {
    // Each segment's head on CTA pairs and its short last block on the
    // single-CTA kernel (pair_head), for a GEMM whose reduction is long
    // enough (kSplitMinK) that the tail tiles' saving outweighs the second
    // launch; the folded combine keeps whole segments on pairs (only the
    // pair kernel folds).  The tail launches read what the head launches
    // read and write other rows.
    const bool split1 = fold == nullptr && d >= kSplitMinK;
    const bool split2 = fold == nullptr && h >= kSplitMinK;
    CUtensorMap t2s;   // w2 in 256-row boxes for the single-CTA GEMM2
    if (split2 && !make_tmap(&t2s, w2, h, static_cast<uint64_t>(E) * d, 256))
      return cudaErrorInvalidValue;
    const long long max_pt = cdiv(N, 256) + E;   // upper bound on pair tiles per n-tile
    int np = static_cast<int>(std::min<long long>(num_sms() / 2, max_pt * cdiv(h, 128)));
    a.seg_part = split1 ? 1 : 0;
    cudaError_t e = launch_pair<UpPairPolicy>(tx, t1, t3, a, np, s);
    if (e != cudaSuccess) return e;
    if (split1) {   // at most one 128-row tail tile per (expert, n-tile)
      a.seg_part = 2;
      e = launch<UpStagedPolicy>(tx, t1, t3, a,
                                 static_cast<int>(std::min<long long>(
                                     num_sms(), 1LL * E * cdiv(h, 128))),
                                 s);
      if (e != cudaSuccess) return e;
    }
    a.K = h;
    a.n_out = d;
    a.out = static_cast<__nv_bfloat16*>(y);
    a.gu_out = nullptr;
    a.row_scale = row_scale;
    if (fold) {
      a.comb_out = fold->out;
      a.comb_tok = fold->tok;
      a.comb_w = fold->w;
      a.comb_T = fold->T;
    }
    np = static_cast<int>(std::min<long long>(num_sms() / 2, max_pt * cdiv(d, 256)));
    a.seg_part = split2 ? 1 : 0;
    e = launch_pair<DownPairPolicy>(th, t2, t2, a, np, s);
    if (e != cudaSuccess || !split2) return e;
    a.seg_part = 2;
    return launch<DownStagedPolicy>(th, t2s, t2s, a,
                                    static_cast<int>(std::min<long long>(
                                        num_sms(), 1LL * E * cdiv(d, 256))),
                                    s);
  }
  int grid = static_cast<int>(std::min<long long>(num_sms(), 1LL * max_mt * cdiv(h, 128)));
  cudaError_t e = gather ? launch<UpGatherPolicy>(tx, t1, t3, a, grid, s)
                         : launch<UpStagedPolicy>(tx, t1, t3, a, grid, s);
  if (e != cudaSuccess) return e;
  // GEMM2: y = H w2^T (* row_scale)
  a.K = h;
  a.n_out = d;
  a.out = static_cast<__nv_bfloat16*>(y);
  a.row_scale = row_scale;
  grid = static_cast<int>(std::min<long long>(num_sms(), 1LL * max_mt * cdiv(d, 256)));
  return launch<DownStagedPolicy>(th, t2, t2, a, grid, s);
}

cudaError_t launch_swiglu_tc_train(const void* x_perm, const int32_t* offsets, const void* w1,
                                   const void* w3, const void* w2, int N, int d, int h, int E,
                                   void* y, void* H, void* GU, int* status, cudaStream_t s) {
  return swiglu_tc_impl(x_perm, N, nullptr, offsets, w1, w3, w2, nullptr, N, d, h, E, y, H,
                        status, s, GU);
}

// Backward of the grouped SwiGLU: four launches on `s`.
//   1. dG | dU = SwiGLU'(G, U) applied to dY w2     (DownBwdPolicy, into dGU)
//   2. dx_perm = dG w1 + dU w3                       (UpBwdPolicy)
//   3. dw2 = dY^T H per expert                       (WgradPolicy)
//   4. dw1 | dw3 = (dG | dU)^T x_perm per expert     (WgradPolicy, rows split at h)
cudaError_t launch_swiglu_bwd_tc(const void* x_perm, const int32_t* offsets, const void* w1,
                                 const void* w3, const void* w2, const void* H, const void* GU,
                                 const void* dY, int N, int d, int h, int E, void* dX, void* dW1,
                                 void* dW3, void* dW2, void* dGU, int* status, cudaStream_t s) {
  using namespace tc;
  const uint64_t Eh = static_cast<uint64_t>(E) * h, Ed = static_cast<uint64_t>(E) * d;
  const int max_mt = cdiv(N, BM) + E;
  CUtensorMap t_dy, t_w2, t_dgu, t_w1, t_w3;
  if (!make_tmap(&t_dy, dY, d, N, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&t_w2, w2, h, Ed, 64)) return cudaErrorInvalidValue;
  if (!make_tmap(&t_dgu, dGU, 2 * static_cast<uint64_t>(h), N, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&t_w1, w1, d, Eh, 64)) return cudaErrorInvalidValue;
  if (!make_tmap(&t_w3, w3, d, Eh, 64)) return cudaErrorInvalidValue;
  Args a{};
  a.M = N;
  a.E = E;
  a.offsets = offsets;
  a.status = status;
  // 1. data gradient of GEMM2 and the SwiGLU backward
  a.K = d;
  a.n_out = h;
  a.out = static_cast<__nv_bfloat16*>(dGU);
  a.gu_in = static_cast<const __nv_bfloat16*>(GU);
  int grid = static_cast<int>(std::min<long long>(num_sms(), 1LL * max_mt * cdiv(h, 256)));
  cudaError_t e = launch<DownBwdPolicy>(t_dy, t_w2, t_w2, a, grid, s);
  if (e != cudaSuccess) return e;
  // 2. data gradient of GEMM1
  a.K = 2 * h;
  a.n_out = d;
  a.out = static_cast<__nv_bfloat16*>(dX);
  a.gu_in = nullptr;
  grid = static_cast<int>(std::min<long long>(num_sms(), 1LL * max_mt * cdiv(d, 256)));
  e = launch<UpBwdPolicy>(t_dgu, t_w1, t_w3, a, grid, s);
  if (e != cudaSuccess) return e;
  // 3. dw2[e] = dY_e^T H_e: output rows d (A = dY columns), columns h
  CUtensorMap m_dy, m_h, m_dgu, m_x;
  if (!make_tmap(&m_dy, dY, d, N, 64)) return cudaErrorInvalidValue;
  if (!make_tmap(&m_h, H, h, N, 64)) return cudaErrorInvalidValue;
  if (!make_tmap(&m_dgu, dGU, 2 * static_cast<uint64_t>(h), N, 64)) return cudaErrorInvalidValue;
  if (!make_tmap(&m_x, x_perm, d, N, 64)) return cudaErrorInvalidValue;
  a.K = 0;
  a.Ma = d;
  a.split = d;
  a.n_out = h;
  a.out = static_cast<__nv_bfloat16*>(dW2);
  a.out1 = nullptr;
  grid = static_cast<int>(std::min<long long>(num_sms(), 1LL * E * cdiv(d, BM) * cdiv(h, 256)));
  e = launch<WgradPolicy>(m_dy, m_h, m_h, a, grid, s);
  if (e != cudaSuccess) return e;
  // 4. dw1[e] = dG_e^T x_e, dw3[e] = dU_e^T x_e: output rows 2h, columns d
  a.Ma = 2 * h;
  a.split = h;
  a.n_out = d;
  a.out = static_cast<__nv_bfloat16*>(dW1);
  a.out1 = static_cast<__nv_bfloat16*>(dW3);
  grid = static_cast<int>(std::min<long long>(num_sms(), 1LL * E * cdiv(2 * h, BM) * cdiv(d, 256)));
  return launch<WgradPolicy>(m_dgu, m_x, m_x, a, grid, s);
}

// Token segments of the gate's weight gradient: enough (E, d) tiles x
// segments to fill about kRouterTargetTiles SMs, segments of >= 256 tokens,
// at most 63 (the offsets fit in 256 bytes).  Sizes only: workspace sizes
// are computed on the host without a device.
int gate_splits(int T, int d, int E) {
  const int tiles = cdiv(E, tc::BM) * cdiv(d, 256);
  return std::max(1, std::min(std::min(kRouterTargetTiles / tiles, T / 256), 63));
}

// Gradients of the gate logits = x . w_router^T for dz16 [T, E] (bf16):
//   dw_router = dz^T x   (WgradPolicy over S token segments into fp32
//                         partials, then summed in segment order)
//   dx        = dz w_router (DgradPolicy, K = E, one segment)
cudaError_t launch_gate_backward_tc(const void* dz16, const void* x, const void* w_router, int T,
                                    int d, int E, void* dw_router, void* dx, int32_t* offsets,
                                    float* gpart, int* status, cudaStream_t s) {
  using namespace tc;
  if (T == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  Args a{};
  a.M = T;
  a.status = status;
  a.offsets = offsets;
  if (dw_router) {
    const int S = gate_splits(T, d, E);
    e = launch_uniform_segments(offsets, S, T, s);
    if (e != cudaSuccess) return e;
    CUtensorMap m_dz, m_x;
    if (!make_tmap(&m_dz, dz16, E, T, 64)) return cudaErrorInvalidValue;
    if (!make_tmap(&m_x, x, d, T, 64)) return cudaErrorInvalidValue;
    a.E = S;
    a.Ma = E;
    a.split = E;
    a.n_out = d;
    a.out = nullptr;
    a.out1 = nullptr;
    a.out_f32 = gpart;
    const int grid = std::min(num_sms(), S * cdiv(E, BM) * cdiv(d, 256));
    e = launch<WgradPolicy>(m_dz, m_x, m_x, a, grid, s);
    if (e == cudaSuccess)
      e = launch_sum_partials_bf16(gpart, S, static_cast<size_t>(E) * d, dw_router, s);
    if (e != cudaSuccess) return e;
    a.out_f32 = nullptr;
  }
  if (dx) {
    e = launch_single_segment(offsets, T, s);
    if (e != cudaSuccess) return e;
    a.E = 1;
    CUtensorMap t_dz, t_wr;
    if (!make_tmap(&t_dz, dz16, E, T, BM)) return cudaErrorInvalidValue;
    if (!make_tmap(&t_wr, w_router, d, E, 64)) return cudaErrorInvalidValue;
    a.K = E;
    a.n_out = d;
    a.out = static_cast<__nv_bfloat16*>(dx);
    a.out1 = nullptr;
    a.row_scale = nullptr;
    const int grid = std::min(num_sms(), cdiv(T, BM) * cdiv(d, 256));
    e = launch<DgradPolicy>(t_dz, t_wr, t_wr, a, grid, s);
  }
  return e;
}

}  // namespace moe
