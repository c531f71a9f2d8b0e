// fp32 grouped SwiGLU on CUDA cores ([HP] _run_experts_for_loop semantics):
// fp32 in, fp32 accumulate, fp32 out.  Used for fp32 layers, where tensor
// cores (tf32) could not meet a 1e-5 relative tolerance.  32 x 32 output
// tiles inside one expert segment; the tile schedule is built per block from
// the device offsets, so no host synchronisation is needed.  The backward
// of the same function (and the fp32 gate gradients of the router) run on
// one segmented fp32 contraction kernel with strided operands.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int SB = 32;   // rows, columns and K step of a tile

// Per-block tile schedule over expert segments (m-tiles of SB rows).
// Returns false if the offsets are not a valid segmentation of [0, N).
__device__ bool simt_schedule(const int32_t* offsets, int E, int N, int* off, int* cum,
                              int* status) {
  __shared__ int ok;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0, good = (off[0] == 0) && (off[E] == N);
    for (int e = 0; e < E; ++e) {
      const int c = off[e + 1] - off[e];
      good &= c >= 0;
      cum[e] = run;
      run += c > 0 ? cdiv(c, SB) : 0;
    }
    cum[E] = run;
    ok = good;
    if (!good && blockIdx.x == 0 && blockIdx.y == 0) set_status(status, MOE_DEV_BAD_OFFSETS);
  }
  __syncthreads();
  return ok != 0;
}

__device__ void simt_locate(const int* off, const int* cum, int E, int tile, int& row0,
                            int& valid) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int mt = tile - cum[lo];
  row0 = off[lo] + mt * SB;
  valid = min(SB, off[lo + 1] - row0);
}

// H[s, n] = silu(sum_i x[s,i] w1[e,n,i]) * (sum_i x[s,i] w3[e,n,i])
__global__ void __launch_bounds__(256) swiglu_up_f32_kernel(
    const float* __restrict__ x, const int32_t* __restrict__ src_row, int x_rows,
    const int32_t* __restrict__ offsets, const float* __restrict__ w1,
    const float* __restrict__ w3, int N, int d, int h, int E, float* __restrict__ H,
    float* __restrict__ GU, int* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int off[kMaxExperts + 1], cum[kMaxExperts + 1];
  __shared__ float xs[SB][SB + 1], as[SB][SB + 1], bs[SB][SB + 1];
  __shared__ int xrow[SB];
  if (!simt_schedule(offsets, E, N, off, cum, status)) return;
  const int tile = blockIdx.x;
  if (tile >= cum[E]) return;
  int row0, valid;
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  simt_locate(off, cum, E, tile, row0, valid);
  const int n0 = blockIdx.y * SB;
  const int ty = threadIdx.x >> 3, tx = threadIdx.x & 7;   // row ty, columns tx*4..+3
  // source row of every tile row: the slot itself, or its token when gathering
  if (threadIdx.x < SB) {
    const int r = threadIdx.x;
    int src = -1;
    if (r < valid) {
      src = src_row ? src_row[row0 + r] : row0 + r;
      if (static_cast<unsigned>(src) >= static_cast<unsigned>(x_rows)) src = -1;
    }
    xrow[r] = src;
  }
  __syncthreads();
  const float* W1 = w1 + static_cast<size_t>(e) * h * d;
  const float* W3 = w3 + static_cast<size_t>(e) * h * d;
  float g[4] = {0, 0, 0, 0}, u[4] = {0, 0, 0, 0};
  for (int k0 = 0; k0 < d; k0 += SB) {
    for (int i = threadIdx.x; i < SB * SB; i += blockDim.x) {
      const int r = i / SB, c = i % SB;
      const bool kin = k0 + c < d;
      xs[r][c] = (xrow[r] >= 0 && kin) ? x[static_cast<size_t>(xrow[r]) * d + k0 + c] : 0.f;
      const bool nin = n0 + r < h;
      as[r][c] = (nin && kin) ? W1[static_cast<size_t>(n0 + r) * d + k0 + c] : 0.f;
      bs[r][c] = (nin && kin) ? W3[static_cast<size_t>(n0 + r) * d + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SB; ++kk) {
      const float xv = xs[ty][kk];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        g[c] = fmaf(xv, as[tx * 4 + c][kk], g[c]);
        u[c] = fmaf(xv, bs[tx * 4 + c][kk], u[c]);
      }
    }
    __syncthreads();
  }
  if (ty < valid) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int n = n0 + tx * 4 + c;
      if (n < h) {
        const size_t r = static_cast<size_t>(row0 + ty);
        H[r * h + n] = g[c] / (1.0f + expf(-g[c])) * u[c];
        if (GU) {   // training forward: G | U for the backward
          GU[r * 2 * h + n] = g[c];
          GU[r * 2 * h + h + n] = u[c];
        }
      }
    }
  }
}

// y[s, n] = (sum_j H[s,j] w2[e,n,j]) * row_scale[s]
__global__ void __launch_bounds__(256) swiglu_down_f32_kernel(
    const float* __restrict__ H, const int32_t* __restrict__ offsets,
    const float* __restrict__ w2, const float* __restrict__ row_scale, int N, int d, int h, int E,
    float* __restrict__ y, int* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int off[kMaxExperts + 1], cum[kMaxExperts + 1];
  __shared__ float hs[SB][SB + 1], ws[SB][SB + 1];
  if (!simt_schedule(offsets, E, N, off, cum, status)) return;
  const int tile = blockIdx.x;
  if (tile >= cum[E]) return;
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  int row0, valid;
  simt_locate(off, cum, E, tile, row0, valid);
  const int n0 = blockIdx.y * SB;
  const int ty = threadIdx.x >> 3, tx = threadIdx.x & 7;
  const float* W2 = w2 + static_cast<size_t>(e) * d * h;
  float acc[4] = {0, 0, 0, 0};
  for (int k0 = 0; k0 < h; k0 += SB) {
    for (int i = threadIdx.x; i < SB * SB; i += blockDim.x) {
      const int r = i / SB, c = i % SB;
      const bool kin = k0 + c < h;
      hs[r][c] = (r < valid && kin) ? H[static_cast<size_t>(row0 + r) * h + k0 + c] : 0.f;
      ws[r][c] = (n0 + r < d && kin) ? W2[static_cast<size_t>(n0 + r) * h + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SB; ++kk) {
      const float hv = hs[ty][kk];
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] = fmaf(hv, ws[tx * 4 + c][kk], acc[c]);
    }
    __syncthreads();
  }
  if (ty < valid) {
    const float sc = row_scale ? row_scale[row0 + ty] : 1.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int n = n0 + tx * 4 + c;
      if (n < d) y[static_cast<size_t>(row0 + ty) * d + n] = acc[c] * sc;
    }
  }
}

// ------------------------------------------------------------------ backward
// One fp32 contraction per segment on CUDA cores:
//   C_e[m, n] (+)= sum_k A(m, k) B_e(n, k)
// with (m, k) of A at A[m sam + k sak], (n, k) of B_e at B[e b_e + n sbn +
// k sbk] and (m, n) of C_e at C[e c_e + m scm + n scn].  seg_k = 0: segment
// e holds the rows m (tokens) and B_e is expert e's weight (K fixed);
// seg_k = 1: segment e holds the reduction rows k (tokens) and C_e is expert
// e's weight gradient (M and N fixed; an empty segment gives zeros).
// offsets NULL: one segment of all rows.  With dgu set (seg_k = 0, N = h)
// the epilogue is the SwiGLU derivative: acc = dA and, from gu = G | U,
//   dgu[m, n] = dA u silu'(g),  dgu[m, h + n] = dA silu(g).
struct SegGemmF32 {
  const float* A;
  long long sam, sak;
  const float* B;
  long long sbn, sbk, b_e;
  float* C;
  long long scm, scn, c_e;
  int M, N, K;   // seg_k = 0: M = rows; seg_k = 1: K = rows
  int E;
  const int32_t* offsets;
  int seg_k, accumulate;
  const float* gu;
  float* dgu;
};

__global__ void __launch_bounds__(256) seg_gemm_f32_kernel(SegGemmF32 p, int* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int off[kMaxExperts + 1], cum[kMaxExperts + 1];
  __shared__ float as[SB][SB + 1], bs[SB][SB + 1];
  const int rows = p.seg_k ? p.K : p.M;
  const int E = p.offsets ? p.E : 1;
  if (p.offsets) {
    if (!simt_schedule(p.offsets, E, rows, off, cum, status)) return;
  } else {
    if (threadIdx.x == 0) {
      off[0] = 0;
      off[1] = rows;
      cum[0] = 0;
      cum[1] = cdiv(rows, SB);
    }
    __syncthreads();
  }
  int e, m0, mvalid, k_lo, k_hi;
  if (!p.seg_k) {
    const int tile = blockIdx.x;
    if (tile >= cum[E]) return;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cum[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    simt_locate(off, cum, E, tile, m0, mvalid);
    k_lo = 0;
    k_hi = p.K;
  } else {
    const int mtiles = cdiv(p.M, SB);
    e = blockIdx.x / mtiles;
    if (e >= E) return;
    m0 = (blockIdx.x - e * mtiles) * SB;
    mvalid = min(SB, p.M - m0);
    k_lo = off[e];
    k_hi = off[e + 1];
  }
  const int n0 = blockIdx.y * SB;
  const int ty = threadIdx.x >> 3, tx = threadIdx.x & 7;   // row ty, columns tx*4..+3
  const float* Be = p.B + static_cast<long long>(e) * p.b_e;
  float acc[4] = {0, 0, 0, 0};
  for (int k0 = k_lo; k0 < k_hi; k0 += SB) {
    // the element pairs of a tile are walked along whichever index is
    // contiguous in memory
    for (int i = threadIdx.x; i < SB * SB; i += blockDim.x) {
      int r, c;
      if (p.sak == 1) { r = i / SB; c = i % SB; } else { c = i / SB; r = i % SB; }
      const int k = k0 + c;
      as[r][c] = (r < mvalid && k < k_hi) ? p.A[(m0 + r) * p.sam + k * p.sak] : 0.f;
      if (p.sbk == 1) { r = i / SB; c = i % SB; } else { c = i / SB; r = i % SB; }
      const int kb = k0 + c;
      bs[r][c] = (n0 + r < p.N && kb < k_hi) ? Be[(n0 + r) * p.sbn + kb * p.sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SB; ++kk) {
      const float av = as[ty][kk];
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] = fmaf(av, bs[tx * 4 + c][kk], acc[c]);
    }
    __syncthreads();
  }
  if (ty >= mvalid) return;
  const long long m = m0 + ty;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int n = n0 + tx * 4 + c;
    if (n >= p.N) continue;
    if (p.dgu) {
      const long long r = m * 2 * p.N;
      const float g = p.gu[r + n], u = p.gu[r + p.N + n];
      const float sg = 1.0f / (1.0f + expf(-g));
      p.dgu[r + n] = acc[c] * u * (sg * (1.0f + g * (1.0f - sg)));
      p.dgu[r + p.N + n] = acc[c] * (g * sg);
    } else {
      float* dst = p.C + static_cast<long long>(e) * p.c_e + m * p.scm + n * p.scn;
      *dst = p.accumulate ? *dst + acc[c] : acc[c];
    }
  }
}

cudaError_t launch_seg_gemm_f32(const SegGemmF32& p, int* status, cudaStream_t s) {
  const int ny = cdiv(p.N, SB);
  dim3 grid;
  if (!p.seg_k) {
    grid = dim3(cdiv(p.M, SB) + (p.offsets ? p.E : 1), ny);
  } else {
    grid = dim3((p.offsets ? p.E : 1) * cdiv(p.M, SB), ny);
  }
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  return launch_k(seg_gemm_f32_kernel, grid, dim3(256), 0, s, p, status);
}

SegGemmF32 seg_gemm(const float* A, long long sam, long long sak, const float* B, long long sbn,
                    long long sbk, long long b_e, float* C, long long scm, long long scn,
                    long long c_e, int M, int N, int K, int E, const int32_t* offsets, int seg_k,
                    int accumulate) {
  SegGemmF32 p{};
  p.A = A;
  p.sam = sam;
  p.sak = sak;
  p.B = B;
  p.sbn = sbn;
  p.sbk = sbk;
  p.b_e = b_e;
  p.C = C;
  p.scm = scm;
  p.scn = scn;
  p.c_e = c_e;
  p.M = M;
  p.N = N;
  p.K = K;
  p.E = E;
  p.offsets = offsets;
  p.seg_k = seg_k;
  p.accumulate = accumulate;
  return p;
}

}  // namespace

cudaError_t launch_swiglu_simt_f32_train(const float* x_perm, const int32_t* offsets,
                                         const float* w1, const float* w3, const float* w2,
                                         int N, int d, int h, int E, float* y, float* H,
                                         float* GU, int* status, cudaStream_t s) {
  const int max_tiles = cdiv(N, SB) + E;
  launch_k(swiglu_up_f32_kernel, dim3(max_tiles, cdiv(h, SB)), dim3(256), 0, s, x_perm,
           nullptr, N, offsets, w1, w3, N, d, h, E, H, GU, status);
  launch_k(swiglu_down_f32_kernel, dim3(max_tiles, cdiv(d, SB)), dim3(256), 0, s, H, offsets, w2,
           nullptr, N, d, h, E, y, status);
  return cudaGetLastError();
}

// Backward of the fp32 grouped SwiGLU, per expert segment S with rows s:
// dA = dY w2[e] with the SwiGLU derivative in its epilogue (-> dGU), dX = dG
// w1[e] + dU w3[e], dw1[e] = dG^T S, dw3[e] = dU^T S, dw2[e] = dY^T H.
cudaError_t launch_swiglu_bwd_simt_f32(const float* x_perm, const int32_t* offsets,
                                       const float* w1, const float* w3, const float* w2,
                                       const float* H, const float* GU, const float* dY, int N,
                                       int d, int h, int E, float* dX, float* dW1, float* dW3,
                                       float* dW2, float* dGU, int* status, cudaStream_t s) {
  const long long hd = static_cast<long long>(h) * d;
  // dA[s, j] = sum_i dY[s, i] w2[e][i, j]
  SegGemmF32 p = seg_gemm(dY, d, 1, w2, 1, h, hd, nullptr, 0, 0, 0, N, h, d, E, offsets, 0, 0);
  p.gu = GU;
  p.dgu = dGU;
  cudaError_t e = launch_seg_gemm_f32(p, status, s);
  // dX[s, i] = sum_j dG[s, j] w1[e][j, i] + dU[s, j] w3[e][j, i]
  if (e == cudaSuccess)
    e = launch_seg_gemm_f32(seg_gemm(dGU, 2LL * h, 1, w1, 1, d, hd, dX, d, 1, 0, N, d, h, E,
                                     offsets, 0, 0),
                            status, s);
  if (e == cudaSuccess)
    e = launch_seg_gemm_f32(seg_gemm(dGU + h, 2LL * h, 1, w3, 1, d, hd, dX, d, 1, 0, N, d, h, E,
                                     offsets, 0, 1),
                            status, s);
  // dw1[e][j, i] = sum_s dG[s, j] x[s, i]; dw3 with dU
  if (e == cudaSuccess)
    e = launch_seg_gemm_f32(seg_gemm(dGU, 1, 2LL * h, x_perm, 1, d, 0, dW1, d, 1, hd, h, d, N, E,
                                     offsets, 1, 0),
                            status, s);
  if (e == cudaSuccess)
    e = launch_seg_gemm_f32(seg_gemm(dGU + h, 1, 2LL * h, x_perm, 1, d, 0, dW3, d, 1, hd, h, d,
                                     N, E, offsets, 1, 0),
                            status, s);
  // dw2[e][i, j] = sum_s dY[s, i] H[s, j]
  if (e == cudaSuccess)
    e = launch_seg_gemm_f32(seg_gemm(dY, 1, d, H, 1, h, 0, dW2, h, 1, hd, d, h, N, E, offsets, 1,
                                     0),
                            status, s);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

// fp32 gate gradients for dz [T, E] fp32: dw_router = dz^T x [E, d] and
// dx = dz w_router [T, d], each optional.
cudaError_t launch_gate_backward_f32(const float* dz, const float* x, const float* w_router,
                                     int T, int d, int E, float* dw_router, float* dx,
                                     cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  // dw_router[e, i] = sum_t dz[t, e] x[t, i]
  if (dw_router)
    e = launch_seg_gemm_f32(seg_gemm(dz, 1, E, x, 1, d, 0, dw_router, d, 1, 0, E, d, T, 1,
                                     nullptr, 1, 0),
                            nullptr, s);
  // dx[t, i] = sum_e dz[t, e] w_router[e, i]
  if (e == cudaSuccess && dx)
    e = launch_seg_gemm_f32(seg_gemm(dz, E, 1, w_router, 1, d, 0, dx, d, 1, 0, T, d, E, 1,
                                     nullptr, 0, 0),
                            nullptr, s);
  return e;
}

cudaError_t launch_swiglu_simt_f32(const float* x_perm, const int32_t* offsets,
                                   const float* w1, const float* w3, const float* w2,
                                   const float* row_scale, int N, int d, int h, int E, float* y,
                                   float* H, int* status, cudaStream_t s) {
  return launch_swiglu_simt_f32_gather(x_perm, N, nullptr, offsets, w1, w3, w2, row_scale, N, d,
                                       h, E, y, H, status, s);
}

cudaError_t launch_swiglu_simt_f32_gather(const float* x, int x_rows, const int32_t* src_row,
                                          const int32_t* offsets, const float* w1,
                                          const float* w3, const float* w2,
                                          const float* row_scale, int N, int d, int h, int E,
                                          float* y, float* H, int* status, cudaStream_t s) {
  const int max_tiles = cdiv(N, SB) + E;   // upper bound over all segmentations
  dim3 g1(max_tiles, cdiv(h, SB));
  launch_k(swiglu_up_f32_kernel, dim3(g1), dim3(256), 0, s, x, src_row, x_rows, offsets, w1, w3, N, d, h, E, H,
                                          nullptr, status);
  dim3 g2(max_tiles, cdiv(d, SB));
  launch_k(swiglu_down_f32_kernel, dim3(g2), dim3(256), 0, s, H, offsets, w2, row_scale, N, d, h, E, y, status);
  return cudaGetLastError();
}

}  // namespace moe
