// fp32 grouped SwiGLU on CUDA cores ([HP] _run_experts_for_loop semantics):
// fp32 in, fp32 accumulate, fp32 out.  Used for fp32 layers, where tensor
// cores (tf32) could not meet a 1e-5 relative tolerance.  32 x 32 output
// tiles inside one expert segment; the tile schedule is built per block from
// the device offsets, so no host synchronisation is needed.
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
    int* status) {
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
      if (n < h) H[static_cast<size_t>(row0 + ty) * h + n] = g[c] / (1.0f + expf(-g[c])) * u[c];
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

}  // namespace

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
                                          status);
  dim3 g2(max_tiles, cdiv(d, SB));
  launch_k(swiglu_down_f32_kernel, dim3(g2), dim3(256), 0, s, H, offsets, w2, row_scale, N, d, h, E, y, status);
  return cudaGetLastError();
}

}  // namespace moe
