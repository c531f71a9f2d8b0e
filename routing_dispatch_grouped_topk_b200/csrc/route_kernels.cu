// CUDA-core kernels of libmoe: dispatch (histogram, scan, stable rank,
// 16-byte row scatter), EP local regroup, combine, and the fp32 router.
//
// Dispatch follows [HP] MoE.permutation: the expert-major order is a stable
// sort of the flat expert ids, computed here without a sort and without
// global atomics: per-block histograms, one scan over (block, bin), then a
// warp-synchronous stable rank (match.any + popc) inside each block.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {

// --------------------------------------------------------------- dispatch

// K1: histogram of the keys of each block of `tb` tokens, stored bin-major
// (blk[bin * nblk + block]) so that K2 scans contiguous columns.
// Every block also records in flags[block] (after the table and the column
// scan's ticket) whether it met an expert id outside [0, E); the column
// scan's last block turns the flags into the status word, so the dispatch
// entry points need no cleared status word before them.
__global__ void dispatch_hist_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int R,
                                     int L, int S, int tb, int nbins, int32_t* __restrict__ blk) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int hist[];
  __shared__ int bad;
  const int nblk = gridDim.x;
  int32_t* ticket = blk + static_cast<size_t>(nbins) * nblk;
  // the column scan's completion ticket sits after the table
  if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0;
  if (threadIdx.x == 0) bad = 0;
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * tb;
  const int t1 = min(T, t0 + tb);
  const long long f0 = 1LL * t0 * k, f1 = 1LL * t1 * k;
  for (long long f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
    const int e = idx[f];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {
      bad |= e != kDroppedCopy;   // a copy the capacity policy dropped is no error
      continue;
    }
    atomicAdd(&hist[dispatch_key(e, static_cast<int>(f / k), R, L, S)], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nbins; i += blockDim.x)
    blk[static_cast<size_t>(i) * nblk + blockIdx.x] = hist[i];
  if (threadIdx.x == 0) ticket[1 + blockIdx.x] = bad;
}

// Block-wide exclusive scan of `n` ints held in shared memory `a` (in place);
// returns the total.  blockDim.x must be a multiple of 32 and <= 1024.
__device__ int block_exclusive_scan(int* a, int n, int* warp_sums) {
  const int nt = blockDim.x;
  const int per = (n + nt - 1) / nt;
  const int i0 = min(n, threadIdx.x * per), i1 = min(n, i0 + per);
  int local = 0;
  for (int i = i0; i < i1; ++i) local += a[i];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, sh);
    if (lane >= sh) incl += v;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = nt >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
    int si = s;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, si, sh);
      if (lane >= sh) si += v;
    }
    if (lane < nw) warp_sums[lane] = si - s;   // exclusive warp offsets
    if (lane == 31) warp_sums[32] = si;        // total
  }
  __syncthreads();
  int run = warp_sums[w] + incl - local;
  for (int i = i0; i < i1; ++i) {
    const int v = a[i];
    a[i] = run;
    run += v;
  }
  const int total = warp_sums[32];
  __syncthreads();
  return total;
}

// Exclusive block-wide scan of one value per thread; *total receives the sum.
// Every thread of the block must call it.
__device__ int block_scan_value(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int sh = 1; sh < 32; sh <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, sh);
    if (lane >= sh) incl += u;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    const int s = lane < nw ? warp_sums[lane] : 0;
    int si = s;
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, si, sh);
      if (lane >= sh) si += u;
    }
    if (lane < nw) warp_sums[lane] = si - s;
    if (lane == 31) warp_sums[32] = si;
  }
  __syncthreads();
  const int ex = warp_sums[w] + incl - v;
  *total = warp_sums[32];
  __syncthreads();
  return ex;
}

// K2: for every bin (one block per bin, grid-stride), the exclusive prefix of
// its column over the token blocks, in place; the column total is counts[bin].
// The last block to finish (a ticket counter after the table, zeroed by the
// kernel that wrote the table) scans the totals into offsets[0..nbins] and
// marks the slots that invalid expert ids left empty (src_row = -1): every
// scatter block then reads only the entries of the bins it touches.
__global__ void dispatch_colscan_kernel(int32_t* __restrict__ blk, int nblk, int nbins,
                                        int32_t* __restrict__ counts,
                                        int32_t* __restrict__ offsets,
                                        int32_t* __restrict__ src_row, long long n_slots,
                                        int* status_out) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int osm[];      // nbins (last block only)
  __shared__ int wsum[33];
  __shared__ int last;
  for (int bin = blockIdx.x; bin < nbins; bin += gridDim.x) {
    int32_t* col = blk + static_cast<size_t>(bin) * nblk;
    int carry = 0;
    for (int base = 0; base < nblk; base += blockDim.x) {
      const int i = base + threadIdx.x;
      const int v = i < nblk ? col[i] : 0;
      int tot;
      const int ex = block_scan_value(v, wsum, &tot);
      if (i < nblk) col[i] = carry + ex;
      carry += tot;
    }
    if (threadIdx.x == 0) counts[bin] = carry;
  }
  // completion ticket: the block that takes the last one sees every count
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int* ticket = blk + static_cast<size_t>(nbins) * nblk;
    last = atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) osm[i] = __ldcg(counts + i);
  __syncthreads();
  const int total = block_exclusive_scan(osm, nbins, wsum);
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) offsets[i] = osm[i];
  if (threadIdx.x == 0) offsets[nbins] = total;
  for (long long sl = total + threadIdx.x; sl < n_slots; sl += blockDim.x) src_row[sl] = -1;
  // the entry point's status word, from the histogram blocks' flags
  if (status_out) {
    const int32_t* flags = blk + static_cast<size_t>(nbins) * nblk + 1;
    int any = 0;
    for (int b = threadIdx.x; b < nblk; b += blockDim.x) any |= __ldcg(flags + b);
    any = __syncthreads_or(any);
    if (threadIdx.x == 0) *status_out = any ? MOE_DEV_BAD_EXPERT : 0;
  }
}

// Eight bf16 or four fp32 values times w (fp32 product, rounded once).
__device__ __forceinline__ uint4 scale_vec(uint4 v, float w, int bf16) {
  uint32_t u[4] = {v.x, v.y, v.z, v.w};
  if (bf16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = pack_bf16x2(bf16_lo(u[i]) * w, bf16_hi(u[i]) * w);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * w);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

// K3: stable slot of every copy, then the row copies (all warps): each token
// row is read once and written to its k slots with 16-byte stores.  A block
// reads only what its own copies need: for every key it touches, the bin's
// offset plus the block's column prefix; warp 0 then ranks the copies in
// flat order (match.any + popc), so equal keys keep their flat order.
__global__ void __launch_bounds__(1024) dispatch_scatter_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ idx,
                                        int T, int k, int E, int R, int L, int S, int tb,
                                        int nbins, const int32_t* __restrict__ blk,
                                        const int32_t* __restrict__ offsets,
                                        int32_t* __restrict__ src_row,
                                        int32_t* __restrict__ dst_pos, uint4* __restrict__ x_perm,
                                        int row_vec, const float* __restrict__ row_w, int bf16,
                                        int* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int sm[];
  int* run = sm;                   // nbins (only the touched keys are set)
  int* slot = sm + nbins;          // tb * k: the key, then the slot of each copy
  const int nblk = gridDim.x;
  const int t0 = blockIdx.x * tb;
  const int t1 = min(T, t0 + tb);
  const int nf = (t1 - t0) * k;
  const long long f0 = 1LL * t0 * k;
  for (int i = threadIdx.x; i < nf; i += blockDim.x) {
    const int e = idx[f0 + i];
    int key = -1;
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
      key = dispatch_key(e, static_cast<int>((f0 + i) / k), R, L, S);
      // every copy with this key writes the same base (benign)
      run[key] = offsets[key] + blk[static_cast<size_t>(key) * nblk + blockIdx.x];
    }
    slot[i] = key;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const unsigned lt = (1u << lane) - 1u;
    for (int c0 = 0; c0 < nf; c0 += 32) {
      const int i = c0 + lane;
      const int key = i < nf ? slot[i] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, key >= 0 ? key : -1 - lane);
      const int rank = __popc(peers & lt);
      const int leader = __ffs(peers) - 1;
      int sl = -1;
      if (key >= 0) sl = run[key] + rank;
      // a slot outside [0, T k) can only come from a table overwritten while
      // the call ran: skip the copy, flag it, keep every access in bounds
      if (static_cast<unsigned long long>(static_cast<unsigned>(sl)) >= 1ULL * T * k && sl != -1) {
        sl = -1;
        if (status) set_status(status, MOE_DEV_BAD_OFFSETS);
      }
      __syncwarp();
      if (key >= 0 && lane == leader) run[key] += __popc(peers);
      __syncwarp();
      if (i < nf) {
        const long long f = f0 + i;
        dst_pos[f] = sl;
        slot[i] = sl;
        if (sl >= 0) src_row[sl] = static_cast<int>(f / k);
      }
    }
  }
  __syncthreads();
  if (!x_perm) return;
  // Row copies: a warp per token; each lane issues up to eight 16-byte loads
  // of the row before storing them to the token's k slots.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int t = t0 + warp; t < t1; t += nw) {
    const uint4* src = x + static_cast<size_t>(t) * row_vec;
    const int* sl = slot + (t - t0) * k;
    for (int c0 = 0; c0 < row_vec; c0 += 256) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vec) v[u] = src[c];
      }
      for (int j = 0; j < k; ++j) {
        const int s = sl[j];
        if (s < 0) continue;
        uint4* dst = x_perm + static_cast<size_t>(s) * row_vec;
        // [HP] MoE.forward with score_before_experts: routed row times its weight
        const float wj = row_w ? row_w[static_cast<size_t>(t) * k + j] : 1.0f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < row_vec) dst[c] = row_w ? scale_vec(v[u], wj, bf16) : v[u];
        }
      }
    }
  }
}

DispatchPlan make_dispatch_plan(int T, int E, int top_k, int R, int max_tb) {
  DispatchPlan p{};
  p.T = T;
  p.k = top_k;
  p.E = E;
  p.R = R;
  p.L = E / R;
  p.S = R > 1 ? std::max(1, cdiv(T, R)) : std::max(T, 1);
  p.nbins = E * R;
  // About four blocks per SM, so that the row copies balance across SMs
  // (small blocks also keep the warp-serial ranking short), and at most
  // 2^17 entries in the histogram table: its write and its column scan cost
  // nblk * nbins, which with the E * R bins of the rank-major layout would
  // otherwise outweigh the copies.
  int tb = 8;
  while (tb < std::min(128, max_tb) &&
         (cdiv(T, tb * 2) >= 4 * 148 ||
          static_cast<long long>(cdiv(T, tb)) * p.nbins > (1LL << 17)))
    tb *= 2;
  p.tb = tb;
  p.nblk = std::max(1, cdiv(T, tb));
  return p;
}

size_t dispatch_ws_bytes(const DispatchPlan& p) {
  // the histogram table [nbins, nblk], the column scan's ticket, then one
  // bad-id flag per block
  return align_up((static_cast<size_t>(p.nblk) * p.nbins + 1 + p.nblk) * sizeof(int32_t), 256);
}

cudaError_t launch_dispatch(const DispatchPlan& p, const void* x, const int32_t* topk_idx,
                            int d, moe_dtype_t dt, int32_t* counts, int32_t* offsets,
                            int32_t* src_row, int32_t* dst_pos, void* x_perm, void* ws,
                            int* status, cudaStream_t s, bool hist_done, const float* row_w,
                            bool own_status) {
  int32_t* blk = static_cast<int32_t*>(ws);
  if (p.T == 0) {
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * p.nbins, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (p.nbins + 1), s);
    if (e == cudaSuccess && own_status) e = cudaMemsetAsync(status, 0, sizeof(int), s);
    return e;
  }
  if (!hist_done)
    launch_k(dispatch_hist_kernel, dim3(p.nblk), dim3(256), p.nbins * sizeof(int), s, topk_idx,
             p.T, p.k, p.E, p.R, p.L, p.S, p.tb, p.nbins, blk);
  // own_status: the histogram kernel ran and the colscan writes the whole
  // status word from its flags (the entry points clear nothing first);
  // inside the layer the router wrote the table and the status is shared
  launch_k(dispatch_colscan_kernel, dim3(std::min(p.nbins, num_sms() * 8)), dim3(256),
           p.nbins * sizeof(int), s, blk, p.nblk, p.nbins, counts, offsets, src_row,
           1LL * p.T * p.k, (!hist_done && own_status) ? status : nullptr);
  const int elt = dt == MOE_BF16 ? 2 : 4;
  const int row_vec = d * elt / 16;
  const size_t sm3 = (p.nbins + p.tb * p.k) * sizeof(int);
  // a warp per token row at a time: more warps for larger blocks
  const int threads = std::min(1024, std::max(256, 16 * p.tb));
  launch_k(dispatch_scatter_kernel, dim3(p.nblk), dim3(threads), sm3, s,
           static_cast<const uint4*>(x), topk_idx, p.T, p.k, p.E, p.R, p.L, p.S, p.tb, p.nbins,
           blk, offsets, src_row, dst_pos, static_cast<uint4*>(x_perm), row_vec, row_w,
           dt == MOE_BF16 ? 1 : 0, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- regroup
// One kernel: every block builds the segment tables in shared memory from
// counts_rm (two block scans of S = G*R*L counts), then its warps copy rows
// grid-stride.  Segments are numbered in OUTPUT order o = (g*L + l)*R + r;
// in_start[o] is where segment (g, r, l) starts in the rank-major input,
// out_start[o] (o = 0..S) where it starts in the output; a row's segment is
// found by binary search over out_start in shared memory.  Block 0 writes
// counts_em / offsets_em and the status; if the counts are negative or do
// not add up to `rows`, nothing is copied.
__global__ void __launch_bounds__(256) regroup_kernel(
    const uint4* __restrict__ in, const int32_t* __restrict__ counts_rm, int G, int R, int L,
    int rows, int row_vec, uint4* __restrict__ out, int32_t* __restrict__ counts_em,
    int32_t* __restrict__ offsets_em, int32_t* __restrict__ perm, int32_t* __restrict__ perm_inv,
    int* status, int own_status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int sm[];
  const int S = G * R * L;
  int* a = sm;                 // S: scan scratch
  int* in_start = sm + S;      // S (output numbering)
  int* out_start = sm + 2 * S; // S + 1
  __shared__ int wsum[33];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  // input order (g, r, l): exclusive scan of the counts as given
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const int c = counts_rm[i];
    if (c < 0) bad = 1;
    a[i] = max(c, 0);
  }
  __syncthreads();
  const int total = block_exclusive_scan(a, S, wsum);
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const int g = i / (R * L), r = (i / L) % R, l = i % L;
    in_start[(g * L + l) * R + r] = a[i];
  }
  for (int o = threadIdx.x; o < S; o += blockDim.x) {
    const int g = o / (L * R), l = (o / R) % L, r = o % R;
    out_start[o] = max(counts_rm[(g * R + r) * L + l], 0);
  }
  __syncthreads();
  block_exclusive_scan(out_start, S, wsum);
  if (threadIdx.x == 0) out_start[S] = total;
  __syncthreads();
  const bool ok = (bad == 0) && (total == rows);
  if (blockIdx.x == 0) {
    // block 0 is the only writer: as the call's only kernel it writes the
    // whole status word, inside a longer sequence it adds its bit
    if (threadIdx.x == 0) {
      if (own_status)
        *status = ok ? 0 : MOE_DEV_BAD_COUNTS;
      else if (!ok)
        set_status(status, MOE_DEV_BAD_COUNTS);
    }
    // expert-major counts / offsets: sum over r
    for (int gl = threadIdx.x; gl < G * L; gl += blockDim.x) {
      const int o0 = gl * R;
      counts_em[gl] = out_start[o0 + R] - out_start[o0];
      offsets_em[gl] = out_start[o0];
    }
    if (threadIdx.x == 0) offsets_em[G * L] = total;
  }
  if (!ok) return;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int o = gw; o < rows; o += nw) {
    int lo = 0, hi = S - 1;     // last segment with out_start <= o
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (out_start[mid] <= o) lo = mid; else hi = mid - 1;
    }
    const int src = in_start[lo] + (o - out_start[lo]);
    if (lane == 0) {
      perm[o] = src;
      if (perm_inv) perm_inv[src] = o;
    }
    const uint4* sp = in + static_cast<size_t>(src) * row_vec;
    uint4* dp = out + static_cast<size_t>(o) * row_vec;
    // up to four 16-byte loads per lane in flight before the stores
    for (int c0 = 0; c0 < row_vec; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vec) v[u] = sp[c];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vec) dp[c] = v[u];
      }
    }
  }
}

size_t regroup_ws_bytes(int G, int R, int L) {
  (void)G;
  (void)R;
  (void)L;
  return 0;
}

cudaError_t launch_regroup(const void* in, const int32_t* counts_rm, int G, int R, int L,
                           int rows, int d, moe_dtype_t dt, void* out, int32_t* counts_em,
                           int32_t* offsets_em, int32_t* perm, int32_t* perm_inv, void* ws,
                           int* status, cudaStream_t s, bool own_status) {
  (void)ws;
  const int S = G * R * L;
  const size_t smem = (3 * static_cast<size_t>(S) + 1) * sizeof(int);
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem > 48 * 1024 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(regroup_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         3 * kMaxSegments * 4 + 16);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  const int elt = dt == MOE_BF16 ? 2 : 4;
  const int row_vec = rows > 0 ? d * elt / 16 : 0;
  // one block when there is nothing to copy (the tables are still written)
  const int blocks = rows > 0 ? std::min(cdiv(rows, 8), num_sms() * 4) : 1;
  launch_k(regroup_kernel, dim3(blocks), dim3(256), smem, s, static_cast<const uint4*>(in),
           counts_rm, G, R, L, rows, row_vec, static_cast<uint4*>(out), counts_em, offsets_em,
           perm, perm_inv, status, own_status ? 1 : 0);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- combine
// out[t] = sum_j w[t,j] * y[r(t,j)] in fp32, one warp per token.  Lane j < k
// reads the position and weight of copy j once; they are broadcast by
// shuffle.  Each lane walks the 16-byte chunks of the row and issues the k
// loads of a chunk before accumulating them in order j = 0..k-1.
// Weighted sum over the k copies of one 16-byte chunk (fp32, j in order),
// plus the shared expert's chunk, rounded once.
template <bool BF16, int KMAX>
__device__ __forceinline__ uint4 combine_chunk(const uint4 (&v)[KMAX], const float (&wt)[KMAX],
                                               const int (&pos)[KMAX], int k,
                                               const uint4* shared, const uint4* shared2) {
  float acc[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j >= k || pos[j] < 0) continue;
    const float wj = wt[j];
    if (BF16) {
      acc[0] = fmaf(wj, bf16_lo(v[j].x), acc[0]);
      acc[1] = fmaf(wj, bf16_hi(v[j].x), acc[1]);
      acc[2] = fmaf(wj, bf16_lo(v[j].y), acc[2]);
      acc[3] = fmaf(wj, bf16_hi(v[j].y), acc[3]);
      acc[4] = fmaf(wj, bf16_lo(v[j].z), acc[4]);
      acc[5] = fmaf(wj, bf16_hi(v[j].z), acc[5]);
      acc[6] = fmaf(wj, bf16_lo(v[j].w), acc[6]);
      acc[7] = fmaf(wj, bf16_hi(v[j].w), acc[7]);
    } else {
      acc[0] = fmaf(wj, __uint_as_float(v[j].x), acc[0]);
      acc[1] = fmaf(wj, __uint_as_float(v[j].y), acc[1]);
      acc[2] = fmaf(wj, __uint_as_float(v[j].z), acc[2]);
      acc[3] = fmaf(wj, __uint_as_float(v[j].w), acc[3]);
    }
  }
  // [HP] MoE.forward: out + shared_expert(x); in the backward, the router's
  // and the shared expert's shares of dx
  const uint4* adds[2] = {shared, shared2};
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    if (!adds[a]) continue;
    const uint4 sv = *adds[a];
    if (BF16) {
      acc[0] += bf16_lo(sv.x);
      acc[1] += bf16_hi(sv.x);
      acc[2] += bf16_lo(sv.y);
      acc[3] += bf16_hi(sv.y);
      acc[4] += bf16_lo(sv.z);
      acc[5] += bf16_hi(sv.z);
      acc[6] += bf16_lo(sv.w);
      acc[7] += bf16_hi(sv.w);
    } else {
      acc[0] += __uint_as_float(sv.x);
      acc[1] += __uint_as_float(sv.y);
      acc[2] += __uint_as_float(sv.z);
      acc[3] += __uint_as_float(sv.w);
    }
  }
  if (BF16)
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                    __float_as_uint(acc[3]));
}

template <bool BF16, int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(
    const uint4* __restrict__ y, const int32_t* __restrict__ dst_pos,
    const int32_t* __restrict__ row_map, const float* __restrict__ w, int T, int row_vec, int N,
    int k, const uint4* __restrict__ shared, const uint4* __restrict__ shared2,
    uint4* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
    int my_p = -1;
    float my_w = 0.f;
    if (lane < k) {
      int p = dst_pos[static_cast<size_t>(t) * k + lane];
      if (row_map && static_cast<unsigned>(p) < static_cast<unsigned>(N)) p = row_map[p];
      if (static_cast<unsigned>(p) < static_cast<unsigned>(N)) {
        my_p = p;
        my_w = w ? w[static_cast<size_t>(t) * k + lane] : 1.0f;
      }
    }
    int pos[KMAX];
    float wt[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      pos[j] = __shfl_sync(0xffffffffu, my_p, j);
      wt[j] = __shfl_sync(0xffffffffu, my_w, j);
    }
    uint4* orow = out + static_cast<size_t>(t) * row_vec;
    // Two 16-byte chunks per lane per iteration: 2k row loads in flight.
    for (int c0 = lane; c0 < row_vec; c0 += 64) {
      uint4 v[2][KMAX];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + 32 * h;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (c < row_vec && j < k && pos[j] >= 0)
            v[h][j] = y[static_cast<size_t>(pos[j]) * row_vec + c];
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c0 + 32 * h;
        if (c >= row_vec) break;
        const size_t o = static_cast<size_t>(t) * row_vec + c;
        orow[c] = combine_chunk<BF16, KMAX>(v[h], wt, pos, k, shared ? shared + o : nullptr,
                                            shared2 ? shared2 + o : nullptr);
      }
    }
  }
}

template <bool BF16>
static void combine_launch(const uint4* y, const int32_t* dst_pos, const int32_t* row_map,
                           const float* w, int T, int row_vec, int N, int k,
                           const uint4* shared, const uint4* shared2, uint4* out, int blocks,
                           cudaStream_t s) {
  if (k <= 1)
    launch_k(combine_kernel<BF16, 1>, dim3(blocks), dim3(256), 0, s, y, dst_pos, row_map, w, T, row_vec, N, k, shared, shared2, out);
  else if (k <= 2)
    launch_k(combine_kernel<BF16, 2>, dim3(blocks), dim3(256), 0, s, y, dst_pos, row_map, w, T, row_vec, N, k, shared, shared2, out);
  else if (k <= 4)
    launch_k(combine_kernel<BF16, 4>, dim3(blocks), dim3(256), 0, s, y, dst_pos, row_map, w, T, row_vec, N, k, shared, shared2, out);
  else if (k <= 8)
    launch_k(combine_kernel<BF16, 8>, dim3(blocks), dim3(256), 0, s, y, dst_pos, row_map, w, T, row_vec, N, k, shared, shared2, out);
  else
    launch_k(combine_kernel<BF16, 16>, dim3(blocks), dim3(256), 0, s, y, dst_pos, row_map, w, T, row_vec, N, k, shared, shared2, out);
}

cudaError_t launch_combine(const void* y, const int32_t* dst_pos, const int32_t* row_map,
                           const float* topk_w, int T, int d, int N, int top_k, moe_dtype_t dt,
                           void* out, cudaStream_t s, const void* shared,
                           const void* shared2) {
  if (T == 0) return cudaSuccess;
  const int elt = dt == MOE_BF16 ? 2 : 4;
  const int row_vec = d * elt / 16;
  const int blocks = std::min(cdiv(T, 8), num_sms() * 8);
  const uint4* sh = static_cast<const uint4*>(shared);
  const uint4* sh2 = static_cast<const uint4*>(shared2);
  if (dt == MOE_BF16)
    combine_launch<true>(static_cast<const uint4*>(y), dst_pos, row_map, topk_w, T, row_vec, N,
                         top_k, sh, sh2, static_cast<uint4*>(out), blocks, s);
  else
    combine_launch<false>(static_cast<const uint4*>(y), dst_pos, row_map, topk_w, T, row_vec, N,
                          top_k, sh, sh2, static_cast<uint4*>(out), blocks, s);
  return cudaGetLastError();
}

// -------------------------------------------------------- router backward
// Gradient of the routing weights with respect to the gate logits, one warp
// per token (expert i lives in lane i % 32, register slot i / 32).  With s
// the scores (softmax or sigmoid of the saved fp32 logits), S the selected
// experts and c the route scale: w_j = c s_j / sum_S s (renormalised) or
// c s_j, so ds_j = c (g_j - sum_S g s / sum_S s) / sum_S s or c g_j on S,
// 0 elsewhere; dz = s (ds - <s, ds>) (softmax) or ds s (1 - s) (sigmoid).
// Writes dz in fp32 (dz32, optional) and bf16 (dz16, optional; the operand
// of the gate's gradient GEMMs).
template <int EPL>
__global__ void __launch_bounds__(256) router_backward_kernel(
    const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
    const float* __restrict__ g_w, int T, int E, int k, int sigmoid, int renorm, float scale,
    float* __restrict__ dz32, __nv_bfloat16* __restrict__ dz16,
    const int32_t* __restrict__ lb_counts, float lb_scale) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
    const float* row = logits + static_cast<size_t>(t) * E;
    float sv[EPL];
    bool avail[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      avail[i] = lane + 32 * i < E;
      sv[i] = avail[i] ? row[lane + 32 * i] : -INFINITY;
      mx = fmaxf(mx, sv[i]);
    }
    if (sigmoid) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) sv[i] = avail[i] ? 1.0f / (1.0f + expf(-sv[i])) : 0.f;
    } else {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      float den = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        sv[i] = avail[i] ? expf(sv[i] - mx) : 0.f;
        den += sv[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
#pragma unroll
      for (int i = 0; i < EPL; ++i) sv[i] /= den;
    }
    // lane j < k: the j-th selected expert, its upstream gradient and score
    int my_e = -1;
    float my_g = 0.f;
    if (lane < k) {
      const int e = topk_idx[static_cast<size_t>(t) * k + lane];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        my_e = e;
        my_g = g_w[static_cast<size_t>(t) * k + lane];
        // [HP] _compute_load_balance_loss: coef * E * f_e / T, f_e = c_e / (T k)
        if (lb_counts) my_g += lb_scale * static_cast<float>(lb_counts[e]);
      }
    }
    float my_s = 0.f;
    for (int j = 0; j < k; ++j) {
      const int ej = __shfl_sync(0xffffffffu, my_e, j);
      float v = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (i == (ej >> 5)) v = sv[i];
      v = __shfl_sync(0xffffffffu, v, ej & 31);
      if (lane == j) my_s = ej >= 0 ? v : 0.f;
    }
    float tot = my_s, gs = my_g * my_s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, off);
      gs += __shfl_xor_sync(0xffffffffu, gs, off);
    }
    const float my_ds = my_e < 0 ? 0.f : (renorm ? scale * (my_g - gs / tot) / tot : scale * my_g);
    float ds[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) ds[i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int ej = __shfl_sync(0xffffffffu, my_e, j);
      const float dj = __shfl_sync(0xffffffffu, my_ds, j);
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == ej) ds[i] = dj;
    }
    float c = 0.f;
    if (!sigmoid) {
      c = my_s * my_ds;   // <s, ds> over the selected experts
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if (!avail[i]) continue;
      const float dz = sigmoid ? ds[i] * sv[i] * (1.0f - sv[i]) : sv[i] * (ds[i] - c);
      const size_t o = static_cast<size_t>(t) * E + lane + 32 * i;
      if (dz32) dz32[o] = dz;
      if (dz16) dz16[o] = __float2bfloat16_rn(dz);
    }
  }
}

cudaError_t launch_router_backward(const float* logits, const int32_t* topk_idx,
                                   const float* d_topk_w, int T, int E, int top_k, int sigmoid,
                                   int renorm, float scale, float* dz32, void* dz16,
                                   cudaStream_t s, const int32_t* lb_counts, float lb_scale) {
  if (T == 0) return cudaSuccess;
  const int blocks = std::min(cdiv(T, 8), num_sms() * 8);
  __nv_bfloat16* d16 = static_cast<__nv_bfloat16*>(dz16);
  if (E <= 32)
    launch_k(router_backward_kernel<1>, dim3(blocks), dim3(256), 0, s, logits, topk_idx, d_topk_w, T, E, top_k, sigmoid, renorm, scale, dz32, d16, lb_counts, lb_scale);
  else if (E <= 64)
    launch_k(router_backward_kernel<2>, dim3(blocks), dim3(256), 0, s, logits, topk_idx, d_topk_w, T, E, top_k, sigmoid, renorm, scale, dz32, d16, lb_counts, lb_scale);
  else if (E <= 128)
    launch_k(router_backward_kernel<4>, dim3(blocks), dim3(256), 0, s, logits, topk_idx, d_topk_w, T, E, top_k, sigmoid, renorm, scale, dz32, d16, lb_counts, lb_scale);
  else if (E <= 256)
    launch_k(router_backward_kernel<8>, dim3(blocks), dim3(256), 0, s, logits, topk_idx, d_topk_w, T, E, top_k, sigmoid, renorm, scale, dz32, d16, lb_counts, lb_scale);
  else
    launch_k(router_backward_kernel<16>, dim3(blocks), dim3(256), 0, s, logits, topk_idx, d_topk_w, T, E, top_k, sigmoid, renorm, scale, dz32, d16, lb_counts, lb_scale);
  return cudaGetLastError();
}

// ------------------------------------------------------- capacity drop
// [PF] PaddleFormers moe_gate.py, _probs_drop_policy: a token keeps its
// assignment to an expert when it is routed there and its score is among the
// top `capacity` scores for that expert (ranked over the expert's routed
// copies; equal scores to the lower token).  Every copy gets a unique 64-bit
// key, (score, then the token reversed), and one block per expert finds the
// capacity-th largest key of its copies by an 8-bit radix select (eight
// passes over the keys it gathered in shared memory in one scan of the flat
// copy list, or over that list when they do not fit); the copies below it
// are dropped.
__device__ __forceinline__ unsigned long long capacity_key(float s, int t) {
  const unsigned hi = static_cast<unsigned>(score_key(s != s ? -INFINITY : s)) ^ 0x80000000u;
  return (static_cast<unsigned long long>(hi) << 32) | (0xFFFFFFFFu - static_cast<unsigned>(t));
}

// An expert's routed copies gathered in shared memory by the select kernel
// (more than this: its passes scan the flat copy list instead).
constexpr int kCapKeys = 4096;

// Warp 0 of the select kernel: the bin of hist[0..255] (taken from the top)
// that holds the want-th largest key, and how many keys lie in higher bins.
// Lane l holds bins 8l .. 8l+7; a suffix sum over the lanes finds the lane,
// its own bins the bin.
__device__ __forceinline__ void capacity_find_bin(const unsigned* hist, int want, int& bin,
                                                  int& above) {
  const int lane = threadIdx.x & 31;
  unsigned c[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = hist[8 * lane + j];
    sum += c[j];
  }
  unsigned suf = sum;   // keys in bins >= 8 lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned v = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += v;
  }
  const unsigned w = static_cast<unsigned>(want);
  const unsigned excl = suf - sum;   // keys in higher lanes' bins
  const unsigned ball = __ballot_sync(0xffffffffu, excl < w && w <= suf);
  const int owner = __ffs(ball) - 1;
  int b = 0, a = 0;
  if (lane == owner) {
    unsigned cum = excl;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      if (cum + c[j] >= w) {
        b = 8 * lane + j;
        a = static_cast<int>(cum);
        break;
      }
      cum += c[j];
    }
  }
  bin = __shfl_sync(0xffffffffu, b, owner & 31);
  above = __shfl_sync(0xffffffffu, a, owner & 31);
}

__global__ void __launch_bounds__(512) capacity_select_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ scores, long long n, int k,
    int capacity, unsigned long long* __restrict__ thr, int32_t* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long keys_s[kCapKeys];
  __shared__ unsigned hist[256];
  __shared__ unsigned long long prefix_s;
  __shared__ int want_s, count_s;
  const int e = blockIdx.x;
  if (threadIdx.x == 0) count_s = 0;
  __syncthreads();
  // one scan of the copy list: count the expert's copies, keep their keys
  // while they fit (their order does not matter: the keys are distinct)
  for (long long i = threadIdx.x; i < n; i += blockDim.x)
    if (idx[i] == e) {
      const int p = atomicAdd(&count_s, 1);
      if (p < kCapKeys) keys_s[p] = capacity_key(scores[i], static_cast<int>(i / k));
    }
  __syncthreads();
  const int count = count_s;
  // the copies the expert keeps: all of them, or the `capacity` largest keys
  if (threadIdx.x == 0 && counts) counts[e] = min(count, capacity);
  if (count <= capacity) {   // nothing to drop: keep every key
    if (threadIdx.x == 0) thr[e] = 0ull;
    return;
  }
  const bool in_smem = count <= kCapKeys;
  if (threadIdx.x == 0) {
    prefix_s = 0ull;
    want_s = capacity;   // rank (1 = largest) of the key wanted among those left
  }
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const unsigned long long prefix = prefix_s;
    const unsigned long long hi_mask = shift == 56 ? 0ull : ~0ull << (shift + 8);
    if (in_smem) {
      for (int j = threadIdx.x; j < count; j += blockDim.x) {
        const unsigned long long key = keys_s[j];
        if ((key & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
    } else {
      for (long long i = threadIdx.x; i < n; i += blockDim.x) {
        if (idx[i] != e) continue;
        const unsigned long long key = capacity_key(scores[i], static_cast<int>(i / k));
        if ((key & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      int bin = 0, above = 0;
      capacity_find_bin(hist, want_s, bin, above);
      if (threadIdx.x == 0) {
        prefix_s = prefix | (static_cast<unsigned long long>(bin) << shift);
        want_s -= above;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) thr[e] = prefix_s;   // the capacity-th largest key: keep keys >= it
}

__global__ void capacity_apply_kernel(int32_t* __restrict__ idx, float* __restrict__ w,
                                      const float* __restrict__ scores, long long n, int k, int E,
                                      const unsigned long long* __restrict__ thr) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = idx[i];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) continue;
    const unsigned long long t = thr[e];
    if (t && capacity_key(scores[i], static_cast<int>(i / k)) < t) {
      idx[i] = kDroppedCopy;
      w[i] = 0.f;
    }
  }
}

cudaError_t launch_capacity_drop(int32_t* topk_idx, float* topk_w, const float* scores, int T,
                                 int k, int E, int capacity, unsigned long long* thr,
                                 int32_t* counts, cudaStream_t s) {
  const long long n = 1LL * T * k;
  if (n == 0) return cudaSuccess;
  launch_k(capacity_select_kernel, dim3(E), dim3(512), 0, s, topk_idx, scores, n, k, capacity, thr,
           counts);
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 8LL * num_sms()));
  launch_k(capacity_apply_kernel, dim3(blocks), dim3(256), 0, s, topk_idx, topk_w, scores, n, k,
           E, static_cast<const unsigned long long*>(thr));
  return cudaGetLastError();
}

// counts[e] += number of entries of idx [n] equal to e (entries outside
// [0, E) skipped); counts cleared by the caller.
__global__ void expert_hist_kernel(const int32_t* __restrict__ idx, long long n, int E,
                                   int32_t* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int eh[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) eh[e] = 0;
  __syncthreads();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = idx[i];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&eh[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (eh[e]) atomicAdd(&counts[e], eh[e]);
}

cudaError_t launch_expert_hist(const int32_t* idx, long long n, int E, int32_t* counts,
                               cudaStream_t s) {
  const int blocks = static_cast<int>(std::min<long long>(num_sms(), (n + 1023) / 1024));
  if (blocks > 0)
    launch_k(expert_hist_kernel, dim3(blocks), dim3(256), E * sizeof(int), s, idx, n, E, counts);
  return cudaGetLastError();
}

// ------------------------------------------------------- combine backward
// Gradient of out[t] = sum_j w[t, j] y[p(t, j)] for an upstream dout [T, d]:
// dy[p(t, j)] = w[t, j] dout[t] (one rounding of the fp32 product) and, when
// dw is given, dw[t, j] = <dout[t], y[p(t, j)]> accumulated in fp32.  One warp
// per token; each 16-byte chunk of dout is read once and its k products and
// k dot-product terms are formed from registers (k + 1 loads in flight).
__device__ __forceinline__ float dot_chunk(uint4 a, uint4 b, int bf16) {
  if (bf16)
    return bf16_lo(a.x) * bf16_lo(b.x) + bf16_hi(a.x) * bf16_hi(b.x) +
           bf16_lo(a.y) * bf16_lo(b.y) + bf16_hi(a.y) * bf16_hi(b.y) +
           bf16_lo(a.z) * bf16_lo(b.z) + bf16_hi(a.z) * bf16_hi(b.z) +
           bf16_lo(a.w) * bf16_lo(b.w) + bf16_hi(a.w) * bf16_hi(b.w);
  return __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
         __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
}

template <bool BF16, int KMAX>
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const uint4* __restrict__ dout, const uint4* __restrict__ y,
    const int32_t* __restrict__ dst_pos, const float* __restrict__ w, int T, int row_vec, int N,
    int k, uint4* __restrict__ dy, float* __restrict__ dw) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
    int my_p = -1;
    float my_w = 0.f;
    if (lane < k) {
      const int p = dst_pos[static_cast<size_t>(t) * k + lane];
      if (static_cast<unsigned>(p) < static_cast<unsigned>(N)) {
        my_p = p;
        my_w = w ? w[static_cast<size_t>(t) * k + lane] : 1.0f;
      }
    }
    int pos[KMAX];
    float wt[KMAX], dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      pos[j] = __shfl_sync(0xffffffffu, my_p, j);
      wt[j] = __shfl_sync(0xffffffffu, my_w, j);
      dot[j] = 0.f;
    }
    const uint4* grow = dout + static_cast<size_t>(t) * row_vec;
    for (int c = lane; c < row_vec; c += 32) {
      const uint4 g = grow[c];
      uint4 v[KMAX];
      if (dw) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < k && pos[j] >= 0) v[j] = y[static_cast<size_t>(pos[j]) * row_vec + c];
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j >= k || pos[j] < 0) continue;
        if (dy) dy[static_cast<size_t>(pos[j]) * row_vec + c] = scale_vec(g, wt[j], BF16);
        if (dw) dot[j] += dot_chunk(g, v[j], BF16);
      }
    }
    if (dw) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j >= k) break;
        float sdot = dot[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, off);
        if (lane == 0) dw[static_cast<size_t>(t) * k + j] = pos[j] >= 0 ? sdot : 0.f;
      }
    }
  }
}

template <bool BF16>
static void combine_backward_launch(const uint4* dout, const uint4* y, const int32_t* dst_pos,
                                    const float* w, int T, int row_vec, int N, int k, uint4* dy,
                                    float* dw, int blocks, cudaStream_t s) {
  if (k <= 1)
    launch_k(combine_backward_kernel<BF16, 1>, dim3(blocks), dim3(256), 0, s, dout, y, dst_pos, w, T, row_vec, N, k, dy, dw);
  else if (k <= 2)
    launch_k(combine_backward_kernel<BF16, 2>, dim3(blocks), dim3(256), 0, s, dout, y, dst_pos, w, T, row_vec, N, k, dy, dw);
  else if (k <= 4)
    launch_k(combine_backward_kernel<BF16, 4>, dim3(blocks), dim3(256), 0, s, dout, y, dst_pos, w, T, row_vec, N, k, dy, dw);
  else if (k <= 8)
    launch_k(combine_backward_kernel<BF16, 8>, dim3(blocks), dim3(256), 0, s, dout, y, dst_pos, w, T, row_vec, N, k, dy, dw);
  else
    launch_k(combine_backward_kernel<BF16, 16>, dim3(blocks), dim3(256), 0, s, dout, y, dst_pos, w, T, row_vec, N, k, dy, dw);
}

cudaError_t launch_combine_backward(const void* dout, const void* y, const int32_t* dst_pos,
                                    const float* topk_w, int T, int d, int N, int top_k,
                                    moe_dtype_t dt, void* dy, float* d_topk_w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int elt = dt == MOE_BF16 ? 2 : 4;
  const int row_vec = d * elt / 16;
  const int blocks = std::min(cdiv(T, 8), num_sms() * 8);
  if (dt == MOE_BF16)
    combine_backward_launch<true>(static_cast<const uint4*>(dout), static_cast<const uint4*>(y),
                                  dst_pos, topk_w, T, row_vec, N, top_k, static_cast<uint4*>(dy),
                                  d_topk_w, blocks, s);
  else
    combine_backward_launch<false>(static_cast<const uint4*>(dout), static_cast<const uint4*>(y),
                                   dst_pos, topk_w, T, row_vec, N, top_k, static_cast<uint4*>(dy),
                                   d_topk_w, blocks, s);
  return cudaGetLastError();
}

// One thread waits on a barrier that nothing arrives at; the bounded wait
// gives up after kWaitLimitNs and records MOE_DEV_TIMEOUT.
__global__ void selftest_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, nullptr, status);
  }
}

cudaError_t launch_selftest_timeout(int* status, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

__global__ void single_segment_kernel(int32_t* offsets, int n) {
  pdl_wait();
  pdl_trigger();
  offsets[0] = 0;
  offsets[1] = n;
}

cudaError_t launch_single_segment(int32_t* offsets, int n, cudaStream_t s) {
  launch_k(single_segment_kernel, dim3(1), dim3(1), 0, s, offsets, n);
  return cudaGetLastError();
}

// offsets[i] = floor(i n / S), i = 0..S: S near-equal segments of n rows.
__global__ void uniform_segments_kernel(int32_t* offsets, int S, int n) {
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= S; i += blockDim.x)
    offsets[i] = static_cast<int32_t>((static_cast<long long>(i) * n) / S);
}

cudaError_t launch_uniform_segments(int32_t* offsets, int S, int n, cudaStream_t s) {
  launch_k(uniform_segments_kernel, dim3(1), dim3(128), 0, s, offsets, S, n);
  return cudaGetLastError();
}

// out[i] = bf16(sum_{p < S} part[p][i]), fp32 sum in partial order (4 per thread).
__global__ void __launch_bounds__(256) sum_partials_bf16_kernel(const float4* __restrict__ part,
                                                                int S, size_t n4,
                                                                uint2* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float4 a = part[i];
    for (int p = 1; p < S; ++p) {
      const float4 b = part[static_cast<size_t>(p) * n4 + i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    out[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
}

cudaError_t launch_sum_partials_bf16(const float* part, int S, size_t n, void* out,
                                     cudaStream_t s) {
  const size_t n4 = n / 4;
  const int blocks = static_cast<int>(std::min<size_t>((n4 + 255) / 256, 8 * num_sms()));
  launch_k(sum_partials_bf16_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, s,
           reinterpret_cast<const float4*>(part), S, n4, static_cast<uint2*>(out));
  return cudaGetLastError();
}

// ------------------------------------------- folded combine: slot map, output
// The inverse of dst_pos: the token and routing weight of every slot.
__global__ void __launch_bounds__(256) slot_map_kernel(const int32_t* __restrict__ dst_pos,
                                                       const float* __restrict__ topk_w,
                                                       long long n, int top_k, int N,
                                                       int32_t* __restrict__ slot_tok,
                                                       float* __restrict__ slot_w) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int s = dst_pos[i];
    if (static_cast<unsigned>(s) >= static_cast<unsigned>(N)) continue;
    slot_tok[s] = static_cast<int32_t>(i / top_k);
    slot_w[s] = topk_w ? topk_w[i] : 1.0f;
  }
}

cudaError_t launch_slot_map(const int32_t* dst_pos, const float* topk_w, int T, int top_k, int N,
                            int32_t* slot_tok, float* slot_w, cudaStream_t s) {
  const long long n = 1LL * T * top_k;
  if (n == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 8LL * num_sms()));
  launch_k(slot_map_kernel, dim3(blocks), dim3(256), 0, s, dst_pos, topk_w, n, top_k, N,
           slot_tok, slot_w);
  return cudaGetLastError();
}

// out [n] bf16 = in [n] fp32 (RNE), eight values per thread and step.
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ in,
                                                          size_t n8, uint4* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = in[2 * i], b = in[2 * i + 1];
    out[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                        pack_bf16x2(b.z, b.w));
  }
}

cudaError_t launch_f32_to_bf16(const float* in, size_t n, void* out, cudaStream_t s) {
  const size_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<size_t>((n8 + 255) / 256, 8 * num_sms()));
  launch_k(f32_to_bf16_kernel, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const float4*>(in),
           n8, static_cast<uint4*>(out));
  return cudaGetLastError();
}

// ------------------------------------------------------- fp32 / SIMT router
template <typename TX>
__device__ __forceinline__ float to_f(TX v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// logits[t, e] = sum_i x[t, i] * w[e, i], sequential fp32 FMA over i.
template <typename TX>
__global__ void router_logits_kernel(const TX* __restrict__ x, const TX* __restrict__ w, int T,
                                     int d, int E, float* __restrict__ logits) {
  pdl_wait();
  pdl_trigger();
  const long long total = 1LL * T * E;
  for (long long i = blockIdx.x * 1LL * blockDim.x + threadIdx.x; i < total;
       i += 1LL * gridDim.x * blockDim.x) {
    const int t = static_cast<int>(i / E), e = static_cast<int>(i % E);
    const TX* xr = x + static_cast<size_t>(t) * d;
    const TX* wr = w + static_cast<size_t>(e) * d;
    float acc = 0.f;
    for (int q = 0; q < d; ++q) acc = fmaf(to_f<TX>(xr[q]), to_f<TX>(wr[q]), acc);
    logits[i] = acc;
  }
}

cudaError_t launch_router_logits_simt(const void* x, const void* w_router, int T, int d, int E,
                                      moe_dtype_t dt, float* logits, cudaStream_t s) {
  const long long total = 1LL * T * E;
  if (total == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 1LL * num_sms() * 32));
  if (dt == MOE_BF16)
    launch_k(router_logits_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, s, 
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w_router), T, d,
        E, logits);
  else
    launch_k(router_logits_kernel<float>, dim3(blocks), dim3(256), 0, s, static_cast<const float*>(x),
                                                       static_cast<const float*>(w_router), T, d,
                                                       E, logits);
  return cudaGetLastError();
}


// One warp per token; block b owns tokens [b*tpb, (b+1)*tpb).  Lane l holds
// experts l, l+32, ... (EPL of them); the logit is the sum of the nsplit
// partial values in split order.  The k winners come from k rounds of a warp
// arg-max on (key desc, expert asc) done with two redux.sync reductions
// (max of the order-preserving key, then min expert index among the lanes
// holding it); lane j keeps winner j.  NaN scores count as -inf.
//
// Selection keys ([HP] TokenChoiceTopKRouter.forward): the scores are
// s = softmax or sigmoid of the logits; the keys are c = s * route_scale,
// with the experts of groups outside the top `topk_groups` (by the group's
// maximum c) masked, plus expert_bias.  Without a bias and with a positive
// scale c is increasing in the logit, so the keys are the logits themselves
// (no rounding of s can merge or swap them).  Weights are the unbiased s of
// the winners, divided by their sum when renormalising, times route_scale;
// for softmax the division by the softmax denominator and the
// renormalisation are one division of the exponentials.
//
// With `blk` the block also writes its histogram of dispatch keys as column
// b of the dispatch table blk[bin * gridDim.x + b]; `counts` (int) and
// `tokens_per_expert` (float, accumulated with +=) get the expert histogram.
constexpr int kMaskedKey = INT_MIN + 1;   // below score_key(-inf), above "none"

template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(
    const float* __restrict__ parts, int nsplit, int T, int E, int k, int renorm, int tpb,
    RouterOptions opt, float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, int32_t* __restrict__ counts,
    float* __restrict__ tokens_per_expert, int32_t* __restrict__ blk, int nbins, int R, int L,
    int S, float* __restrict__ lb) {
  pdl_wait();
  pdl_trigger();
  // [nbins] dispatch keys (blk), then [E] experts, then [E] weight sums (lb)
  extern __shared__ int sm_bins[];
  __shared__ int gkey[8][32];        // per-warp group maxima (node-limited routing)
  int* dbins = sm_bins;
  int* ebins = sm_bins + (blk ? nbins : 0);
  float* wsum = reinterpret_cast<float*>(ebins + E);
  const bool tally_e = counts != nullptr || tokens_per_expert != nullptr || lb != nullptr;
  if (blk) {
    // the dispatch column scan's completion ticket sits after the table
    if (blockIdx.x == 0 && threadIdx.x == 0) blk[static_cast<size_t>(nbins) * gridDim.x] = 0;
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) dbins[i] = 0;
  }
  if (tally_e)
    for (int i = threadIdx.x; i < E; i += blockDim.x) ebins[i] = 0;
  if (lb)
    for (int i = threadIdx.x; i < E; i += blockDim.x) wsum[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const size_t plane = static_cast<size_t>(T) * E;
  const bool on_logits = opt.bias == nullptr && opt.scale > 0.f;
  const int gsize = opt.groups ? E / opt.groups : 1;
  const int t_end = min(T, (blockIdx.x + 1) * tpb);
  for (int t = blockIdx.x * tpb + warp; t < t_end; t += nwarps) {
    float sv[EPL];
    bool avail[EPL];
    const float* base = parts + static_cast<size_t>(t) * E + lane;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      avail[i] = lane + 32 * i < E;
      sv[i] = avail[i] ? base[32 * i] : 0.f;
    }
    // Splits in order; the loads of four splits are issued before their adds.
    int sp = 1;
    for (; sp + 4 <= nsplit; sp += 4) {
      float q[4][EPL];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          q[u][i] = avail[i] ? base[(sp + u) * plane + 32 * i] : 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < EPL; ++i) sv[i] += q[u][i];
    }
    for (; sp < nsplit; ++sp)
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (avail[i]) sv[i] += base[sp * plane + 32 * i];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if (avail[i] && logits_out) logits_out[static_cast<size_t>(t) * E + lane + 32 * i] = sv[i];
      if (sv[i] != sv[i]) sv[i] = -INFINITY;
      if (avail[i]) mx = fmaxf(mx, sv[i]);
    }
    // ex = exp(z - max z) (softmax numerators) or sigmoid(z); s = ex / den
    float ex[EPL];
    float den = 1.f;
    if (opt.sigmoid) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) ex[i] = avail[i] ? 1.0f / (1.0f + expf(-sv[i])) : 0.f;
    } else {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      den = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        ex[i] = avail[i] ? expf(sv[i] - mx) : 0.f;
        den += ex[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    }
    int key[EPL];
    float kv[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      kv[i] = on_logits ? sv[i] : ex[i] / den * opt.scale;
      key[i] = score_key(kv[i]);
    }
    if (opt.groups) {
      // group maxima of the keys in shared memory, then the kept groups by
      // redux rounds (largest maximum first, ties to the lower group)
      gkey[warp][lane] = INT_MIN;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (avail[i]) atomicMax(&gkey[warp][(lane + 32 * i) / gsize], key[i]);
      __syncwarp();
      const int gk = gkey[warp][lane];
      unsigned kept = 0u;
      bool gavail = lane < opt.groups;
      for (int j = 0; j < opt.topk_groups; ++j) {
        const int mk = __reduce_max_sync(0xffffffffu, gavail ? gk : INT_MIN);
        const int bg = __reduce_min_sync(0xffffffffu, (gavail && gk == mk) ? lane : 31);
        kept |= 1u << bg;
        if (lane == bg) gavail = false;
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (!((kept >> min((lane + 32 * i) / gsize, 31)) & 1u)) key[i] = kMaskedKey;
    }
    if (opt.bias) {
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (avail[i] && key[i] != kMaskedKey) {
          const float b = kv[i] + opt.bias[lane + 32 * i];
          key[i] = score_key(b != b ? -INFINITY : b);
        }
    }
    int my_e = 0;
    float my_x = 0.f;
    for (int j = 0; j < k; ++j) {
      int lk = INT_MIN, li = 0x7fffffff;
      float lx = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (avail[i] && key[i] > lk) {   // experts of a lane ascend with i: first max wins
          lk = key[i];
          li = lane + 32 * i;
          lx = ex[i];
        }
      const int mk = __reduce_max_sync(0xffffffffu, lk);
      const int be = __reduce_min_sync(0xffffffffu, lk == mk ? li : 0x7fffffff);
      const float bx = __shfl_sync(0xffffffffu, lx, be & 31);
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == be) avail[i] = false;
      if (lane == j) {
        my_e = be;
        my_x = bx;
      }
    }
    // weights: the unbiased score of each winner (renormalised), times the scale
    const float wx = lane < k ? my_x : 0.f;
    float sel = wx;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sel += __shfl_xor_sync(0xffffffffu, sel, off);
    if (lane < k) {
      const size_t o = static_cast<size_t>(t) * k + lane;
      topk_idx[o] = my_e;
      const float wout = wx / (renorm ? sel : den) * opt.scale;
      topk_w[o] = wout;
      if (opt.scores_out) opt.scores_out[o] = wx / den;
      if (blk) atomicAdd(&dbins[dispatch_key(my_e, t, R, L, S)], 1);
      if (tally_e) atomicAdd(&ebins[my_e], 1);
      if (lb) atomicAdd(&wsum[my_e], wout);
    }
  }
  __syncthreads();
  if (blk)
    for (int i = threadIdx.x; i < nbins; i += blockDim.x)
      blk[static_cast<size_t>(i) * gridDim.x + blockIdx.x] = dbins[i];
  if (tally_e) {
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
      const int c = ebins[i];
      if (!c) continue;
      if (counts) atomicAdd(&counts[i], c);
      if (tokens_per_expert) atomicAdd(&tokens_per_expert[i], static_cast<float>(c));
      if (lb) {
        atomicAdd(&lb[i], static_cast<float>(c));
        atomicAdd(&lb[E + i], wsum[i]);
      }
    }
  }
}

// [HP] _compute_load_balance_loss from the per-expert copy counts and
// weight sums: E * sum_e (count_e / (T k)) * (wsum_e / T).
__global__ void lb_loss_kernel(const float* __restrict__ lb, int E, int T, int k,
                               float* __restrict__ loss) {
  pdl_wait();
  pdl_trigger();
  __shared__ float part[32];
  float acc = 0.f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) acc += lb[e] * lb[E + e];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += part[w];
    *loss = T > 0 ? static_cast<float>(E) * tot / (static_cast<float>(T) * k * T) : 0.f;
  }
}

cudaError_t launch_lb_loss(const float* lb, int E, int T, int top_k, float* loss, cudaStream_t s) {
  launch_k(lb_loss_kernel, dim3(1), dim3(256), 0, s, lb, E, T, top_k, loss);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const float* parts, int nsplit, int T, int E, int top_k,
                               int renorm, const RouterOptions& o, float* logits_out,
                               int32_t* topk_idx, float* topk_w, int32_t* counts,
                               float* tokens_per_expert, const DispatchPlan* plan,
                               int32_t* blk, cudaStream_t s, float* lb) {
  if (T == 0) return cudaSuccess;
  const bool fuse = plan && blk;
  const int tpb = fuse ? plan->tb : 16;
  const int blocks = cdiv(T, tpb);
  const int nbins = fuse ? plan->nbins : 0;
  const bool tally_e = counts || tokens_per_expert || lb;
  const size_t smem =
      sizeof(int) * ((fuse ? nbins : 0) + (tally_e ? E : 0)) + (lb ? sizeof(float) * E : 0);
  const int R = fuse ? plan->R : 1, L = fuse ? plan->L : E, S = fuse ? plan->S : T;
  int32_t* b = fuse ? blk : nullptr;
  const RouterOptions opt = o;
  if (E <= 32)
    launch_k(router_topk_kernel<1>, dim3(blocks), dim3(256), smem, s, parts, nsplit, T, E, top_k,
             renorm, tpb, opt, logits_out, topk_idx, topk_w, counts, tokens_per_expert, b,
             nbins, R, L, S, lb);
  else if (E <= 64)
    launch_k(router_topk_kernel<2>, dim3(blocks), dim3(256), smem, s, parts, nsplit, T, E, top_k,
             renorm, tpb, opt, logits_out, topk_idx, topk_w, counts, tokens_per_expert, b,
             nbins, R, L, S, lb);
  else if (E <= 128)
    launch_k(router_topk_kernel<4>, dim3(blocks), dim3(256), smem, s, parts, nsplit, T, E, top_k,
             renorm, tpb, opt, logits_out, topk_idx, topk_w, counts, tokens_per_expert, b,
             nbins, R, L, S, lb);
  else if (E <= 256)
    launch_k(router_topk_kernel<8>, dim3(blocks), dim3(256), smem, s, parts, nsplit, T, E, top_k,
             renorm, tpb, opt, logits_out, topk_idx, topk_w, counts, tokens_per_expert, b,
             nbins, R, L, S, lb);
  else
    launch_k(router_topk_kernel<16>, dim3(blocks), dim3(256), smem, s, parts, nsplit, T, E,
             top_k, renorm, tpb, opt, logits_out, topk_idx, topk_w, counts, tokens_per_expert,
             b, nbins, R, L, S, lb);
  return cudaGetLastError();
}

}  // namespace moe
