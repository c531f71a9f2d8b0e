// moe_dispatch_noalloc: moe_dispatch for callers that cannot allocate device
// memory.  Some callers cannot call cudaMalloc (or ask another allocator) at
// the point where they dispatch: code that runs inside an engine or plugin
// whose enqueue path must not allocate, servers whose device memory is
// entirely pre-reserved by another framework's pool, and hot paths that must
// never block on the allocator.  This variant keeps its scratch (the status
// word and the per-block histogram table) in a fixed array in this file
// instead of a caller workspace.  The caller still passes every input and
// output buffer.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr size_t kNoAllocStatusBytes = 256;

// Scratch of the no-allocation dispatch: status word, then the histogram
// table.  Every GPU that loads the library holds it until the process exits.
__device__ __align__(256) unsigned char g_dispatch_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;
void* g_scratch_addr[64] = {nullptr};

// Device address of g_dispatch_scratch on the current device.  In host code
// the symbol itself is only a host-side handle, so the address is looked up
// with that device current.  Outside stream capture it is looked up on every
// call (a device reset or a re-created primary context moves the array);
// while `s` is being captured no lookup is made and the address of the last
// lookup on this device is used (the first call on a device must therefore
// come before any capture).
cudaError_t scratch_address(cudaStream_t s, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (cap == cudaStreamCaptureStatusNone || !g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_dispatch_noalloc(const void* x, const int32_t* topk_idx, int T, int d,
                                             int E, int top_k, moe_dtype_t dt, int32_t* counts,
                                             int32_t* offsets, int32_t* src_row,
                                             int32_t* dst_pos, void* x_perm, void* stream) {
  // the same argument rules, status codes and texts as moe_dispatch
  if (moe_status_t st = check_dispatch_args(x, topk_idx, T, d, E, top_k, 1, dt, counts, offsets,
                                            src_row, dst_pos, x_perm))
    return st;
  const DispatchPlan p = make_dispatch_plan(T, E, top_k, 1);
  const size_t need = kNoAllocStatusBytes + dispatch_ws_bytes(p);
  if (need > MOE_NOALLOC_SCRATCH_BYTES) {
    set_last_error("moe_dispatch_noalloc: T=%d, E=%d need %zu bytes of scratch, more than the "
                   "%d-byte fixed array (use moe_dispatch with a workspace)",
                   T, E, need, MOE_NOALLOC_SCRATCH_BYTES);
    return MOE_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* base = nullptr;
  cudaError_t e = scratch_address(s, &base);
  if (e != cudaSuccess) {
    set_last_error("moe_dispatch_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  int* status = static_cast<int*>(base);
  // the array keeps the last call's bytes: the histogram kernel rewrites the
  // whole table and the column scan the whole status word
  e = launch_dispatch(p, x, topk_idx, d, dt, counts, offsets, src_row, dst_pos,
                      x ? x_perm : nullptr, static_cast<char*>(base) + kNoAllocStatusBytes,
                      status, s, false, nullptr, /*own_status=*/true);
  if (e != cudaSuccess) {
    set_last_error("moe_dispatch_noalloc: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
