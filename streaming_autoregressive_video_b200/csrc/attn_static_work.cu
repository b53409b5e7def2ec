// fd_block_attention_static: the attention call with its per-call work area
// (the block's keys and queries rotated once per call, which the tensor-core
// kernels read) in a static device array of this library instead of the
// call's work set in the caller's cache storage.  For callers that cannot set device memory aside for that
// area -- their storage comes from a pool or arena sized by someone else, or
// they may not call cudaMalloc at all (it can synchronise the device, which a
// real-time serving loop cannot afford).  The method on the pages has no
// counterpart; this is an interface choice.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fd.h"
#include "fd_internal.h"

namespace {

// The work area.  Every GPU that loads this library holds it until the
// process exits.  In host code the name is only a host-side stand-in, never a
// device address: the address comes from cudaGetSymbolAddress below.
__device__ __align__(256) uint8_t g_block_work[FD_STATIC_WORK_BYTES];

std::mutex g_mutex;
void* g_work_addr[fd::kMaxDevices] = {};

// Device address of g_block_work on the current device: looked up once per
// device, with that device current, on the first call made on it.
fd_status work_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FD_ERR_CUDA;
  if (dev < 0 || dev >= fd::kMaxDevices) return FD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_work_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_block_work) != cudaSuccess || p == nullptr)
      return FD_ERR_CUDA;
    g_work_addr[dev] = p;
  }
  *out = g_work_addr[dev];
  return FD_OK;
}

}  // namespace

extern "C" fd_status fd_block_attention_static(fd_cache* cache, int32_t layer,
                                               int32_t n_rollouts,
                                               const void* q, const void* k,
                                               const void* v, void* out,
                                               float* lse, void* stream) {
  fd::NvtxRange nvtx_range("fd_block_attention_static");
  if (cache == nullptr || n_rollouts < 1) return FD_ERR_INVALID_ARG;
  if (fd::block_work_bytes(cache, n_rollouts) > (size_t)FD_STATIC_WORK_BYTES)
    return FD_ERR_CAPACITY;
  void* work = nullptr;
  const fd_status st = work_address(&work);
  if (st != FD_OK) return st;
  // The rotation pass overwrites every row of the area the attention kernel
  // reads, so nothing left by an earlier call is ever read.
  return fd::block_attention_impl(cache, layer, n_rollouts, q, k, v, out, lse,
                                  stream, work);
}
