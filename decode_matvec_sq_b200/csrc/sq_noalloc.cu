// sq_noalloc.cu -- sq_linear_noalloc: sq_linear with its scratch in a fixed
// device array of this library instead of a caller-provided workspace.
//
// Which callers cannot allocate, and why:
//   * a serving process that has handed all free HBM to its KV-cache pool at
//     start-up, so a later cudaMalloc fails or evicts cache blocks;
//   * a caller on a latency-critical path: cudaMalloc and cudaFree can
//     synchronize the device, which stalls every stream of the process;
//   * a plain C host program linking only this library, with no allocator
//     of its own to hand out a workspace.
// For them the scratch is one file-scope __device__ array, resolved to a
// device pointer once per device; nothing is allocated here, ever.
//
// What must start at zero: the per-row arrival counters at the end of the
// scratch (the last roundup(4*N, 256) bytes of the workspace layout that
// sq_linear_workspace_bytes describes).  The first call on each device
// zero-fills the whole array on its own stream before its launch; every call
// leaves the counters zero again; the partial-sum area is overwritten before
// it is read.
//
// Calls share the one array per device: two calls whose kernels overlap in
// time (different streams, or different host threads, without ordering)
// race on it and give wrong results.  Order them on one stream or by events.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/sq.h"

namespace {

constexpr size_t kScratchBytes = SQ_LINEAR_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];  // device address of g_scratch, per device

// The scratch of the current device: on the first call for this device its
// address is looked up and the array is zero-filled on `stream`.
sq_status scratch_of_current_device(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SQ_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, kScratchBytes, stream) != cudaSuccess) return SQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SQ_OK;
}

}  // namespace

extern "C" sq_status sq_linear_noalloc(const sq_packed_weight* w, const int8_t* xq,
                                       const float* sx, const float* x_out, const int32_t* idx,
                                       int32_t n_out, int32_t M, float* y, int32_t* dev_status,
                                       uint32_t flags, void* stream) {
  // sq_linear_workspace_bytes returns 0 for an invalid weight or no usable
  // device; sq_linear then reports the precise error before any device work
  const size_t need = sq_linear_workspace_bytes(w, M);
  if (need == 0)
    return sq_linear(w, xq, sx, x_out, idx, n_out, M, y, nullptr, 0, dev_status, flags, stream);
  if (need > kScratchBytes) return SQ_ERR_WORKSPACE;
  // the scratch is the current device's; a stream of another device would
  // make the kernel use (and race on) the wrong array
  if (stream) {
    int sdev = -1, cur = -1;
    if (cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) != cudaSuccess ||
        cudaGetDevice(&cur) != cudaSuccess)
      return SQ_ERR_CUDA;
    if (sdev != cur) return SQ_ERR_INVALID_ARG;
  }
  void* ws = nullptr;
  const sq_status st = scratch_of_current_device(static_cast<cudaStream_t>(stream), &ws);
  if (st != SQ_OK) return st;
  return sq_linear(w, xq, sx, x_out, idx, n_out, M, y, ws, kScratchBytes, dev_status, flags,
                   stream);
}
