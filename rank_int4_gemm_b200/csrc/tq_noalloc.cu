// tq_noalloc.cu -- tq_w4a4_lr_gemm for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc at all: code running inside a host
// framework whose device allocator is owned by someone else, real-time paths
// that may not allocate (an allocation can synchronise the device), and
// plugins that only ever receive pointers to their inputs and outputs.  Such
// a caller has no way to provide the GEMM's workspace (the status word its
// bounded in-kernel waits write).  This entry point instead uses a fixed
// scratch array in the library's own device memory, so the caller passes only
// inputs, outputs and a stream.
//
// Costs of that convenience: the array exists on every GPU that loads the
// library until the process exits, and it is shared by every call, so calls
// that overlap on the GPU (on different streams without ordering between
// them) race on it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace {

constexpr size_t kScratchBytes = 256;  // largest workspace this entry serves

// The scratch.  In host code this name is only a host-side stand-in for the
// device symbol: a kernel must be given the address cudaGetSymbolAddress
// returns for the current device, never &g_noalloc_scratch.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return TQ_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return TQ_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" int tq_w4a4_lr_gemm_noalloc(const uint8_t* Xq, const float* s_x, const uint8_t* Wq,
                                       const float* s_w, const float* XL1, const uint16_t* L2t,
                                       int M, int N, int K, int r, uint16_t* Y, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return TQ_ERR_INVALID_VALUE;
  // the shape must fit the fixed scratch; checked before anything else runs
  if (tq_gemm_workspace_bytes(M, N, K, r) > kScratchBytes) return TQ_ERR_WORKSPACE;
  void* ws = nullptr;
  if (int st = scratch_for_current_device(&ws)) return st;
  // the status word must start at zero for this call
  if (cudaMemsetAsync(ws, 0, kScratchBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TQ_ERR_CUDA;
  return tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t, M, N, K, r, Y, ws, kScratchBytes, stream);
}
