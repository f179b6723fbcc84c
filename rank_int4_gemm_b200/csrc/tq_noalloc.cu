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
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace {

constexpr size_t kScratchBytes = 256;  // largest workspace this entry serves

// The scratch.  In host code this name is only a host-side stand-in for the
// device symbol: a kernel must be given the address cudaGetSymbolAddress
// returns for the current device, never &g_noalloc_scratch.  Its first word
// is the status word of the kernel's bounded waits (zero at module load;
// written only when a wait gives up; cleared by tq_noalloc_query_status).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch per CUDA context.  A context (not a device
// index) is the key because the module, and with it the array, is loaded
// again into a new primary context after cudaDeviceReset.
constexpr int kMaxContexts = 64;
std::mutex g_mu;
CUcontext g_ctx[kMaxContexts] = {};
void* g_addr[kMaxContexts] = {};
int g_count = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent from the driver, fetched through the runtime (the library
// links the static runtime, not libcuda).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch in the current context, looked up with that
// context current on its first use there and cached.
int scratch_for_current_context(void** out) {
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return TQ_ERR_NO_DEVICE;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return TQ_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (ctx)
    for (int i = 0; i < g_count; ++i)
      if (g_ctx[i] == ctx) {
        *out = g_addr[i];
        return TQ_OK;
      }
  // first use in this context (the lookup also makes the runtime's primary
  // context current if this thread had none yet)
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return TQ_ERR_CUDA;
  }
  if (get(&ctx) != CUDA_SUCCESS || !ctx) return TQ_ERR_NO_DEVICE;
  // a context created after the table is full keeps working, uncached
  if (g_count < kMaxContexts) {
    g_ctx[g_count] = ctx;
    g_addr[g_count] = p;
    ++g_count;
  }
  *out = p;
  return TQ_OK;
}

}  // namespace

extern "C" int tq_w4a4_lr_gemm_noalloc(const uint8_t* Xq, const float* s_x, const uint8_t* Wq,
                                       const float* s_w, const float* XL1, const uint16_t* L2t,
                                       int M, int N, int K, int r, uint16_t* Y, void* stream) {
  // the same argument checks as tq_w4a4_lr_gemm, before any device work
  if (!Y) return TQ_ERR_INVALID_VALUE;
  if (int st = tq::gemm_operand_status(Xq, s_x, Wq, s_w, XL1, L2t, M, N, K, r, Y, nullptr))
    return st;
  // the shape must fit the fixed scratch
  if (tq_gemm_workspace_bytes(M, N, K, r) > kScratchBytes) return TQ_ERR_WORKSPACE;
  if (int st = tq::device_status()) return st;
  void* ws = nullptr;
  if (int st = scratch_for_current_context(&ws)) return st;
  // nothing in the scratch has to start at zero for the result: the kernel
  // only ever writes the status word, and only when a bounded wait gives up
  return tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t, M, N, K, r, Y, ws, kScratchBytes, stream);
}

extern "C" int tq_noalloc_query_status(void* stream) {
  if (int st = tq::device_status()) return st;
  void* ws = nullptr;
  if (int st = scratch_for_current_context(&ws)) return st;
  return tq_query_device_status(ws, stream);
}

extern "C" int tq_debug_noalloc_set_status(int status) {
  if (int st = tq::device_status()) return st;
  void* ws = nullptr;
  if (int st = scratch_for_current_context(&ws)) return st;
  const uint32_t word = static_cast<uint32_t>(status);
  if (cudaMemcpy(ws, &word, sizeof(word), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return TQ_ERR_CUDA;
  }
  return TQ_OK;
}
