// tq_watchdog.cu -- a test of the bounded waits every pipelined kernel of the
// library uses (mbar_wait in tq_ptx.cuh).
//
// One CTA, no cluster, two warps: a producer lane arrives on an mbarrier
// (unless the host asks it to withhold that arrival) and a consumer lane
// waits for it with mbar_wait and a short budget.  When the arrival is
// withheld the wait runs out, writes the timeout code into the caller's
// status word and the kernel returns normally: the context stays usable, and
// tq_query_device_status reports TQ_ERR_TIMEOUT.  No fault, trap or endless
// loop is involved; the wait ends after `budget` SM cycles at the latest.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/tq.h"
#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {
namespace {

__global__ void __launch_bounds__(64, 1)
    watchdog_kernel(uint32_t* status, int withhold, long long budget, int* waited_ok) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 32 && !withhold) mbar_arrive(&bar);  // the producer
  if (threadIdx.x == 0) {                                 // the consumer
    const bool ok = mbar_wait(&bar, 0u, status, &abort_flag, budget);
    *waited_ok = ok ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_watchdog_test(uint32_t* status, int withhold, long long budget,
                                 int* waited_ok, cudaStream_t stream) {
  watchdog_kernel<<<1, 64, 0, stream>>>(status, withhold, budget, waited_ok);
  return cudaGetLastError();
}

}  // namespace tq

extern "C" int tq_debug_watchdog(void* workspace, size_t workspace_bytes, int withhold,
                                 long long budget_cycles, int* waited_ok, void* stream) {
  if (!workspace || !waited_ok) return TQ_ERR_INVALID_VALUE;
  if (workspace_bytes < 256) return TQ_ERR_WORKSPACE;
  // a short wait: at most ~1 s of SM clock, and long enough to be a wait
  if (budget_cycles < 1000 || budget_cycles > 2000000000ll) return TQ_ERR_INVALID_VALUE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(waited_ok) & 3u) != 0)
    return TQ_ERR_MISALIGNED;
  if (int s = tq::device_status()) return s;
  const cudaError_t e = tq::launch_watchdog_test(static_cast<uint32_t*>(workspace), withhold,
                                                 budget_cycles, waited_ok,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
