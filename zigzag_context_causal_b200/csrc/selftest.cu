// Self test of the bounded mbarrier wait that every pipeline stage of the
// attention kernel uses (diagnostic entry point zz_debug_wait_timeout).
#include <cuda_runtime.h>

#include <string>

#include "ptx_sm100.cuh"
#include "nvtx_range.h"
#include "zz_internal.h"

using namespace zz::dev;
namespace zz {
namespace {
// One thread waits, with the attention kernel's own bounded wait, on an
// mbarrier that nothing ever arrives at, then reports what happened:
// status[0] = 1 when the wait gave up (expected), status[1] = elapsed ns.
__global__ void wait_timeout_probe(uint64_t timeout_ns, int64_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  abort_flag = 0;
  const uint64_t t0 = global_timer_ns();
  const bool ok = wait_parity(&bar, 0, &abort_flag, timeout_ns);
  status[0] = ok ? 0 : (abort_flag ? 1 : 2);
  status[1] = int64_t(global_timer_ns() - t0);
}
}  // namespace
}  // namespace zz

extern "C" zz_status_t zz_debug_wait_timeout(int64_t timeout_ns, int64_t* dev_status, void* stream) {
  ZZ_NVTX("zz_debug_wait_timeout");
  using namespace zz;
  if (!dev_status || timeout_ns <= 0 || timeout_ns > 10000000000ll)
    return fail(ZZ_ERR_INVALID_ARG, "zz_debug_wait_timeout: need dev_status and 0 < timeout_ns <= 10 s");
  wait_timeout_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(timeout_ns), dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("wait_timeout_probe: ") + cudaGetErrorString(e));
  return ZZ_OK;
}
