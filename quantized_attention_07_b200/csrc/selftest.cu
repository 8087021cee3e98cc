// Self-test of the bounded-wait path: one CTA waits on an mbarrier that
// nothing ever arrives on, gives up after a caller-chosen number of cycles and
// records a timeout in the status word -- exactly what the attention kernel's
// waits do when a pipeline partner never signals.  No fault, no trap.
#include "common.cuh"
#include "ptx.cuh"

namespace sage {
namespace {

__global__ void wait_timeout_kernel(long long limit_cycles, uint32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = ptx::mbar_try_wait(&bar, 0);
    const long long t0 = clock64();
    while (!ok && clock64() - t0 <= limit_cycles) ok = ptx::mbar_try_wait(&bar, 0);
    if (!ok) set_status(status, ST_TIMEOUT);
  }
}

}  // namespace

cudaError_t launch_wait_timeout(long long limit_cycles, uint32_t* status, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(limit_cycles, status);
  return cudaGetLastError();
}

}  // namespace sage

extern "C" sage_status_t sage_selftest_wait_timeout(long long wait_cycles, void* ws,
                                                    size_t ws_bytes, void* stream) {
  if (wait_cycles < 1 || wait_cycles > (1LL << 31) || !ws ||
      (reinterpret_cast<uintptr_t>(ws) & 15) != 0)
    return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < 256) return SAGE_ERR_WORKSPACE;
  cudaError_t e = sage::launch_wait_timeout(wait_cycles, static_cast<uint32_t*>(ws),
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
