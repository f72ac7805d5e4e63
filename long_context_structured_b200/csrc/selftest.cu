// selftest.cu -- exercises the library's failure path without faulting the GPU.
//
// Every wait of the library's kernels on an mbarrier is bounded: when the
// limit passes, the waiting thread records SATTN_ERR_TIMEOUT and the waiting
// site in the workspace's status word, raises the CTA's abort flag, and
// returns, so the kernel ends normally and the CUDA context stays usable.
// This kernel waits, through the same bounded wait, on a barrier that
// nothing arrives at, with a caller-chosen short limit.
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kSelftestSite = 99;

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_i;
  if (threadIdx.x == 0) {
    abort_i = 0;
    mbar_init(&bar, 1);  // one arrival expected; none is made
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &abort_i;
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, abort_flag, status, kSelftestSite, limit_ns);
  __syncthreads();
}

}  // namespace

}  // namespace sattn

extern "C" int sattn_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
  if (!ws || ws_bytes < sattn::kStatusBytes || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (limit_ns == 0 || limit_ns > sattn::kWaitLimitNs) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sattn::kStatusBytes, st) != cudaSuccess) return SATTN_ERR_CUDA;
  sattn::wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<int32_t*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA;
}
