// selftest.cu -- exercises the bounded-wait machinery the pipelined kernels rely on.
//
// Every mbarrier wait in this library gives up after a time limit, records the
// fault in the workspace status word and lets the kernel return, so that a
// broken pipeline can never hang the GPU.  moe_selftest_wait_timeout runs one
// CTA whose thread 0 waits, through the same mbar_wait the GEMM kernels use, on
// an mbarrier that nothing will ever complete; the wait expires after
// timeout_ns, the kernel writes the timeout code to the status word and exits.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kSiteSelftest = 6;

__global__ void bounded_wait_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t never;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);   // one arrival expected; none will come
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&never, 0, timeout_ns))
    report_error(status, kDevTimeout, kSiteSelftest);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_selftest_wait_timeout(void* workspace, size_t ws_bytes,
                                                 unsigned long long timeout_ns, void* stream) {
  if (!workspace || ws_bytes < 1024 + sizeof(int)) return MOE_ERR_INVALID_ARG;
  if (timeout_ns == 0 || timeout_ns > 2000000000ull) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  moe_status s = ensure_device(&dev);
  if (s) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = reinterpret_cast<int*>((reinterpret_cast<uintptr_t>(workspace) + kWsAlign - 1) &
                                       ~uintptr_t(kWsAlign - 1));
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  bounded_wait_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
