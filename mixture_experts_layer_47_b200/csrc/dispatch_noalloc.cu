// dispatch_noalloc.cu -- moe_dispatch for callers that cannot allocate device memory.
//
// moe_dispatch needs a little scratch memory (per-block expert histograms, the
// grouped GEMM's tile schedule, a status word) that normally lives in the
// caller's workspace.  Some callers cannot hand out device memory at all: a
// plug-in running inside a host application that owns every device
// allocation through its own pool and forbids its plug-ins from calling
// cudaMalloc, or a latency-critical loop in which cudaMalloc (which may
// synchronise the device) is not allowed.  moe_dispatch_noalloc serves them
// with the same kernels, using a fixed scratch array compiled into this
// library instead of a workspace.
//
// The scratch is a file-scope __device__ array: every CUDA context in which
// the library's kernels are loaded holds its own copy (about 74 KB) until the
// context or the process ends.  Host code cannot use the array's name as a
// device pointer; every call asks for the array's address in the calling
// thread's current context with cudaGetSymbolAddress (a lookup, not an
// allocation).  The address is not cached: a cached one would belong to a
// context that cudaDeviceReset has destroyed, or to the primary context when
// a host application runs this code under a context of its own.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Largest dispatch this entry point supports: T * k <= 65536 slots (the Hy4
// prefill shape, T = 8192 and k = 8) and E <= 1024 experts (the library's limit).
constexpr int kNoAllocMaxSlots = 65536;
constexpr int kNoAllocMaxBlocks = kNoAllocMaxSlots / kDispatchChunk;  // 16
constexpr int kNoAllocMaxExperts = 1024;
constexpr int kStatusInts = 64;  // status word, padded to 256 bytes
constexpr int kHistInts = kNoAllocMaxBlocks * kNoAllocMaxExperts;
constexpr int kSchedInts = 2 * (kNoAllocMaxExperts + 8 + 1) + 62;  // two schedules, padded
constexpr int kScratchInts = kStatusInts + kHistInts + kSchedInts;

static __device__ __align__(256) int32_t g_dispatch_scratch[kScratchInts];

// Device address of g_dispatch_scratch in the current context.
moe_status scratch_address(int32_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
  if (e != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *out = static_cast<int32_t*>(p);
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(moe_handle h, const int32_t* topk_idx, int T,
                                           int32_t* counts, int32_t* offsets, int32_t* perm,
                                           int32_t* pos, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  Ctx c;
  if (moe_internal_shape(h, &c) != MOE_OK) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!topk_idx || !counts || !offsets || !perm || !pos) return MOE_ERR_INVALID_ARG;
  if ((long long)T * c.k > kNoAllocMaxSlots || c.E > kNoAllocMaxExperts || c.S > 8)
    return MOE_ERR_WORKSPACE;  // larger than the fixed scratch allows
  DeviceInfo* dev;
  moe_status s = ensure_device(&dev);
  if (s) return s;
  int32_t* scratch = nullptr;
  if ((s = scratch_address(&scratch))) return s;
  int* status = reinterpret_cast<int*>(scratch);
  int32_t* blk_hist = scratch + kStatusInts;
  int32_t* sched = blk_hist + kHistInts;
  const int nblk = int((T * c.k + kDispatchChunk - 1) / kDispatchChunk);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The histograms and the schedule are fully rewritten by every call; only the
  // status word must start at zero.
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (launch_dispatch(c, topk_idx, T, nblk > 0 ? nblk : 1, blk_hist, counts, offsets, perm, pos,
                      sched, status, st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
