// gather_combine.cu -- the two memory-bound steps around the expert GEMMs.
//
//  gather   X_perm[p] = x[perm[p] / k] for every routed slot position p, so each
//           expert's tokens form one contiguous run of rows for the grouped
//           GEMM's TMA loads (the shared expert reads x directly).  One warp
//           copies one row with 16-byte loads and stores.
//  combine  the merge of the chosen experts' results into the layer output
//           (m.xxqk.cn Hy4-preview MoE explainer, section 2.2; the shared
//           expert of the ZAKER release news is added with weight 1):
//             y[t] = sum_s Y[T*k + s*T + t] + sum_i w[t][i] * Y[pos[t*k + i]]
//           in fp32, in that fixed order, then rounded once to bf16.  Each
//           thread owns 8 consecutive features of one token.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kGatherThreads)
    gather_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                       const int32_t* __restrict__ offsets, int T, int k, int E, int d,
                       uint16_t* __restrict__ x_perm) {
  const int nslots = T * k;
  const int nrows = min(nslots, max(0, offsets[E]));
  const int warps_total = gridDim.x * (kGatherThreads / 32);
  const int lane = threadIdx.x & 31;
  const int vec = d / 8;  // 16-byte vectors per row
  for (int p = blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); p < nrows;
       p += warps_total) {
    const int s = perm[p];
    if (s < 0 || s >= nslots) continue;
    const uint4* __restrict__ src = reinterpret_cast<const uint4*>(x + size_t(s / k) * d);
    uint4* __restrict__ dst = reinterpret_cast<uint4*>(x_perm + size_t(p) * d);
    int i = lane;
    for (; i + 96 < vec; i += 128) {
      const uint4 a = src[i], b = src[i + 32], c = src[i + 64], e = src[i + 96];
      dst[i] = a;
      dst[i + 32] = b;
      dst[i + 64] = c;
      dst[i + 96] = e;
    }
    for (; i < vec; i += 32) dst[i] = src[i];
  }
}

__device__ __forceinline__ void fma8(float (&acc)[8], float w, const float* __restrict__ row) {
  const float4 a = *reinterpret_cast<const float4*>(row);
  const float4 b = *reinterpret_cast<const float4*>(row + 4);
  acc[0] = fmaf(w, a.x, acc[0]);
  acc[1] = fmaf(w, a.y, acc[1]);
  acc[2] = fmaf(w, a.z, acc[2]);
  acc[3] = fmaf(w, a.w, acc[3]);
  acc[4] = fmaf(w, b.x, acc[4]);
  acc[5] = fmaf(w, b.y, acc[5]);
  acc[6] = fmaf(w, b.z, acc[6]);
  acc[7] = fmaf(w, b.w, acc[7]);
}

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const float* __restrict__ Y, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ pos, int T, int k, int S, int d,
                   uint16_t* __restrict__ y) {
  const int t = blockIdx.x;
  const int c = (blockIdx.y * kCombineThreads + threadIdx.x) * 8;
  if (c >= d) return;
  const size_t nslots = size_t(T) * k;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < S; ++s) {
    const float* row = Y + (nslots + size_t(s) * T + t) * d + c;
    const float4 a = *reinterpret_cast<const float4*>(row);
    const float4 b = *reinterpret_cast<const float4*>(row + 4);
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
  for (int i = 0; i < k; ++i) {
    const int p = pos[size_t(t) * k + i];
    if (p < 0 || size_t(p) >= nslots) continue;
    fma8(acc, topk_w[size_t(t) * k + i], Y + size_t(p) * d + c);
  }
  uint4 out;
  out.x = pack_bf16x2(acc[0], acc[1]);
  out.y = pack_bf16x2(acc[2], acc[3]);
  out.z = pack_bf16x2(acc[4], acc[5]);
  out.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(y + size_t(t) * d + c) = out;
}

}  // namespace

cudaError_t launch_gather(const Ctx& c, const uint16_t* x, const int32_t* perm,
                          const int32_t* offsets, int T, uint16_t* x_perm, int num_sms,
                          cudaStream_t st) {
  const int rows = T * c.k;
  const int warps_per_block = kGatherThreads / 32;
  int blocks = (rows + warps_per_block - 1) / warps_per_block;
  blocks = blocks < num_sms * 8 ? blocks : num_sms * 8;
  if (blocks < 1) blocks = 1;
  gather_rows_kernel<<<blocks, kGatherThreads, 0, st>>>(x, perm, offsets, T, c.k, c.E, c.d,
                                                        x_perm);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Ctx& c, const float* Y, const float* topk_w, const int32_t* pos,
                           int T, uint16_t* y, cudaStream_t st) {
  dim3 grid(T, (c.d / 8 + kCombineThreads - 1) / kCombineThreads);
  combine_kernel<<<grid, kCombineThreads, 0, st>>>(Y, topk_w, pos, T, c.k, c.S, c.d, y);
  return cudaGetLastError();
}

}  // namespace moe
