// route.cu -- the router of the MoE layer on sm_100a CUDA cores.
//
// m.xxqk.cn Hy4-preview MoE explainer, section 2.2 "router mechanism": every
// token is scored against every expert and the K best-scoring experts are
// activated.  Readings applied (identical in the CPU oracle): the score is a
// linear projection of the token (plus an optional per-expert bias), the gate
// is a softmax renormalised over the selected k, ties go to the lower expert.
//
// Two kernels:
//  router_partial  logits over a K-chunk, fp32 FFMA (no TF32: the index parity
//                  needs logits accurate to well below 1e-5), x widened from
//                  bf16 exactly.  A CTA computes a BT x 64 tile of
//                  (tokens x experts) for one K-chunk; the chunk count is
//                  chosen so the grid fills the GPU even for 16 tokens.
//  router_topk     one warp per token adds the chunk partials in a fixed
//                  order, then k rounds of a warp arg-max (value desc, expert
//                  asc) select the experts; the gate of choice i is
//                  exp(l_i - l_0) / sum_j exp(l_j - l_0).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kBE = 64;   // experts per CTA tile
constexpr int kBK = 32;   // K per shared-memory stage

template <int BT>
__global__ void __launch_bounds__(kRouterThreads)
    router_partial_kernel(const uint16_t* __restrict__ x, const float* __restrict__ Wr, int T,
                          int d, int E, int kchunk, float* __restrict__ part) {
  constexpr int TT = BT / 16;  // tokens per thread
  constexpr int TE = 4;        // experts per thread
  __shared__ __align__(16) float xs[kBK][BT + 4];
  __shared__ __align__(16) float ws[kBK][kBE + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.x * BT, e0 = blockIdx.y * kBE, ks = blockIdx.z;
  const int kbeg = ks * kchunk;

  float acc[TT][TE];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

  for (int k0 = kbeg; k0 < kbeg + kchunk; k0 += kBK) {
    // x tile: BT tokens x 32 bf16, 16-byte loads, widened to fp32, stored K-major.
    for (int i = tid; i < BT * (kBK / 8); i += kRouterThreads) {
      const int r = i / (kBK / 8), c8 = (i % (kBK / 8)) * 8;
      const int t = t0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < T) v = *reinterpret_cast<const uint4*>(x + size_t(t) * d + k0 + c8);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        xs[c8 + 2 * q][r] = bf16_bits_to_float(w4[q] & 0xFFFFu);
        xs[c8 + 2 * q + 1][r] = bf16_bits_to_float(w4[q] >> 16);
      }
    }
    // W tile: 64 experts x 32 fp32.
    for (int i = tid; i < kBE * (kBK / 4); i += kRouterThreads) {
      const int r = i / (kBK / 4), c4 = (i % (kBK / 4)) * 4;
      const int e = e0 + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E) v = *reinterpret_cast<const float4*>(Wr + size_t(e) * d + k0 + c4);
      ws[c4][r] = v.x;
      ws[c4 + 1][r] = v.y;
      ws[c4 + 2][r] = v.z;
      ws[c4 + 3][r] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kBK; ++kk) {
      float a[TT], b[TE];
#pragma unroll
      for (int i = 0; i < TT; ++i) a[i] = xs[kk][ty * TT + i];
      const float4 bv = *reinterpret_cast<const float4*>(&ws[kk][tx * TE]);
      b[0] = bv.x;
      b[1] = bv.y;
      b[2] = bv.z;
      b[3] = bv.w;
#pragma unroll
      for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TT; ++i) {
    const int t = t0 + ty * TT + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < TE; ++j) {
      const int e = e0 + tx * TE + j;
      if (e < E) part[(size_t(ks) * T + t) * E + e] = acc[i][j];
    }
  }
}

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

// EPL = experts per lane (E <= 32 * EPL); expert e lives in lane e % 32, slot e / 32.
template <int EPL>
__global__ void __launch_bounds__(kRouterThreads)
    router_topk_kernel(const float* __restrict__ part, const float* __restrict__ bias, int T, int E,
                       int k, int ksplit, int32_t* __restrict__ topk_idx,
                       float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (kRouterThreads / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[EPL];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    if (e < E) {
      float s = 0.f;
      for (int ks = 0; ks < ksplit; ++ks) s += part[(size_t(ks) * T + t) * E + e];
      if (bias) s += bias[e];
      v[j] = (s == s) ? s : -INFINITY;  // a NaN score is never preferred
    } else {
      v[j] = -INFINITY;
      taken |= 1u << j;
    }
  }
  float my_l = 0.f, l0 = 0.f;
  int my_e = 0;
  for (int i = 0; i < k; ++i) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (!((taken >> j) & 1u) && better(v[j], e, bv, be)) {
        bv = v[j];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (better(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (i == 0) l0 = bv;
    if (lane == i) {
      my_l = bv;
      my_e = be;
    }
  }
  float ex = (lane < k) ? expf(my_l - l0) : 0.f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    topk_idx[size_t(t) * k + lane] = my_e;
    topk_w[size_t(t) * k + lane] = ex / sum;
  }
}

}  // namespace

RouterPlan router_plan(const Ctx& c, int T, int num_sms) {
  RouterPlan rp;
  rp.bt = T <= 16 ? 16 : 64;
  const int tiles = ((T + rp.bt - 1) / rp.bt) * ((c.E + kBE - 1) / kBE);
  const int kblocks = c.d / kBK;
  const int want = (2 * (num_sms > 0 ? num_sms : 148) + tiles - 1) / tiles;
  int ks = 1;
  for (int cand = 1; cand <= kblocks && cand <= 64; ++cand)
    if (kblocks % cand == 0 && cand <= want) ks = cand;
  rp.ksplit = ks;
  rp.kchunk = c.d / ks;
  return rp;
}

cudaError_t launch_router(const Ctx& c, const RouterPlan& rp, const uint16_t* x, const float* Wr,
                          const float* bias, int T, float* part, int32_t* topk_idx, float* topk_w,
                          cudaStream_t st) {
  dim3 grid((T + rp.bt - 1) / rp.bt, (c.E + kBE - 1) / kBE, rp.ksplit);
  if (rp.bt == 16)
    router_partial_kernel<16><<<grid, kRouterThreads, 0, st>>>(x, Wr, T, c.d, c.E, rp.kchunk,
                                                              part);
  else
    router_partial_kernel<64><<<grid, kRouterThreads, 0, st>>>(x, Wr, T, c.d, c.E, rp.kchunk,
                                                              part);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int blocks = (T + kRouterThreads / 32 - 1) / (kRouterThreads / 32);
  const int epl = (c.E + 31) / 32;
#define MOE_TOPK_CASE(N)                                                                       \
  case N:                                                                                      \
    router_topk_kernel<N><<<blocks, kRouterThreads, 0, st>>>(part, bias, T, c.E, c.k,          \
                                                             rp.ksplit, topk_idx, topk_w);     \
    break;
  const int epl_p2 = epl <= 1 ? 1 : epl <= 2 ? 2 : epl <= 4 ? 4 : epl <= 8 ? 8 : epl <= 16 ? 16
                                                                                         : 32;
  switch (epl_p2) {
    MOE_TOPK_CASE(1)
    MOE_TOPK_CASE(2)
    MOE_TOPK_CASE(4)
    MOE_TOPK_CASE(8)
    MOE_TOPK_CASE(16)
    MOE_TOPK_CASE(32)
  }
#undef MOE_TOPK_CASE
  return cudaGetLastError();
}

}  // namespace moe
