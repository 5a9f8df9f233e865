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
//                  bf16 exactly.  A CTA computes a (tokens x experts) tile --
//                  16 x 64, 64 x 64 or 128 x 128 by batch size -- for one
//                  K-chunk; the chunk count is chosen so the grid fills the GPU
//                  even for 16 tokens.
//  router_topk     one CTA per token adds the chunk partials in a fixed order,
//                  then k rounds of a warp arg-max (value desc, expert asc)
//                  select the experts; the gate of choice i is
//                  exp(l_i - l_0) / sum_j exp(l_j - l_0).
#include <math.h>

#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kBK = 16;   // K per shared-memory stage

// Partial logits of a BT x BE (tokens x experts) tile over one K chunk, fp32
// FFMA.  256 threads, each owning TT tokens x TE experts (split in two halves
// of the tile for conflict-free 16-byte shared loads when TT, TE = 8); the K
// loop is double-buffered: the next stage's global loads are issued before
// the current stage's FMAs.
template <int BT, int BE, int TT, int TE>
__global__ void __launch_bounds__(kRouterThreads)
    router_partial_kernel(const uint16_t* __restrict__ x, const float* __restrict__ Wr, int T,
                          int d, int E, int kchunk, float* __restrict__ part) {
  static_assert((BT / TT) * (BE / TE) == kRouterThreads, "thread tiling");
  static_assert(TE == 4 || TE == 8, "experts per thread");
  constexpr int NTX = BE / TE;                 // threads along experts
  constexpr int HT = (TT == 8) ? TT / 2 : TT;  // tokens per half
  constexpr int HE = (TE == 8) ? TE / 2 : TE;
  constexpr int X_LOADS = BT * kBK / 8;        // 16-byte loads of x per stage
  constexpr int W_LOADS = BE * kBK / 4;        // 16-byte loads of W per stage
  constexpr int XL = (X_LOADS + kRouterThreads - 1) / kRouterThreads;
  constexpr int WL = (W_LOADS + kRouterThreads - 1) / kRouterThreads;
  __shared__ __align__(16) float xs[2][kBK][BT + 4];
  __shared__ __align__(16) float ws[2][kBK][BE + 4];

  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  const int tx = tid % NTX, ty = tid / NTX;
  const int t0 = blockIdx.x * BT, e0 = blockIdx.y * BE;
  const int kbeg = blockIdx.z * kchunk;
  const int nk = kchunk / kBK;

  uint4 xr[XL];
  float4 wr[WL][1];
  auto load_global = [&](int k0) {
#pragma unroll
    for (int l = 0; l < XL; ++l) {
      const int i = tid + l * kRouterThreads;
      xr[l] = make_uint4(0, 0, 0, 0);
      if (i < X_LOADS) {
        const int r = i / (kBK / 8), c8 = (i % (kBK / 8)) * 8;
        if (t0 + r < T) xr[l] = *reinterpret_cast<const uint4*>(x + size_t(t0 + r) * d + k0 + c8);
      }
    }
#pragma unroll
    for (int l = 0; l < WL; ++l) {
      const int i = tid + l * kRouterThreads;
      wr[l][0] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < W_LOADS) {
        const int r = i / (kBK / 4), c4 = (i % (kBK / 4)) * 4;
        if (e0 + r < E)
          wr[l][0] = *reinterpret_cast<const float4*>(Wr + size_t(e0 + r) * d + k0 + c4);
      }
    }
  };
  auto store_smem = [&](int buf) {
#pragma unroll
    for (int l = 0; l < XL; ++l) {
      const int i = tid + l * kRouterThreads;
      if (i < X_LOADS) {
        const int r = i / (kBK / 8), c8 = (i % (kBK / 8)) * 8;
        const uint32_t w4[4] = {xr[l].x, xr[l].y, xr[l].z, xr[l].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xs[buf][c8 + 2 * q][r] = bf16_bits_to_float(w4[q] & 0xFFFFu);
          xs[buf][c8 + 2 * q + 1][r] = bf16_bits_to_float(w4[q] >> 16);
        }
      }
    }
#pragma unroll
    for (int l = 0; l < WL; ++l) {
      const int i = tid + l * kRouterThreads;
      if (i < W_LOADS) {
        const int r = i / (kBK / 4), c4 = (i % (kBK / 4)) * 4;
        ws[buf][c4][r] = wr[l][0].x;
        ws[buf][c4 + 1][r] = wr[l][0].y;
        ws[buf][c4 + 2][r] = wr[l][0].z;
        ws[buf][c4 + 3][r] = wr[l][0].w;
      }
    }
  };

  float acc[TT][TE];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

  load_global(kbeg);
  store_smem(0);
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load_global(kbeg + (kt + 1) * kBK);
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[TT], b[TE];
      if constexpr (HT == 4) {   // 16-byte shared loads: a float4 per half tile
#pragma unroll
        for (int h = 0; h < TT / 4; ++h) {
          const float4 v =
              *reinterpret_cast<const float4*>(&xs[buf][kk][h * (BT / 2) * (TT / 4 - 1) + ty * 4]);
          a[4 * h] = v.x; a[4 * h + 1] = v.y; a[4 * h + 2] = v.z; a[4 * h + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < TT; ++i) a[i] = xs[buf][kk][ty * TT + i];
      }
#pragma unroll
      for (int h = 0; h < TE / 4; ++h) {
        const float4 v =
            *reinterpret_cast<const float4*>(&ws[buf][kk][h * (BE / 2) * (TE / 4 - 1) + tx * 4]);
        b[4 * h] = v.x; b[4 * h + 1] = v.y; b[4 * h + 2] = v.z; b[4 * h + 3] = v.w;
      }
#pragma unroll
      for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nk) store_smem(buf ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TT; ++i) {
    const int t = t0 + (i / HT) * (BT / 2) * (TT / HT - 1) + ty * HT + (i % HT);
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < TE; ++j) {
      const int e = e0 + (j / HE) * (BE / 2) * (TE / HE - 1) + tx * HE + (j % HE);
      if (e < E) part[(size_t(blockIdx.z) * T + t) * E + e] = acc[i][j];
    }
  }
}

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

// TPC tokens per CTA.  The threads of a token add the K-chunk partials of its
// experts in chunk order (plus the bias) into shared memory; the token's first
// warp then takes k rounds of a warp arg-max (value desc, expert asc) over the E
// logits and writes the experts and their renormalised softmax gates.
// TPC = 1 (all of a CTA's threads per token) suits many partials per logit (the
// small-batch split); TPC = 8 (a warp per token) suits few.
template <int TPC>
__global__ void __launch_bounds__(1024)
    router_topk_kernel(const float* __restrict__ part, const float* __restrict__ bias, int T, int E,
                       int k, int ksplit, int nsub, int32_t* __restrict__ topk_idx,
                       float* __restrict__ topk_w) {
  extern __shared__ float logit_all[];  // [TPC][E], then (TPC == 1) [nsub][E] partial sums
  pdl_wait();
  pdl_launch_dependents();
  const int per_tok = blockDim.x / TPC;                 // threads per token
  const int grp = threadIdx.x / per_tok, tid = threadIdx.x % per_tok;
  const int t = blockIdx.x * TPC + grp;
  if (t >= T) return;   // whole token groups (warps) leave together
  float* logit = logit_all + grp * E;
  // With one CTA per token and threads to spare, nsub threads share an expert: each adds a
  // contiguous run of the split-K partials in order, and the runs are added in order after
  // (nsub is 1 for TPC > 1; the launch sizes shared memory for [1 + nsub][E] floats).
  const int run = (ksplit + nsub - 1) / nsub;
  float* sub = logit_all + TPC * E;
  for (int idx = tid; idx < E * nsub; idx += per_tok) {
    const int e = idx % E, q = idx / E;
    float s = 0.f;
    const float* p = part + size_t(t) * E + e;
    const size_t stride = size_t(T) * E;
    const int k1 = min(ksplit, (q + 1) * run);
    int ks = q * run;
    for (; ks + 8 <= k1; ks += 8) {   // eight independent loads in flight, added in order
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = p[(ks + j) * stride];
#pragma unroll
      for (int j = 0; j < 8; ++j) s += v[j];
    }
    for (; ks < k1; ++ks) s += p[ks * stride];
    if (nsub == 1) {
      if (bias) s += bias[e];
      logit[e] = (s == s) ? s : -INFINITY;  // a NaN score is never preferred
    } else {
      sub[q * E + e] = s;
    }
  }
  if (nsub > 1) {
    __syncthreads();
    for (int e = tid; e < E; e += per_tok) {
      float s = sub[e];
      for (int q = 1; q < nsub; ++q) s += sub[q * E + e];
      if (bias) s += bias[e];
      logit[e] = (s == s) ? s : -INFINITY;
    }
  }
  if (TPC == 1) __syncthreads(); else __syncwarp();
  if (tid >= 32) return;
  const int lane = tid;
  float my_l = 0.f, l0 = 0.f;
  int my_e = 0;
  for (int i = 0; i < k; ++i) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = logit[e];
      if (better(v, e, bv, be)) {
        bv = v;
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
    // every lane holds the winner; its owner removes it from further rounds
    if ((be & 31) == lane) logit[be] = __int_as_float(0xff800001u);  // NaN: never 'better'
    __syncwarp();
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

template <int BT, int BE, int TT, int TE>
cudaError_t launch_partial(const Ctx& c, const RouterPlan& rp, const uint16_t* x, const float* Wr,
                           int T, float* part, cudaStream_t st) {
  dim3 grid((T + BT - 1) / BT, (c.E + BE - 1) / BE, rp.ksplit);
  return launch_pdl(router_partial_kernel<BT, BE, TT, TE>, grid, dim3(kRouterThreads), 0, st, 1,
                    x, Wr, T, c.d, c.E, rp.kchunk, part);
}

}  // namespace

// Path and tile shape by batch size.  The score GEMM runs on the tensor cores
// (router_tc.cu) for more than 32 tokens and on fp32 FFMA tiles otherwise;
// the context's router mode (MOE_ROUTER=tc|ffma at moe_create) forces one.  Both compute fp32-accurate logits.  The FFMA K split is chosen
// so the grid fills the GPU (about two CTAs per SM, counted for a 148-SM part so that the plan,
// and with it the summation order, is the same on every device).
RouterPlan router_plan(const Ctx& c, int T, int num_sms) {
  RouterPlan rp;
  if (c.router == RouterMode::kFfma)
    rp.tc = false;
  else if (c.router == RouterMode::kTensorCore)
    rp.tc = true;
  else
    rp.tc = T > 32;   // below that the FFMA tiles finish first (measured on B200)
  if (rp.tc) {
    rp.bt = 128;
    rp.ksplit = router_tc_ksplit(c, T, num_sms);
    rp.kchunk = c.d / rp.ksplit;
    return rp;
  }
  rp.bt = T <= 16 ? 16 : (T <= 256 ? 64 : 128);
  const int be = rp.bt == 128 ? 128 : 64;
  const int tiles = ((T + rp.bt - 1) / rp.bt) * ((c.E + be - 1) / be);
  const int kblocks = c.d / kBK;
  const int slots = 2 * (num_sms > 0 ? num_sms : 148);
  int best = 1;
  double best_eff = -1.0;
  const int max_split = rp.bt == 128 ? 8 : 64;
  for (int cand = 1; cand <= kblocks && cand <= max_split; ++cand) {
    if (kblocks % cand) continue;
    const int n = tiles * cand;
    const int waves = (n + slots - 1) / slots;
    double eff = double(n) / double(waves * slots);
    if (n < slots / 2) eff *= 0.5;   // too few CTAs to cover the SMs
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = cand;
    }
  }
  rp.ksplit = best;
  rp.kchunk = c.d / best;
  return rp;
}

cudaError_t launch_router(const Ctx& c, const RouterPlan& rp, const uint16_t* x, const float* Wr,
                          const float* bias, int T, float* part, uint16_t* wparts, int* status,
                          int num_sms, int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  cudaError_t err;
  if (rp.tc)
    err = launch_router_tc(c, rp.ksplit, x, Wr, T, wparts, part, status, num_sms, st);
  else if (rp.bt == 16)
    err = launch_partial<16, 64, 1, 4>(c, rp, x, Wr, T, part, st);
  else if (rp.bt == 64)
    err = launch_partial<64, 64, 4, 4>(c, rp, x, Wr, T, part, st);
  else
    err = launch_partial<128, 128, 8, 8>(c, rp, x, Wr, T, part, st);
  if (err != cudaSuccess) return err;
  if (rp.ksplit <= 4)   // a warp per token, 8 tokens per CTA
    return launch_pdl(router_topk_kernel<8>, dim3((T + 7) / 8), dim3(256), 8 * c.E * sizeof(float),
                      st, 1, static_cast<const float*>(part), bias, T, c.E, c.k, rp.ksplit, 1,
                      topk_idx, topk_w);
  // a CTA per token; up to four threads per expert share its partial sums
  const int nsub = std::max(1, std::min(4, std::min(rp.ksplit / 8, 1024 / std::max(1, c.E))));
  const int threads = std::min(1024, std::max(32, (nsub * c.E + 31) / 32 * 32));
  const size_t smem = size_t(1 + nsub) * c.E * sizeof(float);
  return launch_pdl(router_topk_kernel<1>, dim3(T), dim3(threads), smem, st, 1,
                    static_cast<const float*>(part), bias, T, c.E, c.k, rp.ksplit, nsub, topk_idx,
                    topk_w);
}

}  // namespace moe
