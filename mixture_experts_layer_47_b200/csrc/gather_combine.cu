// gather_combine.cu -- the two memory-bound steps around the expert GEMMs.
//
//  gather   X_perm[p] = x[perm[p] / k] for every routed slot position p, so each
//           expert's tokens form one contiguous run of rows for the grouped
//           GEMM's TMA loads (the shared expert reads x directly).  Inside
//           moe_forward a warp takes a token, reads its row once and writes it
//           to its k positions (pos); moe_expert_ffn, given perm only, copies
//           position by position.
//  combine  the merge of the chosen experts' results into the layer output
//           (m.xxqk.cn Hy4-preview MoE explainer, section 2.2; the shared
//           expert of the ZAKER release news is added with weight 1):
//             y[t] = sum_s Y[T*k + s*T + t] + sum_i w[t][i] * Y[pos[t*k + i]]
//           in fp32, in that fixed order, then rounded once to bf16.  Each
//           thread owns 8 consecutive features of one token.  Y is fp32 for
//           moe_combine and bf16 inside moe_forward (half the traffic).  For a
//           shard of the layer (moe_forward_partial) the sum is written in fp32
//           unrounded, and
//  reduce   adds the shards' fp32 partial outputs in rank order and rounds the
//           total once to bf16 (moe_reduce_partials).
//  iHC      the layer inside n parallel residual streams H [T][n][d] (ZAKER Hy4
//           Preview release news, iHC paragraphs: identity Hyper-Connections, four
//           streams recombined at every layer, the identity path kept):
//             mix     x[t]     = sum_j alpha[j] H[t][j]                    -> bf16
//             update  H'[t][i] = H[t][i] + sum_j B[i][j] H[t][j] + gamma[i] y[t]
//           where the update is done by the combine itself, with y[t] its fp32 sum.
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
  pdl_wait();
  pdl_launch_dependents();
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

// Token-major gather: a warp reads a segment of a token's row of x once (held
// in registers) and writes it to the token's k positions pos[t*k + i].  x is
// read once instead of k times, so the X_perm write stream cannot push it out of
// L2.  Work items are (token, segment) pairs; segments are seg_vecs 16-byte
// vectors (a multiple of 32, at most 256), chosen short when there are few
// tokens so that enough warps are in flight.
__global__ void __launch_bounds__(kGatherThreads)
    gather_tokens_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ pos, int T,
                         int k, int d, int seg_vecs, uint16_t* __restrict__ x_perm) {
  pdl_wait();
  pdl_launch_dependents();
  const int nslots = T * k;
  const int warps_total = gridDim.x * (kGatherThreads / 32);
  const int lane = threadIdx.x & 31;
  const int vec = d / 8;  // 16-byte vectors per row
  const int nseg = (vec + seg_vecs - 1) / seg_vecs;
  const int per_lane = seg_vecs / 32;
  constexpr int kChunk = 8;  // vectors per lane held at once (seg_vecs <= 256)
  const int64_t items = int64_t(T) * nseg;
  for (int64_t item = blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); item < items;
       item += warps_total) {
    const int t = int(item / nseg);
    const int base = int(item - int64_t(t) * nseg) * seg_vecs;
    const uint4* __restrict__ src = reinterpret_cast<const uint4*>(x + size_t(t) * d);
    uint4 v[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      const int i = base + lane + 32 * j;
      if (j < per_lane && i < vec) v[j] = src[i];
    }
    for (int c = 0; c < k; ++c) {
      const int p = pos[size_t(t) * k + c];
      if (p < 0 || p >= nslots) continue;
      uint4* __restrict__ dst = reinterpret_cast<uint4*>(x_perm + size_t(p) * d);
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        const int i = base + lane + 32 * j;
        if (j < per_lane && i < vec) dst[i] = v[j];
      }
    }
  }
}

// Eight consecutive values of a row: loaded raw (Raw), then widened to fp32.
struct RowF32 {
  struct Raw {
    float4 a, b;
  };
  __device__ static Raw load(const float* __restrict__ row) {
    return {*reinterpret_cast<const float4*>(row), *reinterpret_cast<const float4*>(row + 4)};
  }
  __device__ static void widen(const Raw& r, float (&v)[8]) {
    v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
    v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
  }
  __device__ static void load8(const float* __restrict__ row, float (&v)[8]) { widen(load(row), v); }
};
struct RowBF16 {
  using Raw = uint4;
  __device__ static Raw load(const uint16_t* __restrict__ row) {
    return *reinterpret_cast<const uint4*>(row);
  }
  __device__ static void widen(const Raw& a, float (&v)[8]) {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[2 * q] = bf16_bits_to_float(w[q] & 0xFFFFu);
      v[2 * q + 1] = bf16_bits_to_float(w[q] >> 16);
    }
  }
  __device__ static void load8(const uint16_t* __restrict__ row, float (&v)[8]) {
    widen(load(row), v);
  }
};

// Store 8 fp32 sums: rounded once to bf16, or (partial output) as they are.
__device__ __forceinline__ void store8(const float (&acc)[8], uint16_t* __restrict__ out) {
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(out) = o;
}
__device__ __forceinline__ void store8(const float (&acc)[8], float* __restrict__ out) {
  *reinterpret_cast<float4*>(out) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  *reinterpret_cast<float4*>(out + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// The merge of token t's rows for features c .. c+7, in fp32: the shared experts' rows,
// then the k weighted rows in order.  TY = float (Y in fp32) or uint16_t (Y in bf16).
template <typename TY, typename Row>
__device__ __forceinline__ void combine_sum8(const TY* __restrict__ Y,
                                             const float* __restrict__ topk_w,
                                             const int32_t* __restrict__ pos, int T, int k,
                                             int S, int d, int t, int c, float (&acc)[8]) {
  const size_t nslots = size_t(T) * k;
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  float v[8];
  for (int s = 0; s < S; ++s) {
    Row::load8(Y + (nslots + size_t(s) * T + t) * d + c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += v[j];
  }
  // The routed rows kChunk at a time: every load of a chunk is issued before its rows are
  // added (in slot order), so a thread keeps several rows in flight.
  constexpr int kChunk = 4;
  for (int i0 = 0; i0 < k; i0 += kChunk) {
    typename Row::Raw r[kChunk];
    float w[kChunk];
    bool live[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      const int i = i0 + j;
      const int p = i < k ? pos[size_t(t) * k + i] : -1;
      live[j] = p >= 0 && size_t(p) < nslots;
      w[j] = live[j] ? topk_w[size_t(t) * k + i] : 0.f;
      if (live[j]) r[j] = Row::load(Y + size_t(p) * d + c);
    }
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      if (!live[j]) continue;
      Row::widen(r[j], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(w[j], v[e], acc[e]);
    }
  }
}

// TOut = uint16_t (y in bf16) or float (a shard's unrounded partial output).
template <typename TY, typename Row, typename TOut>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const TY* __restrict__ Y, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ pos, int T, int k, int S, int d,
                   TOut* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const int c = (blockIdx.y * kCombineThreads + threadIdx.x) * 8;
  if (c >= d) return;
  float acc[8];
  combine_sum8<TY, Row>(Y, topk_w, pos, T, k, S, d, t, c, acc);
  store8(acc, y + size_t(t) * d + c);
}

// The iHC stream update done by the combine: y[t] stays in fp32 registers, every stream's
// 8 features are read once, and H'[t][i] = H[t][i] + sum_j B[i][j] H[t][j] + gamma[i] y[t]
// (identity term, then the exchange terms in j order, then the layer output) is rounded once
// to bf16.  H_out may be H: each thread reads its elements of all streams before writing.
__global__ void __launch_bounds__(kCombineThreads)
    combine_ihc_kernel(const uint16_t* __restrict__ Y, const float* __restrict__ topk_w,
                       const int32_t* __restrict__ pos, int T, int k, int S, int d,
                       const uint16_t* H, const float* __restrict__ Bm,
                       const float* __restrict__ gamma, int n, uint16_t* H_out) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const int c = (blockIdx.y * kCombineThreads + threadIdx.x) * 8;
  if (c >= d) return;
  float acc[8];
  combine_sum8<uint16_t, RowBF16>(Y, topk_w, pos, T, k, S, d, t, c, acc);
  float h[kMaxStreams][8];
#pragma unroll
  for (int j = 0; j < kMaxStreams; ++j)
    if (j < n) RowBF16::load8(H + (size_t(t) * n + j) * d + c, h[j]);
#pragma unroll
  for (int i = 0; i < kMaxStreams; ++i) {
    if (i < n) {
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = h[i][e];
#pragma unroll
      for (int j = 0; j < kMaxStreams; ++j) {
        if (j < n) {
          const float b = Bm[i * n + j];
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = fmaf(b, h[j][e], o[e]);
        }
      }
      const float g = gamma[i];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = fmaf(g, acc[e], o[e]);
      store8(o, H_out + (size_t(t) * n + i) * d + c);
    }
  }
}

// iHC layer input: x[t] = bf16(sum_j alpha[j] H[t][j]), fp32 in j order.
__global__ void __launch_bounds__(kCombineThreads)
    ihc_mix_kernel(const uint16_t* __restrict__ H, const float* __restrict__ alpha, int n,
                   int d, uint16_t* __restrict__ x) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const int c = (blockIdx.y * kCombineThreads + threadIdx.x) * 8;
  if (c >= d) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < n; ++j) {
    float v[8];
    RowBF16::load8(H + (size_t(t) * n + j) * d + c, v);
    const float a = alpha[j];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(a, v[e], acc[e]);
  }
  store8(acc, x + size_t(t) * d + c);
}

// y[i] = bf16(sum_{r < n} part_r[i]) in fp32, r in order; 8 elements per thread per step.
__global__ void __launch_bounds__(kCombineThreads)
    reduce_partials_kernel(PartialPtrs parts, int n, size_t n_vec8, uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t v = size_t(blockIdx.x) * kCombineThreads + threadIdx.x; v < n_vec8;
       v += size_t(gridDim.x) * kCombineThreads) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < kMaxPartials; ++r) {   // unrolled: the pointers stay in registers
      if (r < n) {
        float x[8];
        RowF32::load8(parts.p[r] + v * 8, x);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += x[j];
      }
    }
    store8(acc, y + v * 8);
  }
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
  return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(kGatherThreads), 0, st, 1, x, perm,
                    offsets, T, c.k, c.E, c.d, x_perm);
}

cudaError_t launch_gather_tokens(const Ctx& c, const uint16_t* x, const int32_t* pos, int T,
                                 uint16_t* x_perm, int num_sms, cudaStream_t st) {
  const int warps_per_block = kGatherThreads / 32;
  const int vec = c.d / 8;
  // 4 KB segments, or 1 KB ones when 4 KB segments would leave most SMs idle
  int seg_vecs = 256;
  if (int64_t(T) * ((vec + 255) / 256) < int64_t(4) * num_sms) seg_vecs = 64;
  const int64_t items = int64_t(T) * ((vec + seg_vecs - 1) / seg_vecs);
  int64_t blocks = (items + warps_per_block - 1) / warps_per_block;
  if (blocks > int64_t(num_sms) * 8) blocks = int64_t(num_sms) * 8;
  if (blocks < 1) blocks = 1;
  return launch_pdl(gather_tokens_kernel, dim3(unsigned(blocks)), dim3(kGatherThreads), 0, st, 1,
                    x, pos, T, c.k, c.d, seg_vecs, x_perm);
}

cudaError_t launch_combine(const Ctx& c, const float* Y, const float* topk_w, const int32_t* pos,
                           int T, uint16_t* y, cudaStream_t st) {
  dim3 grid(T, (c.d / 8 + kCombineThreads - 1) / kCombineThreads);
  return launch_pdl(combine_kernel<float, RowF32, uint16_t>, grid, dim3(kCombineThreads), 0, st,
                    1, Y, topk_w, pos, T, c.k, c.S, c.d, y);
}

cudaError_t launch_combine_bf16(const Ctx& c, const uint16_t* Y, const float* topk_w,
                                const int32_t* pos, int T, uint16_t* y, cudaStream_t st) {
  dim3 grid(T, (c.d / 8 + kCombineThreads - 1) / kCombineThreads);
  return launch_pdl(combine_kernel<uint16_t, RowBF16, uint16_t>, grid, dim3(kCombineThreads), 0,
                    st, 1, Y, topk_w, pos, T, c.k, c.S, c.d, y);
}

cudaError_t launch_combine_partial(const Ctx& c, const uint16_t* Y, const float* topk_w,
                                   const int32_t* pos, int T, float* y_partial,
                                   cudaStream_t st) {
  dim3 grid(T, (c.d / 8 + kCombineThreads - 1) / kCombineThreads);
  return launch_pdl(combine_kernel<uint16_t, RowBF16, float>, grid, dim3(kCombineThreads), 0, st,
                    1, Y, topk_w, pos, T, c.k, c.S, c.d, y_partial);
}

cudaError_t launch_ihc_mix(const Ctx& c, const uint16_t* H, const float* alpha, int n, int T,
                           uint16_t* x, cudaStream_t st) {
  dim3 grid(T, (c.d / 8 + kCombineThreads - 1) / kCombineThreads);
  return launch_pdl(ihc_mix_kernel, grid, dim3(kCombineThreads), 0, st, 1, H, alpha, n, c.d, x);
}

cudaError_t launch_combine_ihc(const Ctx& c, const uint16_t* Y, const float* topk_w,
                               const int32_t* pos, int T, const uint16_t* H, const float* B,
                               const float* gamma, int n, uint16_t* H_out, cudaStream_t st) {
  dim3 grid(T, (c.d / 8 + kCombineThreads - 1) / kCombineThreads);
  return launch_pdl(combine_ihc_kernel, grid, dim3(kCombineThreads), 0, st, 1, Y, topk_w, pos, T,
                    c.k, c.S, c.d, H, B, gamma, n, H_out);
}

cudaError_t launch_reduce_partials(const PartialPtrs& parts, int n, size_t elems, uint16_t* y,
                                   int num_sms, cudaStream_t st) {
  const size_t n_vec8 = elems / 8;
  size_t blocks = (n_vec8 + kCombineThreads - 1) / kCombineThreads;
  const size_t cap = size_t(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_pdl(reduce_partials_kernel, dim3(unsigned(blocks)), dim3(kCombineThreads), 0, st,
                    1, parts, n, n_vec8, y);
}

}  // namespace moe
