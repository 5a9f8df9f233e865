// dispatch.cu -- group the (token, choice) slots by expert on sm_100a.
//
// The pages' explainer (m.xxqk.cn Hy4-preview MoE, section 2.2) has the
// activated experts process the tokens routed to them; grouping the slots
// s = t*k + i per expert makes each expert's tokens one contiguous segment
// that a grouped GEMM can read.  The grouping is a stable counting sort,
// deterministic by construction (no order-dependent atomics):
//   dispatch_count    per block of 4096 slots, a shared-memory histogram
//                     (integer atomics: the counts do not depend on order);
//   dispatch_scan     one CTA: for every expert the exclusive prefix over
//                     blocks, counts, the exclusive scan over experts
//                     (offsets), and the grouped GEMMs' tile schedules;
//   dispatch_scatter  per block, each warp owns a contiguous run of slots;
//                     __match_any_sync gives each slot its rank among equal
//                     experts in the warp; per-warp, per-expert running
//                     counts make the order ascending in slot index.
// Up to 4096 slots and 256 experts the three steps run in one CTA
// (dispatch_single).
//
// The experts grouped are the E experts e_base .. e_base + E - 1 of a layer of
// e_all routed experts (e_base = 0, e_all = E for the whole layer; a range of
// them when the experts are sharded over GPUs).  A slot routed to an expert
// outside the range is skipped (pos = -1); an index outside [0, e_all) is
// skipped too and flagged in the status word.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kCountThreads = 512;
constexpr int kScatterWarps = 8;
constexpr int kScanThreads = 1024;
constexpr int kTileM = 128;   // rows (tokens) per grouped-GEMM tile of the 1-SM tilings

// The local group of a routed expert index g, or -1 when g is outside the
// local range [e_base, e_base + E).
__device__ __forceinline__ int local_group(int g, int e_base, int E) {
  const int e = g - e_base;
  return (e >= 0 && e < E) ? e : -1;
}

__global__ void __launch_bounds__(kCountThreads)
    dispatch_count_kernel(const int32_t* __restrict__ idx, int n, int E, int e_base, int e_all,
                          int32_t* __restrict__ blk_hist, int* status) {
  extern __shared__ int32_t hist[];
  pdl_wait();
  pdl_launch_dependents();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int beg = blockIdx.x * kDispatchChunk;
  const int end = min(n, beg + kDispatchChunk);
  bool bad = false;
  for (int s = beg + threadIdx.x; s < end; s += blockDim.x) {
    const int g = idx[s];
    const int e = local_group(g, e_base, E);
    if (e >= 0) atomicAdd(&hist[e], 1);
    if (g < 0 || g >= e_all) bad = true;
  }
  if (bad) report_error(status, kDevBadIndex, kSiteDispatch);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) blk_hist[size_t(blockIdx.x) * E + e] = hist[e];
}

// Inclusive block-wide scan of one int per thread (blockDim.x == kScanThreads).
__device__ int block_inclusive_scan(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int r = v + (warp > 0 ? warp_sums[warp - 1] : 0);
  __syncthreads();
  return r;
}

// Grouped-GEMM schedules: sched[g] = sum over groups g' < g of ceil(rows_g' / 128),
// routed groups first (rows = count), then S shared groups of T rows each; the
// same for 256-row tiles (the 2-SM GEMMs) at sched[G + 1 + g], G = E + S.  The
// row-tiled GEMMs read them as M tiles per group, the weight-major ones as
// token tiles per group.
__device__ void write_schedule(int count, int E, int S, int T, int32_t* sched, int* warp_sums) {
  const int e = threadIdx.x;
  const int G1 = E + S + 1;
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const int tm = which == 0 ? kTileM : 2 * kTileM;
    int32_t* out = sched + which * G1;
    const int mt = (e < E) ? (count + tm - 1) / tm : 0;
    const int incl = block_inclusive_scan(mt, warp_sums);
    if (e < E) out[e] = incl - mt;
    if (e == E - 1) {
      const int mts = (T + tm - 1) / tm;
      for (int s = 0; s <= S; ++s) out[E + s] = incl + s * mts;
    }
  }
}

__global__ void __launch_bounds__(kScanThreads)
    dispatch_scan_kernel(int32_t* __restrict__ blk_hist, int nblk, int E, int S, int T,
                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ sched) {
  __shared__ int warp_sums[32];
  pdl_wait();
  pdl_launch_dependents();
  const int e = threadIdx.x;
  int c = 0;
  if (e < E) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      const int h = blk_hist[size_t(b) * E + e];
      blk_hist[size_t(b) * E + e] = run;
      run += h;
    }
    c = run;
    counts[e] = c;
  }
  const int incl = block_inclusive_scan(c, warp_sums);
  const int excl = incl - c;
  if (e < E) {
    offsets[e] = excl;
    for (int b = 0; b < nblk; ++b) blk_hist[size_t(b) * E + e] += excl;
  }
  if (e == E - 1) offsets[E] = incl;
  write_schedule(c, E, S, T, sched, warp_sums);
}

__global__ void __launch_bounds__(kScanThreads)
    schedule_from_offsets_kernel(const int32_t* __restrict__ offsets, int E, int S, int T,
                                 int32_t* __restrict__ sched) {
  __shared__ int warp_sums[32];
  pdl_wait();
  pdl_launch_dependents();
  const int e = threadIdx.x;
  int c = 0;
  // A group never holds more than T slots (a token picks an expert once).
  if (e < E) c = min(T, max(0, offsets[e + 1] - offsets[e]));
  write_schedule(c, E, S, T, sched, warp_sums);
}

// The dense FFN as a one-group layer: offsets = {0, T} and the schedules of
// one routed group of T rows and no shared group.
__global__ void __launch_bounds__(kScanThreads)
    dense_schedule_kernel(int T, int32_t* __restrict__ offsets, int32_t* __restrict__ sched) {
  __shared__ int warp_sums[32];
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    offsets[0] = 0;
    offsets[1] = T;
  }
  write_schedule(threadIdx.x == 0 ? T : 0, 1, 0, T, sched, warp_sums);
}

__global__ void __launch_bounds__(kScatterWarps * 32)
    dispatch_scatter_kernel(const int32_t* __restrict__ idx, int n, int E, int e_base,
                            const int32_t* __restrict__ blk_base, int32_t* __restrict__ perm,
                            int32_t* __restrict__ pos) {
  extern __shared__ int32_t cnt[];  // [kScatterWarps][E]
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  constexpr int kPerWarp = kDispatchChunk / kScatterWarps;
  const int beg = blockIdx.x * kDispatchChunk + warp * kPerWarp;
  const int end = min(n, beg + kPerWarp);
  int32_t* my = cnt + warp * E;

  for (int s0 = beg; s0 < end; s0 += 32) {
    const int s = s0 + lane;
    const int e = (s < end) ? local_group(idx[s], e_base, E) : -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(m) - 1) my[e] += __popc(m);
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = blk_base[size_t(blockIdx.x) * E + e];
    for (int w = 0; w < kScatterWarps; ++w) {
      const int c = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int s0 = beg; s0 < end; s0 += 32) {
    const int s = s0 + lane;
    const int e = (s < end) ? local_group(idx[s], e_base, E) : -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(m & ((1u << lane) - 1u));
    const int base = (e >= 0) ? my[e] : 0;
    __syncwarp();
    if (e >= 0) {
      const int p = base + rank;
      perm[p] = s;
      pos[s] = p;
      if (lane == __ffs(m) - 1) my[e] = base + __popc(m);
    } else if (s < end) {
      pos[s] = -1;   // a skipped slot: no position, left out of the combine
    }
    __syncwarp();
  }
}

// Small dispatches (n <= 4096 slots, E <= 256) in one CTA of 1024 threads:
// per-warp counts (as in dispatch_scatter), then per expert the prefix over
// warps and the totals, the exclusive scan over experts and the schedules,
// then the stable scatter.  One launch instead of three.
constexpr int kSingleWarps = kScanThreads / 32;
constexpr int kSingleMaxExperts = 256;

__global__ void __launch_bounds__(kScanThreads)
    dispatch_single_kernel(const int32_t* __restrict__ idx, int n, int E, int e_base, int e_all,
                           int S, int T, int32_t* __restrict__ counts,
                           int32_t* __restrict__ offsets,
                           int32_t* __restrict__ perm, int32_t* __restrict__ pos,
                           int32_t* __restrict__ sched, int* status) {
  extern __shared__ int32_t cnt[];  // [kSingleWarps][E]
  __shared__ int warp_sums[32];
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kSingleWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  constexpr int kPerWarp = kDispatchChunk / kSingleWarps;
  const int beg = warp * kPerWarp;
  const int end = min(n, beg + kPerWarp);
  int32_t* my = cnt + warp * E;
  bool bad = false;
  for (int s0 = beg; s0 < end; s0 += 32) {
    const int s = s0 + lane;
    const int g = (s < end) ? idx[s] : 0;
    if (g < 0 || g >= e_all) bad = true;
    const int e = (s < end) ? local_group(g, e_base, E) : -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(m) - 1) my[e] += __popc(m);
    __syncwarp();
  }
  if (bad) report_error(status, kDevBadIndex, kSiteDispatch);
  __syncthreads();
  const int e = threadIdx.x;
  int c = 0;
  if (e < E) {
    int run = 0;
    for (int w = 0; w < kSingleWarps; ++w) {
      const int v = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += v;
    }
    c = run;
    counts[e] = c;
  }
  const int incl = block_inclusive_scan(c, warp_sums);
  const int excl = incl - c;
  if (e < E) {
    offsets[e] = excl;
    for (int w = 0; w < kSingleWarps; ++w) cnt[w * E + e] += excl;
  }
  if (e == E - 1) offsets[E] = incl;
  write_schedule(c, E, S, T, sched, warp_sums);
  __syncthreads();
  for (int s0 = beg; s0 < end; s0 += 32) {
    const int s = s0 + lane;
    const int e2 = (s < end) ? local_group(idx[s], e_base, E) : -1;
    const unsigned m = __match_any_sync(0xffffffffu, e2);
    const int rank = __popc(m & ((1u << lane) - 1u));
    const int base = (e2 >= 0) ? my[e2] : 0;
    __syncwarp();
    if (e2 >= 0) {
      const int p = base + rank;
      perm[p] = s;
      pos[s] = p;
      if (lane == __ffs(m) - 1) my[e2] = base + __popc(m);
    } else if (s < end) {
      pos[s] = -1;   // a skipped slot: no position, left out of the combine
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_dispatch(const Ctx& c, const int32_t* topk_idx, int T, int nblk,
                            int32_t* blk_hist, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* pos, int32_t* sched, int* status, cudaStream_t st) {
  const int n = T * c.k;
  const int e_all = c.e_all();
  if (n <= kDispatchChunk && c.E <= kSingleMaxExperts) {
    return launch_pdl(dispatch_single_kernel, dim3(1), dim3(kScanThreads),
                      kSingleWarps * c.E * sizeof(int32_t), st, 1, topk_idx, n, c.E, c.e_base,
                      e_all, c.S, T, counts, offsets, perm, pos, sched, status);
  }
  cudaError_t err = launch_pdl(dispatch_count_kernel, dim3(nblk), dim3(kCountThreads),
                               c.E * sizeof(int32_t), st, 1, topk_idx, n, c.E, c.e_base, e_all,
                               blk_hist, status);
  if (err != cudaSuccess) return err;
  err = launch_pdl(dispatch_scan_kernel, dim3(1), dim3(kScanThreads), 0, st, 1, blk_hist, nblk,
                   c.E, c.S, T, counts, offsets, sched);
  if (err != cudaSuccess) return err;
  return launch_pdl(dispatch_scatter_kernel, dim3(nblk), dim3(kScatterWarps * 32),
                    kScatterWarps * c.E * sizeof(int32_t), st, 1, topk_idx, n, c.E, c.e_base,
                    static_cast<const int32_t*>(blk_hist), perm, pos);
}

cudaError_t launch_dense_schedule(int T, int32_t* offsets, int32_t* sched, cudaStream_t st) {
  return launch_pdl(dense_schedule_kernel, dim3(1), dim3(kScanThreads), 0, st, 1, T, offsets,
                    sched);
}

cudaError_t launch_schedule_from_offsets(const Ctx& c, const int32_t* offsets, int T,
                                         int32_t* sched, cudaStream_t st) {
  return launch_pdl(schedule_from_offsets_kernel, dim3(1), dim3(kScanThreads), 0, st, 1, offsets,
                    c.E, c.S, T, sched);
}

}  // namespace moe
