// expert_gemm_swap.cu -- grouped expert GEMMs with the weights as the MMA's M side.
//
// Same contractions as expert_gemm.cu (m.xxqk.cn Hy4-preview MoE explainer,
// section 2.1: each expert is an FFN sub-network; ZAKER Hy4 Preview release
// news: 256 routed experts plus one shared expert):
//   gate/up:  H_g = silu(X_g W_gate_g^T) * (X_g W_up_g^T)   -> bf16
//   down:     Y_g = H_g W_down_g^T                           -> fp32 or bf16
// but each tcgen05.mma computes D^T = W X^T: the A operand is 128 weight rows
// (output features) and the B operand is a tile of the group's tokens.  The
// M side of a tile is then always full, and a group of n tokens is cut into
// ceil(n/128) token tiles of near-equal width rounded up to 16 (the MMA's N
// step), so a group pays for at most 15 padding tokens per tile instead of up
// to 127 padding rows of a 128-row M tile.  At prefill sizes (a few hundred
// tokens per expert) that recovers most of the tensor work the row-tiled
// kernel spends on padding.
//
// Two tilings share the kernel template:
//   1-SM (kPair = false): two M=128 MMAs per K step share one token tile of
//     N <= 128 --
//       gate/up  A0 = 128 gate rows, A1 = the matching 128 up rows, so the two
//                fp32 accumulators hold gate and up of the same features in the
//                same TMEM lanes and the epilogue forms SwiGLU lane-locally;
//       down     A0, A1 = 256 consecutive W_down rows;
//     two 256-column accumulators, double buffered.
//   2-SM (kPair = true): a CTA pair runs tcgen05.mma.cta_group::2 with M = 256
//     weight rows (128 per CTA) and a token tile of N <= 256 whose rows are
//     split between the two CTAs' shared memory --
//       gate/up  a gate MMA and an up MMA per K step,
//       down     two MMAs per K step on 512 consecutive W_down rows,
//     accumulators at TMEM columns [0, N) and [256, 256+N) (one 512-column
//     buffer: the epilogue reads the tile into registers, rounded to bf16, and
//     hands TMEM back before it stores).
//     Each CTA stages its 128 weight rows and half the tokens, so a CTA moves
//     about half the shared-memory bytes per MMA cycle of the 1-SM tiling --
//     on sm_100a the TMA writes and the tensor core's operand reads share the
//     SM's shared-memory bandwidth, which is what limits the 1-SM tilings.
// Roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer (the pair's
// leader CTA issues for both), warps 2-9 epilogue (two per TMEM lane quarter,
// taking alternate 32-token chunks).  The accumulator is
// feature-major (TMEM lane = feature, column = token), so the epilogue
// transposes each 32x32 block through shared memory and stores whole output
// rows.  Every wait is bounded; on expiry the kernel records the fault,
// drains, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tensor_map.cuh"
#include "weight_major.cuh"

namespace moe {
namespace {

constexpr int BK = 64;                     // K elements per stage
constexpr int WM = 128;                    // weight rows per CTA per MMA
constexpr int W_BYTES = WM * BK * 2;       // one A box
constexpr int B_BOX = 128;                 // token rows per CTA per stage
constexpr int B_BYTES = B_BOX * BK * 2;    // one B box
constexpr int EPI_WARPS = 8;               // two per TMEM lane quarter
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int TMEM_COLS = 512;
constexpr int MAX_GROUPS = 1024 + 8;
constexpr int MAX_STAGES = 6;

// Every tiling issues two MMAs per K step that share the token tile (their A operands are
// the gate and up rows, or two consecutive blocks of W_down rows).  Measured on B200 at Hy4
// prefill (T = 8192, two alternating repetitions): 2-SM down tiles of 512 W_down rows (two
// 256-row MMAs per K step) take 2.01-2.04 ms against 2.29-2.30 for 256-row tiles with one
// MMA per K step; the gate/up tiles already issue two MMAs per step and reach about 103
// cycles per MMA where the single-MMA down tiles took 163.
template <bool kGateUp, bool kPair>
struct SwapCfg {
  static constexpr int TN = kPair ? 256 : 128;               // largest token tile (MMA N)
  static constexpr int NUM_A = 2;                            // A boxes per stage
  static constexpr int STAGE_BYTES = NUM_A * W_BYTES + B_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int NUM_ACC = kPair ? 1 : 2;
  static constexpr int ACC_STRIDE = TMEM_COLS / NUM_ACC;
  static constexpr int SECOND = kPair ? 256 : 128;           // TMEM column of the 2nd MMA's D
  static constexpr int A_ROWS = kPair ? 2 * WM : WM;         // weight rows of one MMA's A
  static constexpr int FEAT = kGateUp ? A_ROWS : 2 * A_ROWS; // output features per tile
  static constexpr int MMA_M = kPair ? 256 : 128;
  static constexpr int EPI_THREADS = (kPair ? 2 : 1) * 32 * EPI_WARPS;  // arrivals freeing an acc
};

struct __align__(64) SwapParams {
  CUtensorMap tok_routed;  // gate/up: X_perm [T*k][d]; down: H [T*k+S*T][F]   (box 128 rows)
  CUtensorMap tok_shared;  // gate/up: x [T][d];        down: same as tok_routed
  CUtensorMap w0;          // gate/up: W_gate [E*F][d]; down: W_down [E*d][F]  (box 128 rows)
  CUtensorMap w1;          // gate/up: W_up   [E*F][d]; down: unused
  CUtensorMap s0;          // shared-expert counterparts of w0 / w1
  CUtensorMap s1;
  const int32_t* offsets;  // [E+1]
  const int32_t* sched;    // [E+S+1] prefix sums of ceil(rows / TN) per group
  void* out;               // gate/up: H bf16; down: Y fp32, or bf16 when out_bf16
  int* status;
  int out_bf16;
  int T, E, S, k;
  int K;                   // reduction length (d or F)
  int n_out;               // output features per group (F or d)
  int w_rows;              // weight rows per expert in the w maps (F or d)
  int out_rows;            // rows of the output buffer (T*k + S*T)
  int ksplit;              // down, 1-SM only: K ranges per output tile (1 = no split)
  float* part;             // with ksplit > 1: fp32 parts [ksplit][out_rows][n_out]
  unsigned int* split_count;  // with ksplit > 1: zeroed counters, one per output tile and
                              // epilogue warp, or null (a separate kernel adds the parts)
  int dense_T;             // > 0: one group of dense_T rows (E = 1, S = 0), schedule built here
  // Fused combine (down, bf16 Y rows): after all tiles and a grid-wide barrier,
  //   y[t] = sum_s Y[T*k + s*T + t] + sum_i topk_w[t][i] * Y[pos[t*k + i]]
  int fuse_combine;
  const float* topk_w;     // [T][k]
  const int32_t* pos;      // [T*k]
  uint16_t* y;             // [T][n_out] bf16
  unsigned int* grid_count;  // zero at launch; every CTA adds 1 when its tiles are done
};

struct SharedStorage {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int grid_done;    // fused combine: every CTA passed the grid-wide barrier in time
  int sched[MAX_GROUPS + 1];
  int offsets[MAX_GROUPS + 1];
  float stage_t[EPI_WARPS][16 * wm::STG_LD];   // per epilogue warp: one 16-token x 32 block
};

template <bool kGateUp, bool kPair>
constexpr size_t swap_smem_bytes() {
  return 1024 + size_t(SwapCfg<kGateUp, kPair>::STAGES) * SwapCfg<kGateUp, kPair>::STAGE_BYTES +
         sizeof(SharedStorage);
}
static_assert(swap_smem_bytes<true, false>() <= 227 * 1024, "shared memory budget");
static_assert(swap_smem_bytes<true, true>() <= 227 * 1024, "shared memory budget");
static_assert(swap_smem_bytes<false, true>() <= 227 * 1024, "shared memory budget");

// The merge of the layer's output (m.xxqk.cn Hy4-preview MoE explainer, section 2.2)
// inside the down GEMM.  Every CTA has stored its Y rows; a grid-wide barrier (one counter,
// bounded wait; the grid is at most one CTA per SM, all resident) makes all rows visible,
// then the CTAs share the tokens: 8 features per thread, the shared rows and then the k
// weighted rows added in fp32 in the same order as the separate combine kernel, rounded
// once.  Y is read through L2 (__ldcg): other SMs wrote it.
__device__ __forceinline__ void fused_combine(const SwapParams& p, int& all_done) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(p.grid_count, 1u);
    const uint64_t t0 = globaltimer_ns();
    int ok = 1;
    while (true) {
      unsigned int n;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(n) : "l"(p.grid_count) : "memory");
      if (n >= gridDim.x) break;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        report_error(p.status, kDevTimeout, kSiteGridSync);
        ok = 0;
        break;
      }
    }
    all_done = ok;
  }
  __syncthreads();
  pdl_launch_dependents();
  if (!all_done) return;
  // Only NUM_THREADS threads per SM do the merge, so each keeps many rows in flight: two
  // items (token, 8 features) at a time, and every row of a chunk of up to 4 slots is loaded
  // before the chunk's additions, which stay in the separate combine's order.
  constexpr int kChunk = 4;
  const int d = p.n_out, k = p.k, S = p.S, T = p.T;
  const size_t nslots = size_t(T) * k;
  const uint16_t* Y = static_cast<const uint16_t*>(p.out);
  const int vec = d / 8;
  const int64_t n_items = int64_t(T) * vec;
  const int64_t stride = int64_t(gridDim.x) * NUM_THREADS;
  for (int64_t item0 = int64_t(blockIdx.x) * NUM_THREADS + threadIdx.x; item0 < n_items;
       item0 += 2 * stride) {
    int t[2], c[2];
    bool live[2];
    float acc[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t item = item0 + u * stride;
      live[u] = item < n_items;
      t[u] = live[u] ? int(item / vec) : 0;
      c[u] = live[u] ? int(item - int64_t(t[u]) * vec) * 8 : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[u][j] = 0.f;
    }
    for (int s0 = 0; s0 < S; s0 += kChunk) {
      uint4 v[2][kChunk];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < kChunk; ++j)
          if (live[u] && s0 + j < S)
            v[u][j] = __ldcg(reinterpret_cast<const uint4*>(
                Y + (nslots + size_t(s0 + j) * T + t[u]) * d + c[u]));
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < kChunk; ++j)
          if (live[u] && s0 + j < S) {
            const uint32_t w4[4] = {v[u][j].x, v[u][j].y, v[u][j].z, v[u][j].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[u][2 * q] += bf16_bits_to_float(w4[q] & 0xFFFFu);
              acc[u][2 * q + 1] += bf16_bits_to_float(w4[q] >> 16);
            }
          }
    }
    for (int i0 = 0; i0 < k; i0 += kChunk) {
      int r[2][kChunk];
      float wt[2][kChunk];
      uint4 v[2][kChunk];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
          r[u][j] = -1;
          if (live[u] && i0 + j < k) {
            const int rr = p.pos[size_t(t[u]) * k + i0 + j];
            r[u][j] = (rr >= 0 && size_t(rr) < nslots) ? rr : -1;
            wt[u][j] = p.topk_w[size_t(t[u]) * k + i0 + j];
          }
        }
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < kChunk; ++j)
          if (r[u][j] >= 0)
            v[u][j] = __ldcg(reinterpret_cast<const uint4*>(Y + size_t(r[u][j]) * d + c[u]));
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int j = 0; j < kChunk; ++j)
          if (r[u][j] >= 0) {
            const uint32_t w4[4] = {v[u][j].x, v[u][j].y, v[u][j].z, v[u][j].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[u][2 * q] = fmaf(wt[u][j], bf16_bits_to_float(w4[q] & 0xFFFFu), acc[u][2 * q]);
              acc[u][2 * q + 1] =
                  fmaf(wt[u][j], bf16_bits_to_float(w4[q] >> 16), acc[u][2 * q + 1]);
            }
          }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (live[u]) {
        uint4 o;
        o.x = pack_bf16x2(acc[u][0], acc[u][1]);
        o.y = pack_bf16x2(acc[u][2], acc[u][3]);
        o.z = pack_bf16x2(acc[u][4], acc[u][5]);
        o.w = pack_bf16x2(acc[u][6], acc[u][7]);
        *reinterpret_cast<uint4*>(p.y + size_t(t[u]) * d + c[u]) = o;
      }
  }
}

// The down projection split over K (1-SM tiling).  Epilogue warp w of every K range's CTA
// stores the same share of the output tile's fp32 part (its 32-token chunks of its TMEM lane
// quarter's features in both 128-row halves) and then arrives on that share's counter; the
// warp that arrives last (the ksplit-th) adds the ranges' parts of the share in range order
// and rounds once to bf16 -- the sum a separate kernel would form, in its order.  No barrier
// is involved, so a warp that gives up on a fault leaves its share unsummed and nothing
// waiting.  The parts of other CTAs are read through L2 (__ldcg).
__device__ __forceinline__ void split_sum(const SwapParams& p, const wm::Tile& tl, int ot,
                                          int ksplit, int quarter, int sub, int lane) {
  __threadfence();   // this lane's part stores, before the warp's arrival
  __syncwarp();
  unsigned last = 0;
  if (lane == 0)
    last = atomicAdd(p.split_count + size_t(ot) * EPI_WARPS + (sub * 4 + quarter), 1u) ==
                   unsigned(ksplit - 1)
               ? 1u
               : 0u;
  if (!__shfl_sync(0xffffffffu, last, 0)) return;
  __threadfence();
  const size_t plane = size_t(p.out_rows) * p.n_out;
  // items: (row of a chunk, half, 8 features); 32 rows x 2 halves x 4 pieces per chunk
  for (int c = 32 * sub; c < tl.cnt; c += 64) {
    const int rows = min(32, tl.cnt - c);
    for (int i = lane; i < rows * 8; i += 32) {
      const int row = tl.out_row + c + (i >> 3);
      const int col = tl.f0 + ((i >> 2) & 1) * 128 + quarter * 32 + (i & 3) * 8;
      if (col >= p.n_out || row >= p.out_rows) continue;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const float* src = p.part + size_t(row) * p.n_out + col;
      for (int r = 0; r < ksplit; ++r) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(src + r * plane));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(src + r * plane + 4));
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + size_t(row) * p.n_out + col) = o;
    }
  }
}

template <bool kGateUp, bool kPair>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ SwapParams p) {
  using C = SwapCfg<kGateUp, kPair>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SharedStorage& ss = *reinterpret_cast<SharedStorage*>(smem + C::STAGES * C::STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.E + p.S;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;   // CTA rank inside the pair
  const bool leader = rank == 0;
  const int unit = kPair ? int(blockIdx.x >> 1) : int(blockIdx.x);
  const int n_units = kPair ? int(gridDim.x >> 1) : int(gridDim.x);

  // Prologue that reads no global data (overlaps the previous kernel under PDL).
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.empty[s], 1);
    }
    for (int a = 0; a < C::NUM_ACC; ++a) {
      mbar_init(&ss.tmem_full[a], 1);
      mbar_init(&ss.tmem_empty[a], C::EPI_THREADS);
    }
    mbar_init(&ss.mma_done, 1);
    ss.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tok_routed);
    tma_prefetch_desc(&p.tok_shared);
    tma_prefetch_desc(&p.w0);
    tma_prefetch_desc(&p.s0);
    if (kGateUp) {
      tma_prefetch_desc(&p.w1);
      tma_prefetch_desc(&p.s1);
    }
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&ss.tmem_base, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&ss.tmem_base, TMEM_COLS);
      tmem_relinquish();
    }
  }
  pdl_wait();   // the schedule, offsets and token operands come from earlier kernels
  // With the fused combine every CTA waits for all the others, so the next kernel may not
  // take an SM before all of them are resident: its launch is released after the barrier.
  if (kGateUp || !p.fuse_combine) pdl_launch_dependents();
  if (p.dense_T > 0) {   // one group of dense_T rows in token tiles of at most TN
    if (threadIdx.x == 0) {
      ss.sched[0] = 0;
      ss.sched[1] = (p.dense_T + C::TN - 1) / C::TN;
      ss.offsets[0] = 0;
      ss.offsets[1] = p.dense_T;
    }
  } else {
    for (int i = threadIdx.x; i <= G; i += NUM_THREADS) ss.sched[i] = p.sched[i];
    for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) ss.offsets[i] = p.offsets[i];
  }
  tc_fence_before();
  if (kPair) cluster_sync_all(); else __syncthreads();   // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = ss.tmem_base;

  const int n_wt = (p.n_out + C::FEAT - 1) / C::FEAT;
  // Split over K (down projection of the 1-SM tiling only): tile t covers output tile
  // t / ksplit and K blocks [kper * (t % ksplit), ...); each writes an fp32 part.
  const int ksplit = (!kGateUp && !kPair && p.ksplit > 1) ? p.ksplit : 1;
  const int total = ss.sched[G] * n_wt * ksplit;
  const int kblocks = p.K / BK;
  const int kper = (kblocks + ksplit - 1) / ksplit;
  volatile int* abort_flag = &ss.abort_flag;
  bool aborted = false;

  if (warp == 0) {
    // ---------------- TMA producer (each CTA of a pair loads its own halves) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      for (int t = unit; t < total && !aborted; t += n_units) {
        if (*abort_flag) { aborted = true; break; }
        const int ks = t % ksplit;
        const wm::Tile tl = wm::decode_tile<C::TN, C::FEAT, kGateUp>(
            t / ksplit, n_wt, G, ss.sched, ss.offsets, p.E, p.T, p.k, p.w_rows);
        const int kb0 = ks * kper, kb1 = min(kblocks, kb0 + kper);
        const CUtensorMap* mT = tl.shared ? &p.tok_shared : &p.tok_routed;
        const CUtensorMap* mW0 = tl.shared ? &p.s0 : &p.w0;
        const CUtensorMap* mW1 = kGateUp ? (tl.shared ? &p.s1 : &p.w1) : mW0;
        // this CTA's weight rows and token rows
        const int w0_row = tl.w_row + (kPair ? int(rank) * WM : 0);
        const int w1_row = kGateUp ? w0_row : w0_row + C::A_ROWS;   // down: the next row block
        const int t_row = tl.tok_row + (kPair ? int(rank) * (tl.n >> 1) : 0);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&ss.empty[stage], phase ^ 1)) {
            report_error(p.status, kDevTimeout, kSiteProducer);
            *abort_flag = 1;
            aborted = true;
            break;
          }
          uint8_t* dst = smem + stage * C::STAGE_BYTES;
          const int kc = kb * BK;
          if (kPair) {
            // The leader's full barrier counts the bytes of both CTAs' loads.
            const uint32_t bar = mapa_shared(smem_u32(&ss.full[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&ss.full[stage], 2 * C::STAGE_BYTES);
            tma_load_2d_pair(dst, mW0, bar, kc, w0_row);
            if (C::NUM_A == 2) tma_load_2d_pair(dst + W_BYTES, mW1, bar, kc, w1_row);
            tma_load_2d_pair(dst + C::NUM_A * W_BYTES, mT, bar, kc, t_row);
          } else {
            mbar_arrive_expect_tx(&ss.full[stage], C::STAGE_BYTES);
            tma_load_2d_nohint(dst, mW0, &ss.full[stage], kc, w0_row);
            tma_load_2d_nohint(dst + W_BYTES, mW1, &ss.full[stage], kc, w1_row);
            tma_load_2d_nohint(dst + 2 * W_BYTES, mT, &ss.full[stage], kc, t_row);
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain: loads counted on this CTA's own full barriers must land before it
      // exits (in the normal path the MMA consumed them all).
      if (!kPair || leader) {
        for (int s = 0; s < C::STAGES; ++s)
          if (issued_mask & (1u << s))
            if (!mbar_wait(&ss.full[s], (issued_parity >> s) & 1u, kDrainTimeoutNs))
              report_error(p.status, kDevTimeout, kSiteDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (the pair's leader only) ----------------
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = unit; t < total && !aborted; t += n_units) {
        if (*abort_flag) { aborted = true; break; }
        const int ks = t % ksplit;
        const wm::Tile tl = wm::decode_tile<C::TN, C::FEAT, kGateUp>(
            t / ksplit, n_wt, G, ss.sched, ss.offsets, p.E, p.T, p.k, p.w_rows);
        const int kb0 = ks * kper, kb1 = min(kblocks, kb0 + kper);
        const uint32_t idesc = umma_idesc_bf16_f32(C::MMA_M, tl.n);
        if (!mbar_wait(&ss.tmem_empty[acc], acc_phase ^ 1)) {
          report_error(p.status, kDevTimeout, kSiteMma);
          *abort_flag = 1;
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + uint32_t(acc * C::ACC_STRIDE);
        const uint32_t d1 = d0 + uint32_t(C::SECOND);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&ss.full[stage], phase)) {
            report_error(p.status, kDevTimeout, kSiteMma);
            *abort_flag = 1;
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint64_t a0 = umma_desc_sw128_kmajor(base);
          const uint64_t a1 = umma_desc_sw128_kmajor(base + W_BYTES);
          const uint64_t b = umma_desc_sw128_kmajor(base + C::NUM_A * W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t accum = (kb != kb0 || kk != 0) ? 1u : 0u;
            if (kPair) {
              umma_bf16_pair(d0, a0 + uint64_t(2 * kk), b + uint64_t(2 * kk), idesc, accum);
              if (C::NUM_A == 2)
                umma_bf16_pair(d1, a1 + uint64_t(2 * kk), b + uint64_t(2 * kk), idesc, accum);
            } else {
              umma_bf16(d0, a0 + uint64_t(2 * kk), b + uint64_t(2 * kk), idesc, accum);
              umma_bf16(d1, a1 + uint64_t(2 * kk), b + uint64_t(2 * kk), idesc, accum);
            }
          }
          if (kPair) umma_commit_pair(&ss.empty[stage], 0x3); else umma_commit(&ss.empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        if (kPair) umma_commit_pair(&ss.tmem_full[acc], 0x3); else umma_commit(&ss.tmem_full[acc]);
        if (++acc == C::NUM_ACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // Drain: wait until every MMA issued here has completed.
      if (kPair) umma_commit_pair(&ss.mma_done, 0x1); else umma_commit(&ss.mma_done);
      if (!mbar_wait(&ss.mma_done, 0, kDrainTimeoutNs))
        report_error(p.status, kDevTimeout, kSiteDrain);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9; TMEM lane = output feature) ----------------
    const int quarter = warp & 3;               // TMEM lanes [32*quarter, 32*quarter+32)
    const int sub = (warp - 2) >> 2;            // which of the quarter's two warps
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    float* stg = ss.stage_t[warp - 2];
    const int feat_cta = kPair ? int(rank) * WM : 0;   // this CTA's first feature in a tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = unit; t < total; t += n_units) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { aborted = true; break; }  // warp-uniform
      const int ks = t % ksplit;
      const wm::Tile tl = wm::decode_tile<C::TN, C::FEAT, kGateUp>(
            t / ksplit, n_wt, G, ss.sched, ss.offsets, p.E, p.T, p.k, p.w_rows);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&ss.tmem_full[acc], acc_phase));
      if (!ok) {
        if (lane == 0) report_error(p.status, kDevTimeout, kSiteEpilogue);
        *abort_flag = 1;
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + uint32_t(acc * C::ACC_STRIDE);
      // this warp's 32-token chunks: c = 32 * (2 i + sub)
      bool released = false;
      if (kGateUp && kPair) {
        // The pair's gate/up accumulator fills all 512 columns, so the next tile's
        // MMAs wait for it: read the whole tile into registers first (SwiGLU packed
        // to bf16 pairs, <= 4 chunks per warp), hand TMEM back, then store.
        const int col0 = tl.f0 + feat_cta + quarter * 32;
        const bool cols_ok = col0 < p.n_out;
        uint32_t hp[4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 32 * (2 * j + sub);
          if (c < tl.n) {
            uint32_t g[32], u[32];
            tmem_ld_32cols(tbase + uint32_t(c), g);
            tmem_ld_32cols(tbase + uint32_t(C::SECOND + c), u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              hp[j][i] = pack_bf16x2(
                  wm::swiglu(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                  wm::swiglu(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
          }
        }
        tc_fence_before();
        mbar_arrive_cluster(mapa_shared(smem_u32(&ss.tmem_empty[acc]), 0));
        released = true;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 32 * (2 * j + sub);
          if (c < tl.n && cols_ok) {
            float h[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              h[2 * i] = bf16_bits_to_float(hp[j][i] & 0xFFFFu);
              h[2 * i + 1] = bf16_bits_to_float(hp[j][i] >> 16);
            }
            wm::store_block_transposed<true>(stg, h, lane, p.out, p.n_out, tl.out_row + c,
                                         tl.cnt - c, col0, p.out_rows);
          }
        }
      } else if (kGateUp) {
        const int col0 = tl.f0 + feat_cta + quarter * 32;   // this warp's 32 features
        const bool cols_ok = col0 < p.n_out;                // n_out is a multiple of 64
        int c = 32 * sub;
        uint32_t g[32], u[32];
        if (c < tl.n) {
          tmem_ld_32cols(tbase + uint32_t(c), g);
          tmem_ld_32cols(tbase + uint32_t(C::SECOND + c), u);
        }
#pragma unroll 1
        for (; c < tl.n; c += 64) {
          tmem_ld_wait();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = wm::swiglu(__uint_as_float(g[i]), __uint_as_float(u[i]));
          if (c + 64 < tl.n) {   // next chunk's loads overlap this chunk's stores
            tmem_ld_32cols(tbase + uint32_t(c + 64), g);
            tmem_ld_32cols(tbase + uint32_t(C::SECOND + c + 64), u);
          }
          if (cols_ok)
            wm::store_block_transposed<true>(stg, h, lane, p.out, p.n_out, tl.out_row + c,
                                         tl.cnt - c, col0, p.out_rows);
        }
      } else if (kPair && ksplit == 1 && p.out_bf16) {
        // The pair's down accumulator fills all 512 columns as well: read both row blocks
        // into registers (rounded to bf16, as they are stored), hand TMEM back, then store.
        uint32_t yp[2][4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 32 * (2 * j + sub);
          if (c < tl.n) {
            uint32_t r0[32], r1[32];
            tmem_ld_32cols(tbase + uint32_t(c), r0);
            tmem_ld_32cols(tbase + uint32_t(C::SECOND + c), r1);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              yp[0][j][i] = pack_bf16x2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
              yp[1][j][i] = pack_bf16x2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
            }
          }
        }
        tc_fence_before();
        mbar_arrive_cluster(mapa_shared(smem_u32(&ss.tmem_empty[acc]), 0));
        released = true;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int col0 = tl.f0 + feat_cta + half * C::A_ROWS + quarter * 32;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = 32 * (2 * j + sub);
            if (c < tl.n && col0 < p.n_out) {
              float v[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                v[2 * i] = bf16_bits_to_float(yp[half][j][i] & 0xFFFFu);
                v[2 * i + 1] = bf16_bits_to_float(yp[half][j][i] >> 16);
              }
              wm::store_block_transposed<true>(stg, v, lane, p.out, p.n_out, tl.out_row + c,
                                           tl.cnt - c, col0, p.out_rows);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int col0 = tl.f0 + feat_cta + half * C::A_ROWS + quarter * 32;
          const bool cols_ok = col0 < p.n_out;
          const uint32_t hbase = tbase + uint32_t(half * C::SECOND);
          int c = 32 * sub;
          uint32_t r[32];
          if (c < tl.n) tmem_ld_32cols(hbase + uint32_t(c), r);
#pragma unroll 1
          for (; c < tl.n; c += 64) {
            tmem_ld_wait();
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            if (c + 64 < tl.n) tmem_ld_32cols(hbase + uint32_t(c + 64), r);
            if (cols_ok) {
              if (ksplit > 1)   // this K range's fp32 part; the parts are added afterwards
                wm::store_block_transposed<false>(
                    stg, v, lane, p.part + size_t(ks) * p.out_rows * p.n_out, p.n_out,
                    tl.out_row + c, tl.cnt - c, col0, p.out_rows);
              else if (p.out_bf16)
                wm::store_block_transposed<true>(stg, v, lane, p.out, p.n_out, tl.out_row + c,
                                             tl.cnt - c, col0, p.out_rows);
              else
                wm::store_block_transposed<false>(stg, v, lane, p.out, p.n_out, tl.out_row + c,
                                              tl.cnt - c, col0, p.out_rows);
            }
          }
        }
      }
      if (!released) {
        tc_fence_before();
        if (kPair)
          mbar_arrive_cluster(mapa_shared(smem_u32(&ss.tmem_empty[acc]), 0));
        else
          mbar_arrive(&ss.tmem_empty[acc]);
      }
      if (!kPair && ksplit > 1 && p.split_count)
        split_sum(p, tl, t / ksplit, ksplit, quarter, sub, lane);
      if (++acc == C::NUM_ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  if (kPair && aborted) {
    // A CTA of a pair cannot observe its own loads' completion (they are
    // counted on the leader's barrier): give copies in flight time to land.
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_all(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem_base, TMEM_COLS); else tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (!kGateUp && p.fuse_combine) fused_combine(p, ss.grid_done);
}

template <bool kGateUp, bool kPair>
cudaError_t launch_swap(const SwapParams& sp, int num_sms, cudaStream_t st) {
  static thread_local int attrs_device = -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (attrs_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<kGateUp, kPair>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(swap_smem_bytes<kGateUp, kPair>()));
    if (e != cudaSuccess) return e;
    attrs_device = dev;
  }
  const unsigned grid = kPair ? unsigned(num_sms & ~1) : unsigned(num_sms);
  return launch_pdl(grouped_gemm_swap_kernel<kGateUp, kPair>, dim3(grid), dim3(NUM_THREADS),
                    swap_smem_bytes<kGateUp, kPair>(), st, kPair ? 2 : 1, sp);
}

}  // namespace

// Whether every CTA of the weight-major down GEMM's grid can be resident at once on the
// current device (one CTA per SM by its shared memory; for the pair, as many 2-CTA clusters
// as the grid has), which the fused combine's grid-wide barrier needs.
bool swap_down_all_resident(bool pair) {
  static thread_local int cached_dev = -1, cached[2] = {-1, -1};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cached_dev != dev) {
    cached[0] = cached[1] = -1;
    cached_dev = dev;
  }
  if (cached[pair] < 0) {
    int sms = 0;
    bool ok = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
    const unsigned grid = pair ? unsigned(sms & ~1) : unsigned(sms);
    const size_t smem = pair ? swap_smem_bytes<false, true>() : swap_smem_bytes<false, false>();
    if (ok && pair) {
      ok = cudaFuncSetAttribute(grouped_gemm_swap_kernel<false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) ==
           cudaSuccess;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(grid);
      cfg.blockDim = dim3(NUM_THREADS);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      ok = ok && cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_swap_kernel<false, true>,
                                                &cfg) == cudaSuccess;
      ok = ok && unsigned(clusters) * 2u >= grid;
    } else if (ok) {
      ok = cudaFuncSetAttribute(grouped_gemm_swap_kernel<false, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) ==
           cudaSuccess;
      int per_sm = 0;
      ok = ok && cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                     &per_sm, grouped_gemm_swap_kernel<false, false>, NUM_THREADS, smem) ==
                     cudaSuccess;
      ok = ok && unsigned(per_sm) * unsigned(sms) >= grid;
    }
    if (!ok) cudaGetLastError();
    cached[pair] = ok ? 1 : 0;
  }
  return cached[pair] == 1;
}

moe_status launch_expert_ffn_swap(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                                  bool pair, cudaStream_t st) {
  const int T = a.T;
  const uint64_t nslots = uint64_t(T) * c.k;
  const uint64_t rows = nslots + uint64_t(c.S) * T;
  // schedules of 128-token tiles at sched[0..G], of 256-token tiles at sched[G+1..2G+1]
  const int32_t* sched = a.sched + (pair ? (c.E + c.S + 1) : 0);

  // ---- gate/up + SwiGLU ----
  SwapParams gp;
  memset(&gp, 0, sizeof gp);
  bool ok = encode_bf16_2d(&gp.tok_routed, a.x_perm, nslots, c.d, B_BOX) &&
            encode_bf16_2d(&gp.tok_shared, a.x, uint64_t(T), c.d, B_BOX) &&
            encode_bf16_2d(&gp.w0, a.Wg, uint64_t(c.E) * c.F, c.d, WM) &&
            encode_bf16_2d(&gp.w1, a.Wu, uint64_t(c.E) * c.F, c.d, WM);
  if (c.S > 0)
    ok = ok && encode_bf16_2d(&gp.s0, a.Sg, uint64_t(c.S) * c.F, c.d, WM) &&
         encode_bf16_2d(&gp.s1, a.Su, uint64_t(c.S) * c.F, c.d, WM);
  else {
    gp.s0 = gp.w0;
    gp.s1 = gp.w1;
  }
  if (!ok) return MOE_ERR_CUDA;
  gp.offsets = a.offsets;
  gp.sched = sched;
  gp.dense_T = a.dense_T;
  gp.out = a.h_act;
  gp.status = a.status;
  gp.T = T;
  gp.E = c.E;
  gp.S = c.S;
  gp.k = c.k;
  gp.K = c.d;
  gp.n_out = c.F;
  gp.w_rows = c.F;
  gp.out_rows = int(rows);
  cudaError_t err = pair ? launch_swap<true, true>(gp, dev.num_sms, st)
                         : launch_swap<true, false>(gp, dev.num_sms, st);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (a.after_gate_up && cudaEventRecord(a.after_gate_up, st) != cudaSuccess) return MOE_ERR_CUDA;

  // ---- down projection ----
  SwapParams dp;
  memset(&dp, 0, sizeof dp);
  ok = encode_bf16_2d(&dp.tok_routed, a.h_act, rows, c.F, B_BOX) &&
       encode_bf16_2d(&dp.w0, a.Wd, uint64_t(c.E) * c.d, c.F, WM);
  if (c.S > 0)
    ok = ok && encode_bf16_2d(&dp.s0, a.Sd, uint64_t(c.S) * c.d, c.F, WM);
  else
    dp.s0 = dp.w0;
  if (!ok) return MOE_ERR_CUDA;
  dp.tok_shared = dp.tok_routed;
  dp.w1 = dp.w0;
  dp.s1 = dp.s0;
  dp.offsets = a.offsets;
  dp.sched = sched;
  dp.dense_T = a.dense_T;
  dp.out = a.Y;
  dp.out_bf16 = a.y_bf16 ? 1 : 0;
  dp.status = a.status;
  dp.T = T;
  dp.E = c.E;
  dp.S = c.S;
  dp.k = c.k;
  dp.K = c.F;
  dp.n_out = c.d;
  dp.w_rows = c.d;
  dp.out_rows = int(rows);
  const bool split = !pair && a.down_ksplit > 1 && a.down_part && a.y_bf16;
  dp.ksplit = split ? a.down_ksplit : 1;
  dp.part = split ? a.down_part : nullptr;
  dp.split_count = split ? a.split_count : nullptr;
  if (a.fuse_combine && a.y_bf16 && !split) {   // grid_count was zeroed with the status word
    dp.fuse_combine = 1;
    dp.topk_w = a.topk_w;
    dp.pos = a.pos;
    dp.y = a.y_out;
    dp.grid_count = a.grid_count;
  }
  err = pair ? launch_swap<false, true>(dp, dev.num_sms, st)
             : launch_swap<false, false>(dp, dev.num_sms, st);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (split && !a.split_count) {   // y = bf16(sum of the K ranges' parts, in range order)
    PartialPtrs parts = {};
    for (int j = 0; j < dp.ksplit; ++j) parts.p[j] = a.down_part + size_t(j) * rows * c.d;
    if (launch_reduce_partials(parts, dp.ksplit, size_t(rows) * c.d,
                               static_cast<uint16_t*>(a.Y), dev.num_sms, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // namespace moe
