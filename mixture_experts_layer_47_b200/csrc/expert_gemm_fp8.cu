// expert_gemm_fp8.cu -- grouped expert GEMMs with FP8 (E4M3, block-scaled) weights.
//
// The same contractions as the bf16 path (m.xxqk.cn Hy4-preview MoE explainer,
// section 2.1: each expert is an FFN sub-network; ZAKER Hy4 Preview release
// news: 256 routed experts plus one shared expert, and an FP8 checkpoint):
//   gate/up:  H_g = silu(X_g W_gate_g^T) * (X_g W_up_g^T)   -> bf16
//   down:     Y_g = H_g W_down_g^T                           -> fp32 or bf16
// with every weight stored as an E4M3 code and one power-of-two scale per 32
// consecutive K elements of a row (scales K-block-major, [n][K/32][rows]).
// Weight-only FP8: the codes are decoded to bf16 and the tensor cores run the
// bf16 MMA (kind::f16), so the activations stay bf16 and the result equals the
// bf16 path on the decoded weights (each decoded weight, e4m3 * 2^k, has at most
// 4 significant bits and is an exact bf16 value).  The point is the weight
// stream: at decode sizes the layer is bound by HBM, and FP8 halves the bytes
// per weight.
//
// Weight-major tiles (A = 128 weight rows, B = a tile of at most 32 tokens,
// rounded up to 16), two MMAs per K16 step: gate and up rows, or 256
// consecutive W_down rows.  The decoded weights never touch shared memory:
// each decoder thread owns one weight row, decodes its 64 codes of a K block
// and writes them with tcgen05.st straight into tensor memory, where the MMA
// reads its A operand (shared memory then carries only the raw codes, their
// scales and the token tile -- staging decoded tiles there made the kernel
// bound by shared-memory bandwidth).  Roles:
//   warp 0      TMA producer of a 6-stage ring: per 64-wide K block the token
//               tile (32 rows, bf16, 128-byte swizzle), the two FP8 code boxes
//               (128 rows x 64 bytes, 64-byte swizzle) and their scales;
//   warp 1      TMEM owner and MMA issuer (A from TMEM, B from shared memory);
//               the whole warp runs the loop and its waits, lane 0 issues
//               (2.4-2.9% faster per layer than issue from one lane of an
//               otherwise idle warp, with one wait per K block instead of two);
//   warps 2-9   decoders: warp w decodes buffer (w-2)/4 (gate or first W_down
//               half; up or second half) for TMEM lanes 32 (w % 4) .. +31,
//               one row per thread, into a 4-stage TMEM ring of A tiles;
//   warps 10-13 epilogue: one per TMEM lane quarter, SwiGLU (gate/up) or
//               pass-through (down), 32x32 transposes through shared memory.
// TMEM columns: [0, 128) two double-buffered accumulators of 2 x 32 columns,
// [128, 512) six A stages of 2 x 32 columns (64 bf16 K values per row each), one
// per shared-memory stage, so one MMA commit per K block frees both.
//
// 2-SM form (kPair, optional): at decode the token tile is 16 or 32 wide, so an
// M=128 MMA moves little work per instruction and the MMA issue rate, not HBM,
// bounds the 1-SM kernel.  A CTA pair halves the instructions per weight byte:
// each CTA stages and decodes its own 128 rows of each A tile (gate / up rows
// f0 + 128 r, or W_down rows f0 + 128 r and f0 + 256 + 128 r) into its own
// TMEM, stages half of the token tile, and the pair's leader issues
// tcgen05.mma.cta_group::2 (M = 256) with A from both CTAs' TMEM.  The token
// halves are counted on the leader's barrier; the decoders of both CTAs arrive
// on the leader's "A tile written" barrier; MMA completions are multicast to
// both CTAs' barriers; both CTAs' epilogues arrive on the leader's
// "accumulator free" barrier.  Measured, each 2-SM MMA of this shape costs about
// twice a 1-SM one, so the pair is not faster; it is kept selectable, not default.
// Every wait is bounded; on expiry the kernel records the fault, drains its
// own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "fp8_decode.cuh"
#include "internal.h"
#include "tensor_map.cuh"
#include "weight_major.cuh"

namespace moe {
namespace {

constexpr int BK = 64;                      // K elements per stage
constexpr int WM = 128;                     // weight rows per A tile (tcgen05 M)
constexpr int TN = 32;                      // largest token tile (tcgen05 N)
constexpr int FP8_BLOCK = 32;               // K elements per scale
constexpr int B_BYTES = TN * BK * 2;        // token tile: 4 KB
constexpr int RAW_A = WM * BK;              // one FP8 code box: 8 KB
constexpr int RAW_S = (BK / FP8_BLOCK) * WM;  // its scales: 2 x 128 bytes
constexpr int OFF_A0 = B_BYTES;             // stage layout: B | codes A0 | codes A1 | S0 | S1
constexpr int OFF_A1 = OFF_A0 + RAW_A;
constexpr int OFF_S0 = OFF_A1 + RAW_A;
constexpr int OFF_S1 = OFF_S0 + RAW_S;
constexpr int STAGE_TX = OFF_S1 + RAW_S;
constexpr int STAGE_BYTES = 21 * 1024;      // STAGE_TX rounded up to 1 KB
constexpr int STAGES = 6;
constexpr int A_STAGES = STAGES;            // TMEM A ring, in step with the shared ring
constexpr int DEC_WARPS = 8;
constexpr int NUM_THREADS = 32 * (2 + DEC_WARPS + 4);   // producer, MMA, decoders, epilogue
constexpr uint32_t ACC_COLS = 2 * TN;       // gate | up (or two W_down halves), 32 columns each
constexpr uint32_t A_COL0 = 2 * ACC_COLS;   // first A-stage column
constexpr uint32_t A_STAGE_COLS = 2 * (BK / 2);   // two A tiles, 32 columns each
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_GROUPS = 1024 + 8;
constexpr int A_TX = 2 * RAW_A + 2 * RAW_S;  // one CTA's codes and scales per stage
static_assert(STAGE_TX <= STAGE_BYTES, "stage size");
static_assert(A_COL0 + A_STAGES * A_STAGE_COLS <= TMEM_COLS, "TMEM budget");

struct __align__(64) Fp8Params {
  CUtensorMap tok_routed;  // gate/up: X_perm [T*k][d]; down: H [T*k+S*T][F] (bf16, box 32 rows)
  CUtensorMap tok_shared;  // gate/up: x [T][d];        down: same as tok_routed
  CUtensorMap w0, w1;      // routed codes: gate/up W_gate, W_up [E*F][d]; down W_down [E*d][F]
  CUtensorMap ws0, ws1;    // their scales [E*K/32][rows] (box 2 x 128)
  CUtensorMap s0, s1;      // shared-expert codes
  CUtensorMap ss0, ss1;    // shared-expert scales
  const int32_t* offsets;  // [E+1]
  void* out;               // gate/up: H bf16; down: Y fp32, or bf16 when out_bf16
  int* status;
  int out_bf16;
  int T, E, S, k;
  int K;                   // reduction length (d or F)
  int n_out;               // output features per group (F or d)
  int w_rows;              // weight rows per expert (F or d)
  int out_rows;            // rows of the output buffer (T*k + S*T)
};

struct SharedStorage {
  uint64_t full[STAGES];             // 1-SM: the whole stage; pair: this CTA's codes and scales
  uint64_t bfull[STAGES];            // pair (leader): both CTAs' token rows
  uint64_t empty[STAGES];            // every decoder warp has read its codes and scales
  uint64_t a_full[A_STAGES];         // every decoder warp has written its rows to TMEM
  uint64_t mma_free[STAGES];         // the stage's MMAs are done (token tile and A tile read)
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int sched[MAX_GROUPS + 1];         // prefix sums of ceil(rows / 32) per group
  int offsets[MAX_GROUPS + 1];
  float stage_t[4][16 * wm::STG_LD]; // per epilogue warp: one 16-token x 32 block
};

constexpr size_t fp8_smem_bytes() {
  return 1024 + size_t(STAGES) * STAGE_BYTES + sizeof(SharedStorage);
}
static_assert(fp8_smem_bytes() <= 227 * 1024, "shared memory budget");

// Prefix sums of the 32-token tile counts per group (routed groups clamped to
// [0, T] tokens, then S shared groups of T tokens), by one warp.
__device__ void build_schedule(SharedStorage& ss, int E, int S, int T, int lane) {
  const int G = E + S;
  int carry = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int n = 0;
    if (g < E) n = min(T, max(0, ss.offsets[g + 1] - ss.offsets[g]));
    else if (g < G) n = T;
    const int mt = (n + TN - 1) / TN;
    int incl = mt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (g < G) ss.sched[g] = carry + incl - mt;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) ss.sched[G] = carry;
}

template <bool kGateUp, bool kPair>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ Fp8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  SharedStorage& ss = *reinterpret_cast<SharedStorage*>(ring + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.E + p.S;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;   // CTA rank inside the pair
  const bool leader = rank == 0;
  const int unit = kPair ? int(blockIdx.x >> 1) : int(blockIdx.x);
  const int n_units = kPair ? int(gridDim.x >> 1) : int(gridDim.x);
  constexpr int kCtas = kPair ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.bfull[s], 1);
      mbar_init(&ss.empty[s], DEC_WARPS);
      mbar_init(&ss.a_full[s], kCtas * DEC_WARPS);
      mbar_init(&ss.mma_free[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ss.tmem_full[a], 1);
      mbar_init(&ss.tmem_empty[a], kCtas * 128);
    }
    mbar_init(&ss.mma_done, 1);
    ss.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tok_routed);
    tma_prefetch_desc(&p.tok_shared);
    tma_prefetch_desc(&p.w0);
    tma_prefetch_desc(&p.ws0);
    tma_prefetch_desc(&p.s0);
    tma_prefetch_desc(&p.ss0);
    if (kGateUp) {
      tma_prefetch_desc(&p.w1);
      tma_prefetch_desc(&p.ws1);
      tma_prefetch_desc(&p.s1);
      tma_prefetch_desc(&p.ss1);
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
  pdl_wait();   // the offsets and token operands come from earlier kernels
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) ss.offsets[i] = p.offsets[i];
  __syncthreads();
  if (warp == 0) build_schedule(ss, p.E, p.S, p.T, lane);
  tc_fence_before();
  if (kPair) cluster_sync_all(); else __syncthreads();   // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = ss.tmem_base;

  // Output features per weight tile: gate/up 128 per CTA, down 256 per CTA (two A tiles).
  constexpr int kFeat = (kGateUp ? WM : 2 * WM) * kCtas;
  constexpr int kHalf2 = WM * kCtas;             // down: offset of the second A tile's rows
  const int rofs = int(rank) * WM;               // this CTA's first row inside an A tile
  const int n_wt = (p.n_out + kFeat - 1) / kFeat;
  const int total = ss.sched[G] * n_wt;
  const int kblocks = p.K / BK;
  const int kscales = p.K / FP8_BLOCK;           // scale rows per expert in the scale maps
  volatile int* abort_flag = &ss.abort_flag;
  bool aborted = false;

  if (warp == 0) {
    // ------------- TMA producer: token tile, FP8 code boxes and their scales -------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      for (int t = unit; t < total && !aborted; t += n_units) {
        if (*abort_flag) { aborted = true; break; }
        const wm::Tile tl = wm::decode_tile<TN, kFeat, kGateUp>(t, n_wt, G, ss.sched, ss.offsets,
                                                                p.E, p.T, p.k, p.w_rows);
        const CUtensorMap* mT = tl.shared ? &p.tok_shared : &p.tok_routed;
        const CUtensorMap* mW0 = tl.shared ? &p.s0 : &p.w0;
        const CUtensorMap* mS0 = tl.shared ? &p.ss0 : &p.ws0;
        const CUtensorMap* mW1 = kGateUp ? (tl.shared ? &p.s1 : &p.w1) : mW0;
        const CUtensorMap* mS1 = kGateUp ? (tl.shared ? &p.ss1 : &p.ws1) : mS0;
        const int w0_row = tl.w_row + rofs;
        const int w1_row = kGateUp ? w0_row : tl.w_row + kHalf2 + rofs;   // down: second tile
        const int f0 = tl.f0 + rofs;
        const int f1 = kGateUp ? f0 : tl.f0 + kHalf2 + rofs;
        const int t_row = tl.tok_row + (kPair ? int(rank) * (tl.n >> 1) : 0);
        const int srow = tl.g_local * kscales;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&ss.empty[stage], phase ^ 1) ||
              !mbar_wait(&ss.mma_free[stage], phase ^ 1)) {
            report_error(p.status, kDevTimeout, kSiteProducer);
            *abort_flag = 1;
            aborted = true;
            break;
          }
          uint8_t* dst = ring + stage * STAGE_BYTES;
          const int kc = kb * BK;
          const int kbs = srow + kb * (BK / FP8_BLOCK);
          if (kPair) {
            // codes and scales for this CTA's decoders; the token half for the leader's MMA
            mbar_arrive_expect_tx(&ss.full[stage], A_TX);
            const uint32_t bbar = mapa_shared(smem_u32(&ss.bfull[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&ss.bfull[stage], 2 * (TN / 2) * BK * 2);
            tma_load_2d_pair(dst, mT, bbar, kc, t_row);
          } else {
            mbar_arrive_expect_tx(&ss.full[stage], STAGE_TX);
            tma_load_2d_nohint(dst, mT, &ss.full[stage], kc, t_row);
          }
          tma_load_2d_nohint(dst + OFF_A0, mW0, &ss.full[stage], kc, w0_row);
          tma_load_2d_nohint(dst + OFF_A1, mW1, &ss.full[stage], kc, w1_row);
          tma_load_2d_nohint(dst + OFF_S0, mS0, &ss.full[stage], f0, kbs);
          tma_load_2d_nohint(dst + OFF_S1, mS1, &ss.full[stage], f1, kbs);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain: this CTA's own loads must land before it exits (the leader also sees the
      // token halves on its barrier; the other CTA waits out its halves at the end).
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) {
          if (!mbar_wait(&ss.full[s], (issued_parity >> s) & 1u, kDrainTimeoutNs))
            report_error(p.status, kDevTimeout, kSiteDrain);
          if (kPair && leader &&
              !mbar_wait(&ss.bfull[s], (issued_parity >> s) & 1u, kDrainTimeoutNs))
            report_error(p.status, kDevTimeout, kSiteDrain);
        }
    }
    __syncwarp();
  } else if (warp >= 2 && warp < 2 + DEC_WARPS) {
    // ---------------- decoders: one weight row per thread, into TMEM ----------------
    const int quarter = warp & 3;                // TMEM lanes [32*quarter, 32*quarter+32)
    const int buf = (warp - 2) >> 2;             // A0 (gate / first half) or A1
    const int row = quarter * 32 + lane;         // weight row inside the 128-row tile
    const int sw = (row >> 1) & 3;               // 64-byte swizzle of the code box
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = unit; t < total; t += n_units) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { aborted = true; break; }
      for (int kb = 0; kb < kblocks; ++kb) {
        bool ok = __all_sync(0xffffffffu, mbar_wait(&ss.mma_free[stage], phase ^ 1));
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&ss.full[stage], phase));
        if (!ok) {
          if (lane == 0) report_error(p.status, kDevTimeout, kSiteProducer);
          *abort_flag = 1;
          aborted = true;
          break;
        }
        const uint8_t* src = ring + stage * STAGE_BYTES;
        const uint8_t* codes = src + (buf ? OFF_A1 : OFF_A0) + row * BK;
        const uint8_t* scl = src + (buf ? OFF_S1 : OFF_S0) + row;
        uint4 q[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)     // 16-byte chunk j of the row sits at chunk j ^ sw
          q[j] = *reinterpret_cast<const uint4*>(codes + ((j ^ sw) << 4));
        const uint32_t m0 = scale_pair(scl[0]);    // K elements 0..31 of the block
        const uint32_t m1 = scale_pair(scl[WM]);   // K elements 32..63
        __syncwarp();
        if (lane == 0) mbar_arrive(&ss.empty[stage]);   // codes and scales are in registers
        uint32_t o[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t m = j < 2 ? m0 : m1;
          const uint32_t w4[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            o[8 * j + 2 * i] = decode_pair(prmt(w4[i], kSel01), m);
            o[8 * j + 2 * i + 1] = decode_pair(prmt(w4[i], kSel23), m);
          }
        }
        tmem_st_32cols(tmem_base + lane_addr + A_COL0 + uint32_t(stage) * A_STAGE_COLS +
                           uint32_t(buf) * (BK / 2),
                       o);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kPair)
            mbar_arrive_cluster(mapa_shared(smem_u32(&ss.a_full[stage]), 0));
          else
            mbar_arrive(&ss.a_full[stage]);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (aborted) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer: A from TMEM, token tile from shared memory ----------------
    // The whole warp runs the loop and its waits; lane 0 issues every MMA and commit (a
    // commit tracks the MMAs of the thread that issues it).
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = unit; t < total && !aborted; t += n_units) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { aborted = true; break; }
        const wm::Tile tl = wm::decode_tile<TN, kFeat, kGateUp>(t, n_wt, G, ss.sched, ss.offsets,
                                                                p.E, p.T, p.k, p.w_rows);
        const uint32_t idesc = umma_idesc_bf16_f32(WM * kCtas, tl.n);
        const bool e_ok = kPair ? mbar_wait_cluster(&ss.tmem_empty[acc], acc_phase ^ 1)
                                : mbar_wait(&ss.tmem_empty[acc], acc_phase ^ 1);
        if (!__all_sync(0xffffffffu, e_ok)) {
          if (lane == 0) {
            report_error(p.status, kDevTimeout, kSiteMma);
            *abort_flag = 1;
          }
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + uint32_t(acc) * ACC_COLS;
        const uint32_t d1 = d0 + uint32_t(TN);
        for (int kb = 0; kb < kblocks; ++kb) {
          // 1-SM: the decoders arrive on a_full only after they saw the stage's full
          // barrier, which also counts the token tile, so a_full alone covers both.  The
          // pair's token halves are counted on bfull, which no decoder waits on.
          bool ok = kPair ? mbar_wait_cluster(&ss.a_full[stage], phase)
                          : mbar_wait(&ss.a_full[stage], phase);
          if (kPair) ok = ok && mbar_wait(&ss.bfull[stage], phase);
          if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
              report_error(p.status, kDevTimeout, kSiteMma);
              *abort_flag = 1;
            }
            aborted = true;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a0 = tmem_base + A_COL0 + uint32_t(stage) * A_STAGE_COLS;
            const uint32_t a1 = a0 + uint32_t(BK / 2);
            const uint64_t b = umma_desc_sw128_kmajor(smem_u32(ring + stage * STAGE_BYTES));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
              if (kPair) {
                umma_bf16_pair_tmem_a(d0, a0 + uint32_t(8 * kk), b + uint64_t(2 * kk), idesc,
                                      accum);
                umma_bf16_pair_tmem_a(d1, a1 + uint32_t(8 * kk), b + uint64_t(2 * kk), idesc,
                                      accum);
              } else {
                umma_bf16_tmem_a(d0, a0 + uint32_t(8 * kk), b + uint64_t(2 * kk), idesc, accum);
                umma_bf16_tmem_a(d1, a1 + uint32_t(8 * kk), b + uint64_t(2 * kk), idesc, accum);
              }
            }
            if (kPair) umma_commit_pair(&ss.mma_free[stage], 0x3); else umma_commit(&ss.mma_free[stage]);
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        if (lane == 0) {
          if (kPair) umma_commit_pair(&ss.tmem_full[acc], 0x3); else umma_commit(&ss.tmem_full[acc]);
        }
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (lane == 0) {
        if (kPair) umma_commit_pair(&ss.mma_done, 0x1); else umma_commit(&ss.mma_done);
        if (!mbar_wait(&ss.mma_done, 0, kDrainTimeoutNs))
          report_error(p.status, kDevTimeout, kSiteDrain);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 10..13; TMEM lane = output feature) ----------------
    const int quarter = warp & 3;               // TMEM lanes [32*quarter, 32*quarter+32)
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    float* stg = ss.stage_t[quarter];
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = unit; t < total; t += n_units) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { aborted = true; break; }  // warp-uniform
      const wm::Tile tl = wm::decode_tile<TN, kFeat, kGateUp>(t, n_wt, G, ss.sched, ss.offsets,
                                                              p.E, p.T, p.k, p.w_rows);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&ss.tmem_full[acc], acc_phase));
      if (!ok) {
        if (lane == 0) report_error(p.status, kDevTimeout, kSiteEpilogue);
        *abort_flag = 1;
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + uint32_t(acc) * ACC_COLS;
      if (kGateUp) {
        const int col0 = tl.f0 + rofs + quarter * 32;   // this warp's 32 features
        uint32_t g[32], u[32];
        tmem_ld_32cols(tbase, g);
        tmem_ld_32cols(tbase + uint32_t(TN), u);
        tmem_ld_wait();
        if (col0 < p.n_out) {                       // n_out is a multiple of 64
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = wm::swiglu(__uint_as_float(g[i]), __uint_as_float(u[i]));
          wm::store_block_transposed<true>(stg, h, lane, p.out, p.n_out, tl.out_row, tl.cnt,
                                           col0, p.out_rows);
        }
      } else {
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int col0 = tl.f0 + half * kHalf2 + rofs + quarter * 32;
          uint32_t r[32];
          tmem_ld_32cols(tbase + uint32_t(half * TN), r);
          tmem_ld_wait();
          if (col0 < p.n_out) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            if (p.out_bf16)
              wm::store_block_transposed<true>(stg, v, lane, p.out, p.n_out, tl.out_row, tl.cnt,
                                               col0, p.out_rows);
            else
              wm::store_block_transposed<false>(stg, v, lane, p.out, p.n_out, tl.out_row, tl.cnt,
                                                col0, p.out_rows);
          }
        }
      }
      tc_fence_before();
      if (kPair)
        mbar_arrive_cluster(mapa_shared(smem_u32(&ss.tmem_empty[acc]), 0));
      else
        mbar_arrive(&ss.tmem_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  if (kPair && aborted) {
    // The token halves of the non-leader CTA are counted on the leader's barrier,
    // so it cannot observe their completion: give copies in flight time to land.
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
}

template <bool kGateUp, bool kPair>
cudaError_t launch_fp8(const Fp8Params& fp, int num_sms, cudaStream_t st) {
  static thread_local int attrs_device = -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (attrs_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_fp8_kernel<kGateUp, kPair>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(fp8_smem_bytes()));
    if (e != cudaSuccess) return e;
    attrs_device = dev;
  }
  const unsigned grid = kPair ? unsigned(num_sms & ~1) : unsigned(num_sms);
  return launch_pdl(grouped_gemm_fp8_kernel<kGateUp, kPair>, dim3(grid), dim3(NUM_THREADS),
                    fp8_smem_bytes(), st, kPair ? 2 : 1, fp);
}

// Codes [n*rows][K] (box 128 rows x 64 bytes, 64-byte swizzle) and scales
// [n*K/32][rows] (box 2 x 128, unswizzled).
bool encode_set(CUtensorMap* codes, CUtensorMap* scales, const uint8_t* c, const uint8_t* s,
                int n, int rows, int K) {
  return encode_u8_2d(codes, c, uint64_t(n) * rows, uint64_t(K), WM, BK,
                      CU_TENSOR_MAP_SWIZZLE_64B) &&
         encode_u8_2d(scales, s, uint64_t(n) * (K / FP8_BLOCK), uint64_t(rows),
                      BK / FP8_BLOCK, WM);
}

}  // namespace

moe_status launch_expert_ffn_fp8(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                                 cudaStream_t st) {
  // Decode-size batches go to the warp-MMA form (expert_gemv_fp8.cu): this kernel's MMAs over
  // 16-32 token tiles cost about as much as the bf16 weights' HBM time, twice the FP8 codes'.
  if (a.T <= kGemvMaxT && c.tiles == TilesMode::kAuto) return launch_expert_ffn_gemv_fp8(c, a, dev, st);
  if (!tensor_map_encoder()) return MOE_ERR_CUDA;
  const moe_fp8_expert_weights& R = *a.fp8_routed;
  const moe_fp8_expert_weights* Sh = a.fp8_shared;
  const int T = a.T;
  const uint64_t nslots = uint64_t(T) * c.k;
  const uint64_t rows = nslots + uint64_t(c.S) * T;
  // The 1-SM form unless the 2-SM weight-major tiling is asked for (MOE_GEMM_TILES=swap_pair):
  // measured on B200 at decode, a cta_group::2 MMA with A in TMEM and N = 16 costs about
  // twice a 1-SM one, so the pair takes twice as long (2.0 against 1.03 ms per layer).
  const bool pair = c.tiles == TilesMode::kSwapPair;
  const int tok_box = pair ? TN / 2 : TN;   // token rows one CTA stages per K block

  // ---- gate/up + SwiGLU ----
  Fp8Params gp;
  memset(&gp, 0, sizeof gp);
  bool ok = encode_bf16_2d(&gp.tok_routed, a.x_perm, nslots, c.d, tok_box) &&
            encode_bf16_2d(&gp.tok_shared, a.x, uint64_t(T), c.d, tok_box) &&
            encode_set(&gp.w0, &gp.ws0, R.gate, R.gate_scale, c.E, c.F, c.d) &&
            encode_set(&gp.w1, &gp.ws1, R.up, R.up_scale, c.E, c.F, c.d);
  if (c.S > 0)
    ok = ok && encode_set(&gp.s0, &gp.ss0, Sh->gate, Sh->gate_scale, c.S, c.F, c.d) &&
         encode_set(&gp.s1, &gp.ss1, Sh->up, Sh->up_scale, c.S, c.F, c.d);
  else {
    gp.s0 = gp.w0;
    gp.ss0 = gp.ws0;
    gp.s1 = gp.w1;
    gp.ss1 = gp.ws1;
  }
  if (!ok) return MOE_ERR_CUDA;
  gp.offsets = a.offsets;
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
  if ((pair ? launch_fp8<true, true>(gp, dev.num_sms, st)
            : launch_fp8<true, false>(gp, dev.num_sms, st)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (a.after_gate_up && cudaEventRecord(a.after_gate_up, st) != cudaSuccess) return MOE_ERR_CUDA;

  // ---- down projection ----
  Fp8Params dp;
  memset(&dp, 0, sizeof dp);
  ok = encode_bf16_2d(&dp.tok_routed, a.h_act, rows, c.F, tok_box) &&
       encode_set(&dp.w0, &dp.ws0, R.down, R.down_scale, c.E, c.d, c.F);
  if (c.S > 0)
    ok = ok && encode_set(&dp.s0, &dp.ss0, Sh->down, Sh->down_scale, c.S, c.d, c.F);
  else {
    dp.s0 = dp.w0;
    dp.ss0 = dp.ws0;
  }
  if (!ok) return MOE_ERR_CUDA;
  dp.tok_shared = dp.tok_routed;
  dp.w1 = dp.w0;
  dp.ws1 = dp.ws0;
  dp.s1 = dp.s0;
  dp.ss1 = dp.ss0;
  dp.offsets = a.offsets;
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
  if ((pair ? launch_fp8<false, true>(dp, dev.num_sms, st)
            : launch_fp8<false, false>(dp, dev.num_sms, st)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
