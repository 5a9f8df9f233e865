// expert_gemm.cu -- grouped bf16 expert GEMMs on the sm_100a tensor cores.
//
// The expert FFN of the layer (m.xxqk.cn Hy4-preview MoE explainer, section
// 2.1: every expert is an FFN sub-network standing in for the dense FFN; ZAKER
// Hy4 Preview release news: 256 routed experts plus one shared expert) is, per
// group g (a routed expert's token segment, or the shared expert over all T
// tokens), two dense contractions:
//   gate/up:  H_g = silu(X_g W_gate_g^T) * (X_g W_up_g^T)   -> bf16
//   down:     Y_g = H_g W_down_g^T                           -> fp32
// Both run in one persistent, warp-specialised kernel template:
//   warp 0      TMA producer: 128x64 A tiles and 256x64 B tiles (128-byte
//               swizzle) into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns, one elected lane issues
//               tcgen05.mma (M=128, N=256, K=16) into one of two fp32 TMEM
//               accumulators and commits stage releases / tile completion to
//               mbarriers;
//   warps 2-5   epilogue: tcgen05.ld the accumulator (one TMEM lane per row),
//               apply SwiGLU (gate/up) or pass fp32 through (down), store.
// The gate/up B tile stacks 128 gate rows over the matching 128 up rows, so
// one 256-wide accumulator holds both halves of 128 output features and the
// SwiGLU product is formed in the epilogue without a second pass.
// Tiles are enumerated group by group, N-tile-major inside a group, so CTAs
// running at the same time share a weight tile through L2.  Every wait is
// bounded; on expiry the kernel records the fault in the status word, drains
// its own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tensor_map.cuh"

namespace moe {
namespace {

constexpr int BK = 64;
constexpr int BN = 256;                // MMA N: output features of a tile (gate|up halves or down)
constexpr int A_TILE_BYTES = 128 * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr int ACC_COLS = BN;           // fp32 TMEM columns per accumulator
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int MAX_GROUPS = 1024 + 8;   // E + S upper bound

// kPair = false: one CTA computes a 128 x 256 tile (tcgen05 M=128), loading all 256 B rows.
// kPair = true:  a cluster of two CTAs computes a 256 x 256 tile with the 2-SM MMA
//                (M=256); each CTA loads its own 128 A rows and 128 of the 256 B rows,
//                so each weight byte read from HBM feeds 256 token rows.
template <bool kPair>
struct Cfg {
  static constexpr int TILE_M = kPair ? 256 : 128;
  static constexpr int B_ROWS = kPair ? 128 : 256;  // B rows held by one CTA
  static constexpr int B_TILE_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_TILE_BYTES + B_TILE_BYTES;
  static constexpr int STAGES = kPair ? 6 : 4;
  static constexpr uint32_t IDESC = umma_idesc_bf16_f32(TILE_M, BN);
};

struct __align__(64) GemmParams {
  CUtensorMap a_routed;  // gate/up: X_perm [T*k][d]; down: H [T*k+S*T][F]
  CUtensorMap a_shared;  // gate/up: x [T][d];        down: same as a_routed
  CUtensorMap b0;        // gate/up: W_gate [E*F][d]; down: W_down [E*d][F]
  CUtensorMap b1;        // gate/up: W_up   [E*F][d]; down: unused
  CUtensorMap s0;        // shared counterparts of b0 / b1
  CUtensorMap s1;
  const int32_t* offsets;  // [E+1]
  const int32_t* sched;    // [E+S+1] prefix sums of M tiles (of TILE_M rows) per group
  void* out;               // gate/up: H bf16; down: Y fp32, or bf16 when out_bf16
  int* status;
  int out_bf16;            // down only: store Y rounded to bf16
  int T, E, S, k;
  int K;          // reduction length (d or F)
  int n_out;      // output features per group (F or d)
  int b_rows;     // weight rows per expert in the B maps (F or d)
  int out_rows;   // rows of the output buffer (T*k + S*T)
};

struct SharedStorage {
  uint64_t full[6];
  uint64_t empty[6];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int sched[MAX_GROUPS + 1];
  int offsets[MAX_GROUPS + 1];
};

template <bool kPair>
constexpr size_t smem_bytes() {
  return 1024 /*alignment slack*/ + size_t(Cfg<kPair>::STAGES) * Cfg<kPair>::STAGE_BYTES +
         sizeof(SharedStorage);
}

struct Tile {
  int g, m_idx, n_idx;
  int rows;      // valid rows of group g
  int a_row;     // first A row of this tile (pair: of the pair's 256 rows)
  int out_row;   // first output row of this tile
  int b_row;     // first weight row (in the per-group B maps) of this tile
  bool shared;
};

template <bool kGateUp, bool kPair>
__device__ __forceinline__ Tile decode_tile(int t, int n_tiles, int G, const SharedStorage& ss,
                                            const GemmParams& p) {
  constexpr int TM = Cfg<kPair>::TILE_M;
  const int q = t / n_tiles;
  int lo = 0, hi = G;  // largest g in [0, G) with sched[g] <= q
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ss.sched[mid] <= q) lo = mid; else hi = mid;
  }
  Tile tl;
  tl.g = lo;
  const int mt = ss.sched[lo + 1] - ss.sched[lo];
  const int local = t - ss.sched[lo] * n_tiles;
  tl.n_idx = local / mt;
  tl.m_idx = local - tl.n_idx * mt;
  const int nslots = p.T * p.k;
  constexpr int kOutCols = kGateUp ? BN / 2 : BN;
  if (lo < p.E) {
    tl.shared = false;
    tl.rows = ss.offsets[lo + 1] - ss.offsets[lo];
    tl.a_row = ss.offsets[lo] + tl.m_idx * TM;
    tl.out_row = tl.a_row;
    tl.b_row = lo * p.b_rows + tl.n_idx * kOutCols;
  } else {
    const int s = lo - p.E;
    tl.shared = true;
    tl.rows = p.T;
    tl.out_row = nslots + s * p.T + tl.m_idx * TM;
    tl.a_row = kGateUp ? tl.m_idx * TM : tl.out_row;
    tl.b_row = s * p.b_rows + tl.n_idx * kOutCols;
  }
  return tl;
}

template <bool kGateUp, bool kPair>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<kPair>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * A_TILE_BYTES;
  SharedStorage& ss = *reinterpret_cast<SharedStorage*>(smem + C::STAGES * C::STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.E + p.S;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;   // CTA rank inside the pair
  const bool leader = rank == 0;
  const int unit = kPair ? int(blockIdx.x >> 1) : int(blockIdx.x);        // this pair / CTA
  const int n_units = kPair ? int(gridDim.x >> 1) : int(gridDim.x);

  // Prologue that reads no global data (overlaps the previous kernel under PDL).
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ss.tmem_full[a], 1);
      mbar_init(&ss.tmem_empty[a], kPair ? 256 : 128);
    }
    mbar_init(&ss.mma_done, 1);
    ss.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a_routed);
    tma_prefetch_desc(&p.a_shared);
    tma_prefetch_desc(&p.b0);
    tma_prefetch_desc(&p.s0);
    if (kGateUp) {
      tma_prefetch_desc(&p.b1);
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
  pdl_wait();   // the schedule, offsets and A operands come from earlier kernels
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= G; i += NUM_THREADS) ss.sched[i] = p.sched[i];
  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) ss.offsets[i] = p.offsets[i];
  tc_fence_before();
  if (kPair) cluster_sync_all(); else __syncthreads();   // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = ss.tmem_base;

  constexpr int kOutCols = kGateUp ? BN / 2 : BN;
  const int n_tiles = (p.n_out + kOutCols - 1) / kOutCols;
  const int total = ss.sched[G] * n_tiles;
  const int kblocks = p.K / BK;
  volatile int* abort_flag = &ss.abort_flag;
  bool aborted = false;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs of a pair load their own halves) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      for (int t = unit; t < total && !aborted; t += n_units) {
        if (*abort_flag) { aborted = true; break; }
        const Tile tl = decode_tile<kGateUp, kPair>(t, n_tiles, G, ss, p);
        const CUtensorMap* mA = tl.shared ? &p.a_shared : &p.a_routed;
        const CUtensorMap* mB0 = tl.shared ? &p.s0 : &p.b0;
        const CUtensorMap* mB1 = tl.shared ? &p.s1 : &p.b1;
        const int a_row = tl.a_row + int(rank) * 128;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&ss.empty[stage], phase ^ 1)) {
            report_error(p.status, kDevTimeout, kSiteProducer);
            *abort_flag = 1;
            aborted = true;
            break;
          }
          uint8_t* dA = sA + stage * A_TILE_BYTES;
          uint8_t* dB = sB + stage * C::B_TILE_BYTES;
          const int kc = kb * BK;
          if (kPair) {
            // The leader's full barrier counts the bytes of both CTAs' loads.
            const uint32_t bar = mapa_shared(smem_u32(&ss.full[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&ss.full[stage], 2 * C::STAGE_BYTES);
            tma_load_2d_pair(dA, mA, bar, kc, a_row);
            if (kGateUp)   // CTA 0 holds the gate rows, CTA 1 the matching up rows
              tma_load_2d_pair(dB, rank == 0 ? mB0 : mB1, bar, kc, tl.b_row);
            else           // CTA r holds W_down rows [b_row + 128 r, b_row + 128 r + 128)
              tma_load_2d_pair(dB, mB0, bar, kc, tl.b_row + int(rank) * 128);
          } else {
            mbar_arrive_expect_tx(&ss.full[stage], C::STAGE_BYTES);
            tma_load_2d_nohint(dA, mA, &ss.full[stage], kc, a_row);
            if (kGateUp) {
              tma_load_2d_nohint(dB, mB0, &ss.full[stage], kc, tl.b_row);
              tma_load_2d_nohint(dB + C::B_TILE_BYTES / 2, mB1, &ss.full[stage], kc, tl.b_row);
            } else {
              tma_load_2d_nohint(dB, mB0, &ss.full[stage], kc, tl.b_row);
            }
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain: loads counted on this CTA's own full barriers must have landed
      // before the CTA may exit (in the normal path the MMA consumed them all).
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
        if (!mbar_wait(&ss.tmem_empty[acc], acc_phase ^ 1)) {
          report_error(p.status, kDevTimeout, kSiteMma);
          *abort_flag = 1;
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * ACC_COLS);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&ss.full[stage], phase)) {
            report_error(p.status, kDevTimeout, kSiteMma);
            *abort_flag = 1;
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint64_t a_desc = umma_desc_sw128_kmajor(smem_u32(sA + stage * A_TILE_BYTES));
          const uint64_t b_desc = umma_desc_sw128_kmajor(smem_u32(sB + stage * C::B_TILE_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if (kPair)
              umma_bf16_pair(d_tmem, a_desc + uint64_t(2 * kk), b_desc + uint64_t(2 * kk),
                             C::IDESC, (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16(d_tmem, a_desc + uint64_t(2 * kk), b_desc + uint64_t(2 * kk), C::IDESC,
                        (kb | kk) != 0 ? 1u : 0u);
          }
          if (kPair) umma_commit_pair(&ss.empty[stage], 0x3); else umma_commit(&ss.empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        if (kPair) umma_commit_pair(&ss.tmem_full[acc], 0x3); else umma_commit(&ss.tmem_full[acc]);
        if (++acc == 2) {
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
    // ---------------- epilogue (warps 2..5, one accumulator row per thread) --------
    const int quarter = warp & 3;               // TMEM lanes [32*quarter, 32*quarter+32)
    const int row_in_cta = quarter * 32 + lane;
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = unit; t < total; t += n_units) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) { aborted = true; break; }  // warp-uniform
      const Tile tl = decode_tile<kGateUp, kPair>(t, n_tiles, G, ss, p);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&ss.tmem_full[acc], acc_phase));
      if (!ok) {
        if (lane == 0) report_error(p.status, kDevTimeout, kSiteEpilogue);
        *abort_flag = 1;
        aborted = true;
        break;
      }
      tc_fence_after();
      const int row_in_tile = int(rank) * 128 + row_in_cta;
      const int r = tl.m_idx * C::TILE_M + row_in_tile;
      const int out_row = tl.out_row + row_in_tile;
      const bool valid = r < tl.rows && out_row >= 0 && out_row < p.out_rows;
      const uint32_t tbase = tmem_base + lane_addr + uint32_t(acc * ACC_COLS);
      if (kGateUp) {
        uint16_t* H = reinterpret_cast<uint16_t*>(p.out);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32cols(tbase + uint32_t(c), g);
          tmem_ld_32cols(tbase + uint32_t(BN / 2 + c), u);
          tmem_ld_wait();
          const int col0 = tl.n_idx * (BN / 2) + c;
          if (valid && col0 < p.n_out) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(g[2 * j]), g1 = __uint_as_float(g[2 * j + 1]);
              const float u0 = __uint_as_float(u[2 * j]), u1 = __uint_as_float(u[2 * j + 1]);
              const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
              const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
              packed[j] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(H + size_t(out_row) * p.n_out + col0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                  packed[4 * v + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld_32cols(tbase + uint32_t(c), v);
          tmem_ld_wait();
          const int col0 = tl.n_idx * BN + c;
          if (valid && col0 < p.n_out) {
            if (p.out_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) +
                                                    size_t(out_row) * p.n_out + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(
                    pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                    pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                    pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                    pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
            } else {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) +
                                                      size_t(out_row) * p.n_out + col0);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] =
                    make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
            }
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
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches.
// ---------------------------------------------------------------------------
bool encode_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, int box_rows) {
  return encode_bf16_2d(map, base, rows, cols, box_rows);
}

template <bool kGateUp, bool kPair>
cudaError_t set_attrs() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<kGateUp, kPair>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(smem_bytes<kPair>()));
}

template <bool kGateUp, bool kPair>
cudaError_t launch_gemm(const GemmParams& gp, int num_sms, cudaStream_t st) {
  const unsigned grid = kPair ? unsigned(num_sms & ~1) : unsigned(num_sms);
  return launch_pdl(grouped_gemm_kernel<kGateUp, kPair>, dim3(grid), dim3(NUM_THREADS),
                    smem_bytes<kPair>(), st, kPair ? 2 : 1, gp);
}

}  // namespace

// Tile choice.  The row-tiled kernels here pay ceil(c / M) M-tiles for a group
// of c rows (M = 128, or 256 for 2-SM pairs).  The weight-major kernels
// (expert_gemm_swap.cu) put the weights on the MMA's M side and pad each token
// tile only to a multiple of 16; measured on B200 at d = 6144, d_ff = 2048,
// 256 experts top-8, they are faster at every batch: the 1-SM form while
// groups average fewer than 96 rows, the 2-SM form (half the shared-memory
// traffic per MMA cycle, token tiles up to 256) from there on.
// The context's tiling mode (MOE_GEMM_TILES=single|pair|swap|swap_pair at
// moe_create) overrides the choice (all compute the same result; for tuning
// and tests).
GemmTiling gemm_tiling(const Ctx& c, int T) {
  switch (c.tiles) {
    case TilesMode::kPair: return GemmTiling::kPair;
    case TilesMode::kSingle: return GemmTiling::kSingle;
    case TilesMode::kSwap: return GemmTiling::kSwap;
    case TilesMode::kSwapPair: return GemmTiling::kSwapPair;
    case TilesMode::kAuto: break;
  }
  // the average load of a routed expert: the layer's T*k slots over all its experts
  return int64_t(T) * c.k >= int64_t(kSwapPairMinRowsPerExpert) * c.e_all()
             ? GemmTiling::kSwapPair
             : GemmTiling::kSwap;
}

// The dense layer (E = 1, k = 1, S = 0) at up to 128 tokens runs the 1-SM weight-major
// GEMMs, whose down projection has d / 256 output tiles (24 at d = 6144) for the SMs'
// 148: split its K so that about 148 CTAs stream the weights (planned for a 148-SM part,
// so the summation order is the same on every device).
int dense_down_ksplit(const Ctx& c, int T) {
  if (c.E != 1 || c.k != 1 || c.S != 0 || T < 1 || T > kDenseSplitMaxT) return 1;
  if (gemm_tiling(c, T) != GemmTiling::kSwap) return 1;
  const int tiles = (c.d + 255) / 256;
  int ks = 148 / tiles;
  ks = ks < 1 ? 1 : (ks > kDenseSplitMax ? kDenseSplitMax : ks);
  const int kblocks = c.F / 64;
  if (ks > kblocks) ks = kblocks;
  // every range non-empty: ranges are ceil(kblocks / ks) blocks long, the last the rest
  while (ks > 1 && (ks - 1) * ((kblocks + ks - 1) / ks) >= kblocks) --ks;
  return ks;
}

moe_status launch_expert_ffn(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                             cudaStream_t st) {
  if (!tensor_map_encoder()) return MOE_ERR_CUDA;
  static thread_local int attrs_device = -1;
  if (attrs_device != dev.device) {
    if (set_attrs<true, false>() != cudaSuccess || set_attrs<false, false>() != cudaSuccess ||
        set_attrs<true, true>() != cudaSuccess || set_attrs<false, true>() != cudaSuccess)
      return MOE_ERR_CUDA;
    attrs_device = dev.device;
  }
  if (a.fp8_routed) return launch_expert_ffn_fp8(c, a, dev, st);
  const int T = a.T;
  const GemmTiling tiling = gemm_tiling(c, T);
  if (tiling == GemmTiling::kSwap || tiling == GemmTiling::kSwapPair)
    return launch_expert_ffn_swap(c, a, dev, tiling == GemmTiling::kSwapPair, st);
  const bool pair = tiling == GemmTiling::kPair;
  const int b_box = pair ? 128 : 256;   // B rows one CTA loads per stage (down GEMM)
  const uint64_t nslots = uint64_t(T) * c.k;
  const uint64_t rows = nslots + uint64_t(c.S) * T;
  // schedules of 128-row tiles at sched[0..G], of 256-row tiles at sched[G+1..2G+1]
  const int32_t* sched = a.sched + (pair ? (c.E + c.S + 1) : 0);

  // ---- gate/up + SwiGLU ----
  GemmParams gp;
  memset(&gp, 0, sizeof gp);
  bool ok = encode_2d(&gp.a_routed, a.x_perm, nslots, c.d, 128) &&
            encode_2d(&gp.a_shared, a.x, uint64_t(T), c.d, 128) &&
            encode_2d(&gp.b0, a.Wg, uint64_t(c.E) * c.F, c.d, BN / 2) &&
            encode_2d(&gp.b1, a.Wu, uint64_t(c.E) * c.F, c.d, BN / 2);
  if (c.S > 0)
    ok = ok && encode_2d(&gp.s0, a.Sg, uint64_t(c.S) * c.F, c.d, BN / 2) &&
         encode_2d(&gp.s1, a.Su, uint64_t(c.S) * c.F, c.d, BN / 2);
  else {
    gp.s0 = gp.b0;
    gp.s1 = gp.b1;
  }
  if (!ok) return MOE_ERR_CUDA;
  gp.offsets = a.offsets;
  gp.sched = sched;
  gp.out = a.h_act;
  gp.status = a.status;
  gp.T = T;
  gp.E = c.E;
  gp.S = c.S;
  gp.k = c.k;
  gp.K = c.d;
  gp.n_out = c.F;
  gp.b_rows = c.F;
  gp.out_rows = int(rows);
  cudaError_t err = pair ? launch_gemm<true, true>(gp, dev.num_sms, st)
                         : launch_gemm<true, false>(gp, dev.num_sms, st);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (a.after_gate_up && cudaEventRecord(a.after_gate_up, st) != cudaSuccess) return MOE_ERR_CUDA;

  // ---- down projection ----
  GemmParams dp;
  memset(&dp, 0, sizeof dp);
  ok = encode_2d(&dp.a_routed, a.h_act, rows, c.F, 128) &&
       encode_2d(&dp.b0, a.Wd, uint64_t(c.E) * c.d, c.F, b_box);
  if (c.S > 0)
    ok = ok && encode_2d(&dp.s0, a.Sd, uint64_t(c.S) * c.d, c.F, b_box);
  else
    dp.s0 = dp.b0;
  if (!ok) return MOE_ERR_CUDA;
  dp.a_shared = dp.a_routed;
  dp.b1 = dp.b0;
  dp.s1 = dp.s0;
  dp.offsets = a.offsets;
  dp.sched = sched;
  dp.out = a.Y;
  dp.out_bf16 = a.y_bf16 ? 1 : 0;
  dp.status = a.status;
  dp.T = T;
  dp.E = c.E;
  dp.S = c.S;
  dp.k = c.k;
  dp.K = c.F;
  dp.n_out = c.d;
  dp.b_rows = c.d;
  dp.out_rows = int(rows);
  err = pair ? launch_gemm<false, true>(dp, dev.num_sms, st)
             : launch_gemm<false, false>(dp, dev.num_sms, st);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
