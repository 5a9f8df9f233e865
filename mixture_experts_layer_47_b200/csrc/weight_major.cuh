// weight_major.cuh -- tile enumeration and epilogue stores shared by the
// weight-major grouped GEMMs (expert_gemm_swap.cu, expert_gemm_fp8.cu).
//
// In these kernels each tcgen05.mma computes D^T = W X^T: the A operand is a
// block of weight rows (output features), the B operand a tile of one
// group's tokens, and the fp32 accumulator is feature-major (TMEM lane =
// feature, column = token).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace moe {
namespace wm {

constexpr int STG_LD = 33;   // transpose staging row stride (floats)

struct Tile {
  int w_row;     // first weight row of the tile in the weight maps (of the pair)
  int f0;        // first output feature of the tile (of the pair)
  int tok_row;   // first B row (token) in the token map
  int out_row;   // output row of the tile's first token
  int cnt;       // valid tokens in the tile (1..TN)
  int n;         // MMA N: cnt rounded up to 16
  int g_local;   // expert index inside its set (routed e, or shared s)
  bool shared;
};

// Tiles are numbered group by group; inside a group weight-tile-major with the
// group's token tiles innermost, so the CTAs that share a weight tile run at
// the same time and read it through L2.  A group of r tokens has
// mt = ceil(r / TN) token tiles (sched[g+1] - sched[g]) of ceil(r / mt) tokens
// rounded up to 16 (at most TN, since mt * TN >= r), the last one holding the
// remainder.  Gate/up token rows of the shared expert are rows of x; every
// other token row is a row of the permuted buffer (X_perm or H), where the
// shared rows follow the T*k routed slots.
template <int TN, int FEAT, bool kGateUp>
__device__ __forceinline__ Tile decode_tile(int t, int n_wt, int G, const int* sched,
                                            const int* offsets, int E, int T, int k,
                                            int w_rows) {
  const int q = t / n_wt;
  int lo = 0, hi = G;  // largest g in [0, G) with sched[g] <= q
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sched[mid] <= q) lo = mid; else hi = mid;
  }
  const int mt = sched[lo + 1] - sched[lo];
  const int local = t - sched[lo] * n_wt;
  const int w_idx = local / mt;
  const int j = local - w_idx * mt;
  const bool shared = lo >= E;
  int rows = shared ? T : offsets[lo + 1] - offsets[lo];
  rows = max(0, min(rows, mt * TN));
  const int per = (((rows + mt - 1) / mt) + 15) & ~15;
  Tile tl;
  tl.shared = shared;
  const int first = j * per;
  tl.cnt = max(0, min(per, rows - first));
  tl.n = (tl.cnt + 15) & ~15;
  if (tl.n < 16) tl.n = 16;
  tl.f0 = w_idx * FEAT;
  const int nslots = T * k;
  if (!shared) {
    tl.g_local = lo;
    tl.w_row = lo * w_rows + tl.f0;
    tl.tok_row = offsets[lo] + first;
    tl.out_row = tl.tok_row;
  } else {
    const int s = lo - E;
    tl.g_local = s;
    tl.w_row = s * w_rows + tl.f0;
    tl.out_row = nslots + s * T + first;
    tl.tok_row = kGateUp ? first : tl.out_row;
  }
  return tl;
}

// Store a 32-feature x 32-token block held feature-major (this lane = feature,
// v[i] = token i) as 32 output rows: transpose 16 tokens at a time through the
// warp's staging block (16 x STG_LD floats), then each instruction writes whole
// 16-byte pieces of consecutive rows.
template <bool kBf16>
__device__ __forceinline__ void store_block_transposed(float* stg, const float (&v)[32], int lane,
                                                       void* out, int n_out, int row0, int ntok,
                                                       int col0, int out_rows) {
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
#pragma unroll
    for (int i = 0; i < 16; ++i) stg[i * STG_LD + lane] = v[16 * hb + i];
    __syncwarp();
    if (kBf16) {
      // 4 lanes per token row (64 bytes), 8 rows per instruction
      const int piece = lane & 3;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int tl = (lane >> 2) + 8 * s;
        const float* src = stg + tl * STG_LD + 8 * piece;
        const uint4 val = make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                                     pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
        const int tok = 16 * hb + tl;
        const int row = row0 + tok;
        if (tok < ntok && row >= 0 && row < out_rows)
          *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + size_t(row) * n_out +
                                    col0 + 8 * piece) = val;
      }
    } else {
      // 8 lanes per token row (128 bytes), 4 rows per instruction
      const int piece = lane & 7;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int tl = (lane >> 3) + 4 * s;
        const float* src = stg + tl * STG_LD + 4 * piece;
        const float4 val = make_float4(src[0], src[1], src[2], src[3]);
        const int tok = 16 * hb + tl;
        const int row = row0 + tok;
        if (tok < ntok && row >= 0 && row < out_rows)
          *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + size_t(row) * n_out + col0 +
                                     4 * piece) = val;
      }
    }
    __syncwarp();
  }
}

// silu(g) * u.  The exponent is clamped so that 1 + e^-g stays below 2^126,
// where the fast divide is accurate; below g = -80 silu(g) is -80 e^-80 or
// smaller, which the clamp reproduces to far under the bf16 output's precision.
__device__ __forceinline__ float swiglu(float g, float u) {
  return __fdividef(g, 1.0f + __expf(fminf(-g, 80.0f))) * u;
}

}  // namespace wm
}  // namespace moe
