// expert_gemv_fp8.cu -- the FP8-weight expert FFNs at decode batch sizes (up to 16 tokens).
//
// The contractions of the layer's experts (m.xxqk.cn Hy4-preview MoE explainer, section
// 2.1; ZAKER Hy4 Preview release news: 256 routed experts plus one shared expert):
//   gate/up:  H_g = silu(X_g W_gate_g^T) * (X_g W_up_g^T)   -> bf16
//   down:     Y_g = H_g W_down_g^T                           -> fp32 or bf16
// with every weight an E4M3 code times a power-of-two scale per 32 K elements of its row
// (scales K-block-major, [n][K/32][rows]).  At decode sizes a group holds a handful of
// tokens.  The tensor-core FP8 kernel (codes decoded into tensor memory, tcgen05 MMAs of
// M = 128, N = 16) is then bound by its MMA issue cost, not by the FP8 stream, and a
// CUDA-core dot product spends about ten instructions per weight.  Here each weight costs
// about two: the decoder's (per word of four codes, two byte planes, two PRMTs and two
// bf16x2 multiplies), with the multiply-adds done by warp-level m16n8k16 bf16 MMAs on the
// decoded registers.
//
// Work: an item is 16 feature rows of one group -- the gate and the up rows of 16 features,
// or 32 consecutive W_down rows as two 16-row tiles -- for one unit of up to 8 of the group's
// tokens (one MMA column block; a group of n tokens is ceil(n/8) units, and a second unit
// decodes the rows again, its codes then coming from L2), walked in K blocks of 64.
// A CTA takes items round robin (about 90 per CTA at Hy4 decode); their K blocks are its
// jobs, cut into equal runs for its 8 warps, so every warp has the same number of blocks
// (taking whole items per warp left a tail of up to 9%).  A warp finishes an item it ran
// whole from its registers; an item cut between warps leaves each warp's partial sums in
// shared memory, and the last of its warps to arrive (a shared-memory counter, no waiting)
// adds the parts in warp order and finishes it.
// Fragments: in an m16n8k16 MMA lane l = 4 g + t holds A rows g and g + 8 at k slots
// {2t, 2t+1, 2t+8, 2t+9} and B (token g) at the same slots.  The sum over k does not care
// which K position a slot stands for, so in K block kb, MMA s (0..3), the slots of lane t
// stand for positions kb + 16 t + 4 s .. + 3: a lane's 16 consecutive codes per row (one
// 16-byte load) and its 16 consecutive activations (32 bytes) feed all four MMAs of the
// block, and each 32-wide scale block lies inside one lane's run.
// Stream: each lane copies its rows' codes and its tokens' activations for a block with
// cp.async into a per-warp 8-stage ring in shared memory, seven blocks ahead of the block it
// computes (the ring runs on across items; the lane keeps running source pointers), so the
// loads in flight hold no registers; four lanes also copy the tiles' 16 scale bytes per
// 32-wide K block, read by all lanes after the ring wait and a warp barrier.  Measured on
// B200 at Hy4 decode: 8 warps with deep rings beat 10 x 4, 12 x 4 and 16 x 3 stages, the even
// cut of the jobs gained 7% on gate/up over whole items per warp, and units of 8 tokens (one
// column block: 3 KB stages, 8-value partial slots, so 8 stages fit beside them) took the
// layer from 0.761 to 0.749 ms against 16-token units with 5 stages.
// Arithmetic: exact bf16 weights (the decoder of the tensor-core FP8 kernel) times bf16
// activations into fp32 accumulators, as in the tensor-core path; only the order of the
// fp32 additions differs.  The epilogue applies SwiGLU (gate/up) from registers: a lane's
// gate and up accumulators hold the same (feature, token) pairs.
#include "common.cuh"
#include "fp8_decode.cuh"
#include "internal.h"
#include "weight_major.cuh"

namespace moe {
namespace {

constexpr int GV_WARPS = 8;
constexpr int GV_THREADS = 32 * GV_WARPS;
constexpr int GV_KB = 64;                        // K per block (4 MMAs)
constexpr int GV_STAGES = 8;
constexpr int GV_MAX_GROUPS = 1024 + 8;          // E + S upper bound
constexpr int GV_MAX_TOK = 16;                   // tokens per group
constexpr int GV_UNIT_TOK = 8;                   // tokens per unit: one 8-token MMA column block
// Per warp and stage: codes [tile 2][row half 2][lane 32][16 B], activations [lane 32][32 B],
// scales [tile 2][32-wide K block 2][16 B].
constexpr int GV_CODE_OFF = 0;
constexpr int GV_X_OFF = 2 * 2 * 32 * 16;
constexpr int GV_SCALE_OFF = GV_X_OFF + 32 * 32;
constexpr int GV_STAGE_BYTES = GV_SCALE_OFF + 2 * 2 * 16;
constexpr int GV_RING_BYTES = GV_WARPS * GV_STAGES * GV_STAGE_BYTES;
// After the rings: the partial sums of cut items, [warp][slot 2][value 8][lane 32].
constexpr size_t GV_SMEM = size_t(GV_RING_BYTES) + size_t(GV_WARPS) * 2 * 8 * 32 * sizeof(float);
static_assert(GV_STAGE_BYTES % 16 == 0, "stages stay 16-byte aligned");

struct GemvParams {
  const uint8_t* w[2];         // routed codes: gate/up W_gate, W_up [E][F][d]; down W_down [E][d][F]
  const uint8_t* s[2];         // their scales [E][K/32][rows]
  const uint8_t* sw[2];        // shared-expert codes
  const uint8_t* ss[2];        // shared-expert scales
  const uint16_t* tok_routed;  // gate/up: X_perm [T*k][d]; down: H [T*k+S*T][F]
  const uint16_t* tok_shared;  // gate/up: x [T][d];        down: H
  const int32_t* offsets;      // [E+1]
  void* out;                   // gate/up: H bf16 [T*k+S*T][F]; down: Y fp32 or bf16 [..][d]
  int out_bf16;
  int T, E, S, k;
  int K;                       // reduction length (d or F), a multiple of 64
  int n_out;                   // output features per group = weight rows per expert (F or d)
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// until at most GV_STAGES - 1 of this thread's copy groups are still in flight
__device__ __forceinline__ void cp_async_wait_ring() {
  asm volatile("cp.async.wait_group %0;" ::"n"(GV_STAGES - 1) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// d += A (16 x 16 bf16, row-major fragments a) * B (16 x 8 bf16, column fragments b), fp32.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One warp item: features f .. of group g (rows of tile m: gate/up -> matrix m rows f ..
// f+15, down -> W_down rows f + 16 m .. f + 16 m + 15), its tokens and where its outputs go.
struct Item {
  size_t woff;           // codes of row f in its expert set
  size_t soff;           // scale of row f, K block 0
  const uint16_t* tok;   // first token's activation row
  size_t out_row;        // first token's output row
  int f;                 // first feature
  int nt;                // tokens of this unit, 1..GV_UNIT_TOK; 0 past the last item
  bool shared;           // a shared expert's item
};

template <bool kGateUp>
__device__ __forceinline__ Item describe(const GemvParams& p, const int16_t* units, int G,
                                         int per_unit, int total, int item) {
  constexpr int FEATS = kGateUp ? 16 : 32;
  Item it;
  it.nt = 0;
  if (item >= total) return it;
  const int u = item / per_unit;
  it.f = (item - u * per_unit) * FEATS;
  int lo = 0, hi = G;                                  // units[lo] <= u < units[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (units[mid] <= u) lo = mid; else hi = mid;
  }
  const int g = lo;
  const bool shared = g >= p.E;
  const int gl = shared ? g - p.E : g;
  const int off = shared ? 0 : __ldg(p.offsets + g);
  const int n = shared ? p.T : min(p.T, __ldg(p.offsets + g + 1) - off);
  const int t0 = (u - units[g]) * GV_UNIT_TOK;           // this unit's first token of the group
  it.nt = min(GV_UNIT_TOK, n - t0);
  const size_t row0 = (shared ? size_t(p.T) * p.k + size_t(gl) * p.T : size_t(off)) + t0;
  const size_t tok_row = (shared && kGateUp) ? size_t(t0) : row0;
  it.tok = (shared && kGateUp ? p.tok_shared : p.tok_routed) + tok_row * size_t(p.K);
  it.out_row = row0;
  it.shared = shared;
  it.woff = (size_t(gl) * p.n_out + it.f) * p.K;
  it.soff = size_t(gl) * (p.K / 32) * p.n_out + it.f;
  return it;
}

// What the loop over items needs besides the parameters.  A CTA takes items blockIdx.x,
// blockIdx.x + gridDim.x, ...; their K blocks, in order, are its jobs, and warp w takes the
// jobs [jw, jw+1) with jw = w * jobs / GV_WARPS, so an item may be cut between warps.
struct Walk {
  const int16_t* units;
  int G, per_unit, total, nblk, jobs, lane;
  int j0, j1;          // this warp's jobs
  uint8_t* ring;       // this warp's GV_STAGES stages
  uint32_t ring_s;     // the same, as a shared-memory address
};

__device__ __forceinline__ int warp_first_job(int jobs, int w) { return w * jobs / GV_WARPS; }

// The warp whose jobs hold job j.
__device__ __forceinline__ int warp_of_job(int jobs, int j) {
  int w = 0;
#pragma unroll
  for (int v = 1; v < GV_WARPS; ++v)
    if (warp_first_job(jobs, v) <= j) w = v;
  return w;
}

// The copies run GV_STAGES - 1 blocks ahead of the arithmetic, across items.  The cursor
// keeps this lane's source pointers for its next job: codes of rows g and g + 8 of both
// tiles, the activations of token g, and (lanes 0-3) a scale row.
struct IssueCursor {
  const uint8_t* code[4];   // [tile m * 2 + row half h]
  const uint16_t* x;        // token g
  const uint8_t* scale;     // lane 2 m + b < 4: tile m's scales of 32-wide block 2 blk + b
  int job, blk, nt;         // nt = 0 when this warp's jobs are all issued
};

// The cursor at block blk of an item.
template <bool kGateUp>
__device__ __forceinline__ void cursor_at(const GemvParams& p, const Item& it, int blk,
                                          IssueCursor& ic, int lane) {
  ic.nt = it.nt;
  ic.blk = blk;
  if (it.nt == 0) return;
  const int g = lane >> 2, t = lane & 3;
  const int k0 = blk * GV_KB + 16 * t;
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const uint8_t* base = (it.shared ? p.sw[kGateUp ? m : 0] : p.w[kGateUp ? m : 0]) + it.woff +
                          size_t(kGateUp ? 0 : 16 * m) * p.K + k0;
#pragma unroll
    for (int h = 0; h < 2; ++h) ic.code[m * 2 + h] = base + size_t(g + 8 * h) * p.K;
  }
  ic.x = it.tok + size_t(g) * p.K + k0;
  const int m = (lane >> 1) & 1, b = lane & 1;
  ic.scale = (it.shared ? p.ss[kGateUp ? m : 0] : p.s[kGateUp ? m : 0]) + it.soff +
             (kGateUp ? 0 : 16 * m) + size_t(2 * blk + b) * p.n_out;
}

template <bool kGateUp>
__device__ __forceinline__ Item job_item(const GemvParams& p, const Walk& wk, int q) {
  return describe<kGateUp>(p, wk.units, wk.G, wk.per_unit, wk.total,
                           int(blockIdx.x) + q * int(gridDim.x));
}

// Copies of the cursor's job into a stage, then the cursor moves one job on.
template <bool kGateUp>
__device__ __forceinline__ void issue_next(const GemvParams& p, const Walk& wk, IssueCursor& ic,
                                           int slot) {
  const uint32_t stage = wk.ring_s + uint32_t(slot * GV_STAGE_BYTES);
  const int lane = wk.lane, g = lane >> 2;
  if (ic.nt > 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      cp_async16(stage + uint32_t(GV_CODE_OFF + (i * 32 + lane) * 16), ic.code[i]);
      ic.code[i] += GV_KB;
    }
    if (g < ic.nt) {
      const uint32_t dst = stage + uint32_t(GV_X_OFF + lane * 32);
      cp_async16(dst, ic.x);
      cp_async16(dst + 16, ic.x + 8);
    }
    ic.x += GV_KB;
    if (lane < 4) cp_async16(stage + uint32_t(GV_SCALE_OFF + lane * 16), ic.scale);
    ic.scale += size_t(2) * p.n_out;
    if (++ic.job == wk.j1) {
      ic.nt = 0;
    } else if (++ic.blk == wk.nblk) {
      cursor_at<kGateUp>(p, job_item<kGateUp>(p, wk, ic.job / wk.nblk), 0, ic, lane);
    }
  }
  cp_async_commit();
}

// The four MMAs of one K block.  The activation columns of tokens past the unit's end are
// never copied and hold stale values: an MMA's output column depends on its own B column only,
// and those columns are not stored.
__device__ __forceinline__ void compute_block(const uint8_t* stage, float (&acc)[2][4],
                                              int lane) {
  const int g = lane >> 2, t = lane & 3;
  uint4 code[2][2];
  uint32_t mult[2][2];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      code[m][h] = *reinterpret_cast<const uint4*>(stage + GV_CODE_OFF + ((m * 2 + h) * 32 + lane) * 16);
      // this lane's 16 positions lie in 32-wide block t / 2 of the 64
      mult[m][h] = scale_pair(stage[GV_SCALE_OFF + (m * 2 + (t >> 1)) * 16 + g + 8 * h]);
    }
  const uint4* xsrc = reinterpret_cast<const uint4*>(stage + GV_X_OFF + lane * 32);
  const uint4 xv[2] = {xsrc[0], xsrc[1]};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      // slots 2t, 2t+1 <- codes 4s, 4s+1 of the run; slots 2t+8, 2t+9 <- codes 4s+2, 4s+3
      uint32_t a[4];
      decode_word((&code[m][0].x)[s], mult[m][0], a[0], a[2]);
      decode_word((&code[m][1].x)[s], mult[m][1], a[1], a[3]);
      const uint4& xs = xv[s >> 1];
      mma_bf16_16816(acc[m], a, (s & 1) ? xs.z : xs.x, (s & 1) ? xs.w : xs.y);
    }
  }
}

// After an item's last block: accumulator element i of tile m is (row g + 8 (i / 2), token
// 2 t + i % 2 of the unit).
template <bool kGateUp>
__device__ __forceinline__ void finish_item(const GemvParams& p, const Item& it,
                                            const float (&acc)[2][4], int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tok = 2 * t + (i & 1);
    if (tok >= it.nt) continue;
    const int row = g + 8 * (i >> 1);
    const size_t o = (it.out_row + tok) * size_t(p.n_out) + it.f + row;
    if (kGateUp) {
      reinterpret_cast<uint16_t*>(p.out)[o] =
          uint16_t(pack_bf16x2(wm::swiglu(acc[0][i], acc[1][i]), 0.f) & 0xFFFFu);
    } else {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (p.out_bf16)
          reinterpret_cast<uint16_t*>(p.out)[o + 16 * m] =
              uint16_t(pack_bf16x2(acc[m][i], 0.f) & 0xFFFFu);
        else
          reinterpret_cast<float*>(p.out)[o + 16 * m] = acc[m][i];
      }
    }
  }
}

// This warp's jobs of one item, blocks [blk0, blk0 + nb); slot is the stage the first one
// reads.  A whole item is finished from the registers.  A part of a cut item goes to this
// warp's partial slot (0: the item began before this warp's jobs, 1: it runs past them);
// the last of the item's warps to arrive adds the parts in warp order and finishes it.
template <bool kGateUp>
__device__ __forceinline__ void run_segment(const GemvParams& p, const Walk& wk, const Item& it,
                                            int q, int blk0, int nb, IssueCursor& ic, int& slot,
                                            float* part, int* cut_count, int warp) {
  float acc[2][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
  for (int b = 0; b < nb; ++b) {
    // refill the stage computed last (its reads are done), GV_STAGES - 1 jobs ahead
    issue_next<kGateUp>(p, wk, ic, slot == 0 ? GV_STAGES - 1 : slot - 1);
    cp_async_wait_ring();
    __syncwarp();   // the scale bytes were copied by lanes 0-3
    compute_block(wk.ring + slot * GV_STAGE_BYTES, acc, wk.lane);
    __syncwarp();   // every lane is done with the stage before lanes 0-3 refill it
    slot = slot == GV_STAGES - 1 ? 0 : slot + 1;
  }
  if (blk0 == 0 && nb == wk.nblk) {
    finish_item<kGateUp>(p, it, acc, wk.lane);
    return;
  }
  const int lane = wk.lane;
  const int first_job = q * wk.nblk;
  float* mine = part + ((warp * 2 + (first_job < wk.j0 ? 0 : 1)) * 8) * 32;
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) mine[(4 * m + i) * 32 + lane] = acc[m][i];
  __threadfence_block();
  __syncwarp();
  // the item's parts: the warps from w_first to w_last that have jobs (with fewer jobs than
  // warps, some warps have none)
  const int w_first = warp_of_job(wk.jobs, first_job);
  const int w_last = warp_of_job(wk.jobs, first_job + wk.nblk - 1);
  int parts = 0;
  for (int w = w_first; w <= w_last; ++w)
    parts += warp_first_job(wk.jobs, w + 1) > warp_first_job(wk.jobs, w) ? 1 : 0;
  int arrived = 0;
  if (lane == 0) arrived = atomicAdd(cut_count + w_first, 1);
  arrived = __shfl_sync(0xffffffffu, arrived, 0);
  if (arrived != parts - 1) return;   // another part is still running
  __threadfence_block();
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
  for (int w = w_first; w <= w_last; ++w) {
    const int jw = warp_first_job(wk.jobs, w);
    if (warp_first_job(wk.jobs, w + 1) == jw) continue;   // no jobs, no part
    const float* src = part + ((w * 2 + (first_job < jw ? 0 : 1)) * 8) * 32;
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][i] += src[(4 * m + i) * 32 + lane];
  }
  finish_item<kGateUp>(p, it, acc, lane);
}

template <bool kGateUp>
__global__ void __launch_bounds__(GV_THREADS, 1)
    expert_gemv_fp8_kernel(const __grid_constant__ GemvParams p) {
  constexpr int FEATS = kGateUp ? 16 : 32;
  __shared__ int16_t units[GV_MAX_GROUPS + 1];   // prefix sums of the non-empty groups
  __shared__ int cut_count[GV_WARPS];            // arrivals at each cut item, by its first warp
  extern __shared__ __align__(16) uint8_t smem[];
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.E + p.S;
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int n = 0;
      if (g < p.E) n = min(p.T, max(0, p.offsets[g + 1] - p.offsets[g]));
      else if (g < G) n = p.T;
      int incl = (n + GV_UNIT_TOK - 1) / GV_UNIT_TOK;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (g < G) units[g + 1] = int16_t(carry + incl);
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) units[0] = 0;
    if (lane < GV_WARPS) cut_count[lane] = 0;
  }
  __syncthreads();

  Walk wk;
  wk.units = units;
  wk.G = G;
  wk.per_unit = p.n_out / FEATS;
  wk.total = int(units[G]) * wk.per_unit;
  wk.nblk = p.K / GV_KB;
  const int n_items = int(blockIdx.x) < wk.total
                          ? (wk.total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
  wk.jobs = n_items * wk.nblk;
  wk.j0 = warp_first_job(wk.jobs, warp);
  wk.j1 = warp_first_job(wk.jobs, warp + 1);
  wk.lane = lane;
  wk.ring = smem + size_t(warp) * GV_STAGES * GV_STAGE_BYTES;
  wk.ring_s = smem_u32(wk.ring);
  float* part = reinterpret_cast<float*>(smem + GV_RING_BYTES);

  IssueCursor ic;
  ic.job = wk.j0;
  ic.nt = 0;
  if (wk.j0 < wk.j1)
    cursor_at<kGateUp>(p, job_item<kGateUp>(p, wk, wk.j0 / wk.nblk), wk.j0 % wk.nblk, ic, lane);
  for (int s = 0; s < GV_STAGES - 1; ++s) issue_next<kGateUp>(p, wk, ic, s);

  int slot = 0;
  for (int j = wk.j0; j < wk.j1;) {
    const int q = j / wk.nblk, blk0 = j - q * wk.nblk;
    const int nb = min(wk.j1, (q + 1) * wk.nblk) - j;
    const Item it = job_item<kGateUp>(p, wk, q);
    run_segment<kGateUp>(p, wk, it, q, blk0, nb, ic, slot, part, cut_count, warp);
    j += nb;
  }
  cp_async_wait_all();
}

template <bool kGateUp>
cudaError_t launch_gemv(const GemvParams& gp, int num_sms, cudaStream_t st) {
  static thread_local int attrs_device = -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (attrs_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(expert_gemv_fp8_kernel<kGateUp>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(GV_SMEM));
    if (e != cudaSuccess) return e;
    attrs_device = dev;
  }
  return launch_pdl(expert_gemv_fp8_kernel<kGateUp>, dim3(unsigned(num_sms)), dim3(GV_THREADS),
                    GV_SMEM, st, 1, gp);
}

}  // namespace

moe_status launch_expert_ffn_gemv_fp8(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                                      cudaStream_t st) {
  if (a.T > GV_MAX_TOK) return MOE_ERR_INVALID_ARG;
  const moe_fp8_expert_weights& R = *a.fp8_routed;
  const moe_fp8_expert_weights& Sh = c.S > 0 ? *a.fp8_shared : R;   // unused when S == 0
  GemvParams gp = {};
  gp.w[0] = R.gate;
  gp.s[0] = R.gate_scale;
  gp.w[1] = R.up;
  gp.s[1] = R.up_scale;
  gp.sw[0] = Sh.gate;
  gp.ss[0] = Sh.gate_scale;
  gp.sw[1] = Sh.up;
  gp.ss[1] = Sh.up_scale;
  gp.tok_routed = a.x_perm;
  gp.tok_shared = a.x;
  gp.offsets = a.offsets;
  gp.out = a.h_act;
  gp.out_bf16 = 1;
  gp.T = a.T;
  gp.E = c.E;
  gp.S = c.S;
  gp.k = c.k;
  gp.K = c.d;
  gp.n_out = c.F;
  if (launch_gemv<true>(gp, dev.num_sms, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (a.after_gate_up && cudaEventRecord(a.after_gate_up, st) != cudaSuccess) return MOE_ERR_CUDA;

  GemvParams dp = {};
  dp.w[0] = dp.w[1] = R.down;
  dp.s[0] = dp.s[1] = R.down_scale;
  dp.sw[0] = dp.sw[1] = Sh.down;
  dp.ss[0] = dp.ss[1] = Sh.down_scale;
  dp.tok_routed = a.h_act;
  dp.tok_shared = a.h_act;
  dp.offsets = a.offsets;
  dp.out = a.Y;
  dp.out_bf16 = a.y_bf16 ? 1 : 0;
  dp.T = a.T;
  dp.E = c.E;
  dp.S = c.S;
  dp.k = c.k;
  dp.K = c.F;
  dp.n_out = c.d;
  if (launch_gemv<false>(dp, dev.num_sms, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
