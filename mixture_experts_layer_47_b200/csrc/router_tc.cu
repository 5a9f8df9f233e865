// router_tc.cu -- the router's score GEMM on the sm_100a tensor cores, at fp32 accuracy.
//
// The router scores every token against every expert (m.xxqk.cn Hy4-preview
// MoE explainer, section 2.2): logits = x W_r^T, x bf16 [T][d], W_r fp32 [E][d].
// The index parity of the top-k needs logits good to well under 1e-5, which
// bf16 or tf32 operands alone cannot give.  Two observations make the tensor
// cores usable anyway:
//  * x is exactly bf16, and W_r splits exactly into three bf16 parts
//    W_r = hi + mid + lo (hi = bf16(W_r), mid = bf16(W_r - hi),
//    lo = bf16(W_r - hi - mid); the residual is below 2^-24 |W_r|).  Every
//    product of a bf16 x with a bf16 part is exact in fp32.
//  * Whatever rounding the tensor core's fp32 accumulation applies, it is
//    confined to one 128-wide K chunk: each chunk's 24 MMAs (8 K16 steps x 3
//    parts) go into a fresh TMEM accumulator, and the epilogue warps add the
//    chunk results in fp32 on the CUDA cores, in chunk order (deterministic).
// Layout: a persistent kernel, one CTA per SM, 192 threads.  Warp 0 issues TMA
// loads (128 x 64 x-tile, three 128 x 64 W-part tiles, 128-byte swizzle, 3
// stages); warp 1 owns 512 TMEM columns = a ring of 4 accumulators of 128 x 128
// fp32 and issues tcgen05.mma (M=128, N=128); warps 2-5 drain the ring, one
// token row per thread.  A tile is (128 tokens, 128 experts, one K range); K is
// split across CTAs when there are too few tiles to fill the GPU, and the
// partial logits are added in split order by the top-k kernel.  Measured on B200
// at T = 8192, E = 256 (moe_route: the weight split, this kernel and the top-k):
// 0.109 ms with 128-expert tiles (one wave of 128 tiles) against 0.167 ms with
// 64-expert tiles (256 tiles in 1.7 waves, each x tile staged twice as often).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int RT_BM = 128;
constexpr int RT_BN = 128;
constexpr int RT_BK = 64;
constexpr int RT_STAGES = 3;
constexpr int RT_A_BYTES = RT_BM * RT_BK * 2;
constexpr int RT_B_BYTES = RT_BN * RT_BK * 2;
constexpr int RT_STAGE_BYTES = RT_A_BYTES + 3 * RT_B_BYTES;
constexpr int RT_RING = 4;          // accumulators of RT_BN columns
constexpr int RT_CHUNK_KB = 2;      // 64-wide K blocks accumulated per chunk (K = 128)
constexpr int RT_THREADS = 192;
constexpr uint32_t RT_IDESC = umma_idesc_bf16_f32(RT_BM, RT_BN);

struct __align__(64) RouterTcParams {
  CUtensorMap a;       // x [T][d] bf16, box 128 x 64
  CUtensorMap b;       // W parts [3E][d] bf16 (hi rows, mid rows, lo rows), box 64 x 64
  float* part;         // [ksplit][T][E] partial logits
  int* status;
  int T, E, d, ksplit;
};

struct RtShared {
  uint64_t full[RT_STAGES];
  uint64_t empty[RT_STAGES];
  uint64_t chunk_full[RT_RING];
  uint64_t chunk_free[RT_RING];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kRtSmem = 1024 + size_t(RT_STAGES) * RT_STAGE_BYTES + sizeof(RtShared);

__global__ void __launch_bounds__(RT_THREADS, 1)
    router_tc_kernel(const __grid_constant__ RouterTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  RtShared& ss = *reinterpret_cast<RtShared*>(smem + RT_STAGES * RT_STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int tiles_m = (p.T + RT_BM - 1) / RT_BM;
  const int tiles_n = (p.E + RT_BN - 1) / RT_BN;
  const int total = tiles_m * tiles_n * p.ksplit;
  const int kblocks = p.d / RT_BK / p.ksplit;   // K blocks per tile
  const int nchunks = (kblocks + RT_CHUNK_KB - 1) / RT_CHUNK_KB;   // chunks per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < RT_STAGES; ++s) {
      mbar_init(&ss.full[s], 1);
      mbar_init(&ss.empty[s], 1);
    }
    for (int r = 0; r < RT_RING; ++r) {
      mbar_init(&ss.chunk_full[r], 1);
      mbar_init(&ss.chunk_free[r], 128);
    }
    mbar_init(&ss.mma_done, 1);
    ss.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a);
    tma_prefetch_desc(&p.b);
  }
  if (warp == 1) {
    tmem_alloc(&ss.tmem_base, RT_RING * RT_BN);
    tmem_relinquish();
  }
  pdl_wait();   // x and the split weights come from earlier work on the stream
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ss.tmem_base;
  volatile int* abort_flag = &ss.abort_flag;

  // tile t -> (k split, m tile, n tile); n fastest so concurrent CTAs share the x tile
  auto decode = [&](int t, int& m, int& n, int& ks) {
    n = t % tiles_n;
    m = (t / tiles_n) % tiles_m;
    ks = t / (tiles_n * tiles_m);
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        if (*abort_flag) break;
        int m, n, ks;
        decode(t, m, n, ks);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&ss.empty[stage], phase ^ 1)) {
            report_error(p.status, kDevTimeout, kSiteProducer);
            *abort_flag = 1;
            stop = true;
            break;
          }
          uint8_t* st = smem + stage * RT_STAGE_BYTES;
          const int kc = (ks * kblocks + kb) * RT_BK;
          mbar_arrive_expect_tx(&ss.full[stage], RT_STAGE_BYTES);
          tma_load_2d_nohint(st, &p.a, &ss.full[stage], kc, m * RT_BM);
#pragma unroll
          for (int part = 0; part < 3; ++part)
            tma_load_2d_nohint(st + RT_A_BYTES + part * RT_B_BYTES, &p.b, &ss.full[stage], kc,
                               part * p.E + n * RT_BN);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == RT_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s = 0; s < RT_STAGES; ++s)
        if (issued_mask & (1u << s))
          if (!mbar_wait(&ss.full[s], (issued_parity >> s) & 1u, kDrainTimeoutNs))
            report_error(p.status, kDevTimeout, kSiteDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t chunk = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        if (*abort_flag) break;
        int kb = 0;
        for (int ch = 0; ch < nchunks && !stop; ++ch, ++chunk) {
          const uint32_t slot = chunk % RT_RING;
          const uint32_t use = chunk / RT_RING;
          if (!mbar_wait(&ss.chunk_free[slot], (use & 1u) ^ 1u)) {
            report_error(p.status, kDevTimeout, kSiteMma);
            *abort_flag = 1;
            stop = true;
            break;
          }
          const uint32_t d_tmem = tmem_base + slot * RT_BN;
          for (int sub = 0; sub < RT_CHUNK_KB && kb < kblocks; ++sub, ++kb) {
            if (!mbar_wait(&ss.full[stage], phase)) {
              report_error(p.status, kDevTimeout, kSiteMma);
              *abort_flag = 1;
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(smem + stage * RT_STAGE_BYTES);
            const uint64_t a_desc = umma_desc_sw128_kmajor(st);
#pragma unroll
            for (int kk = 0; kk < RT_BK / 16; ++kk)
#pragma unroll
              for (int part = 0; part < 3; ++part) {
                const uint64_t b_desc =
                    umma_desc_sw128_kmajor(st + RT_A_BYTES + part * RT_B_BYTES);
                umma_bf16(d_tmem, a_desc + uint64_t(2 * kk), b_desc + uint64_t(2 * kk),
                          RT_IDESC, (sub | kk | part) != 0 ? 1u : 0u);
              }
            umma_commit(&ss.empty[stage]);
            if (++stage == RT_STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (stop) break;
          umma_commit(&ss.chunk_full[slot]);
        }
      }
      umma_commit(&ss.mma_done);
      if (!mbar_wait(&ss.mma_done, 0, kDrainTimeoutNs))
        report_error(p.status, kDevTimeout, kSiteDrain);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    uint32_t chunk = 0;
    bool stop = false;
    for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
      int m, n, ks;
      decode(t, m, n, ks);
      float sum[RT_BN];
#pragma unroll
      for (int j = 0; j < RT_BN; ++j) sum[j] = 0.f;
      for (int ch = 0; ch < nchunks; ++ch, ++chunk) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { stop = true; break; }
        const uint32_t slot = chunk % RT_RING;
        const uint32_t use = chunk / RT_RING;
        if (!__all_sync(0xffffffffu, mbar_wait(&ss.chunk_full[slot], use & 1u))) {
          if (lane == 0) report_error(p.status, kDevTimeout, kSiteEpilogue);
          *abort_flag = 1;
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + slot * RT_BN;
#pragma unroll
        for (int half = 0; half < RT_BN / 64; ++half) {
          uint32_t v0[32], v1[32];   // 64 columns in flight, one wait
          tmem_ld_32cols(taddr + uint32_t(64 * half), v0);
          tmem_ld_32cols(taddr + uint32_t(64 * half + 32), v1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            sum[64 * half + j] += __uint_as_float(v0[j]);
            sum[64 * half + 32 + j] += __uint_as_float(v1[j]);
          }
        }
        tc_fence_before();
        mbar_arrive(&ss.chunk_free[slot]);
      }
      if (stop) break;
      const int tok = m * RT_BM + row;
      if (tok < p.T) {
        float* dst = p.part + (size_t(ks) * p.T + tok) * p.E + n * RT_BN;
        const int valid = min(RT_BN, p.E - n * RT_BN);
        if (valid == RT_BN && (p.E % 4) == 0) {
#pragma unroll
          for (int j = 0; j < RT_BN; j += 4)
            *reinterpret_cast<float4*>(dst + j) =
                make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < RT_BN; ++j)
            if (j < valid) dst[j] = sum[j];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, RT_RING * RT_BN);
  }
}

// W_r fp32 -> three bf16 parts with hi + mid + lo == W_r to within 2^-24 |W_r|.
__global__ void __launch_bounds__(256)
    split_router_weights_kernel(const float* __restrict__ Wr, size_t n,
                                uint16_t* __restrict__ parts) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    const float w = Wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    parts[i] = *reinterpret_cast<const uint16_t*>(&hi);
    parts[n + i] = *reinterpret_cast<const uint16_t*>(&mid);
    parts[2 * n + i] = *reinterpret_cast<const uint16_t*>(&lo);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode_rt = nullptr;
std::once_flag g_encode_rt_once;

bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    int box_rows) {
  std::call_once(g_encode_rt_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_rt = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode_rt) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {uint32_t(RT_BK), uint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return g_encode_rt(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int router_tc_ksplit(const Ctx& c, int T, int num_sms) {
  const int tiles = ((T + RT_BM - 1) / RT_BM) * ((c.E + RT_BN - 1) / RT_BN);
  const int kblocks = c.d / RT_BK;
  const int sms = num_sms > 0 ? num_sms : 148;
  int best = 1;
  for (int cand = 1; cand <= kblocks; ++cand)
    if (kblocks % cand == 0 && tiles * cand <= sms) best = cand;
  return best;
}

cudaError_t launch_router_tc(const Ctx& c, int ksplit, const uint16_t* x, const float* Wr, int T,
                             uint16_t* wparts, float* part, int* status, int num_sms,
                             cudaStream_t st) {
  static thread_local int attr_device = -1;
  int dev = -1;
  cudaGetDevice(&dev);
  if (attr_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(kRtSmem));
    if (e != cudaSuccess) return e;
    attr_device = dev;
  }
  const size_t n = size_t(c.E) * c.d;
  cudaError_t err = launch_pdl(split_router_weights_kernel,
                               dim3((unsigned)std::min<size_t>((n + 255) / 256, 4096)), dim3(256),
                               0, st, 1, Wr, n, wparts);
  if (err != cudaSuccess) return err;
  RouterTcParams p;
  memset(&p, 0, sizeof p);
  if (!encode_bf16_2d(&p.a, x, uint64_t(T), c.d, RT_BM) ||
      !encode_bf16_2d(&p.b, wparts, 3ull * c.E, c.d, RT_BN))
    return cudaErrorInvalidValue;
  p.part = part;
  p.status = status;
  p.T = T;
  p.E = c.E;
  p.d = c.d;
  p.ksplit = ksplit;
  const int tiles = ((T + RT_BM - 1) / RT_BM) * ((c.E + RT_BN - 1) / RT_BN) * ksplit;
  const int grid = std::min(tiles, num_sms > 0 ? num_sms : 148);
  return launch_pdl(router_tc_kernel, dim3(grid), dim3(RT_THREADS), kRtSmem, st, 1, p);
}

}  // namespace moe
