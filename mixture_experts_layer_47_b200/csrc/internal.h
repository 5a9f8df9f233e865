// internal.h -- host-side declarations shared by the translation units of
// libmoe.so (not part of the public ABI; see include/moe.h for that).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

// Launch a kernel with programmatic stream serialisation (and optionally a
// cluster shape); the kernel must call pdl_wait() before reading global data.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Forced choices of the router path and the GEMM tiling (tuning and tests).  They are
// read from the environment once, when the context is created (MOE_ROUTER,
// MOE_GEMM_TILES), so the workspace size and every later call of one context
// agree on the plan whatever the environment does afterwards.
enum class RouterMode { kAuto, kTensorCore, kFfma };
enum class TilesMode { kAuto, kSingle, kPair, kSwap, kSwapPair };

// A layer shape.  For a shard of the layer (moe_forward_partial) the expert
// stages see E = the local experts e_base .. e_base + E - 1 of the layer's
// E_all routed experts and S = the shared experts computed on this GPU.
struct Ctx {
  int d, E, k, F, S;
  RouterMode router = RouterMode::kAuto;
  TilesMode tiles = TilesMode::kAuto;
  bool fused_combine = false;   // MOE_FUSED_COMBINE=1 at moe_create
  int e_base = 0;   // first local expert
  int E_all = 0;    // routed experts of the whole layer (0: E)
  int e_all() const { return E_all > 0 ? E_all : E; }
};

// Geometry of the router's split-K partial sums for T tokens.
struct RouterPlan {
  bool tc;     // tensor-core score GEMM (router_tc.cu) rather than fp32 FFMA tiles
  int bt;      // FFMA: tokens per CTA tile (16, 64 or 128)
  int ksplit;  // number of K chunks (partial logits added in order by the top-k)
  int kchunk;  // d / ksplit
};
RouterPlan router_plan(const Ctx& c, int T, int num_sms);

// Workspace carve-up for T tokens (offsets from the 1024-aligned base).
struct Layout {
  size_t status, part, wparts, topk_idx, topk_w, counts, offsets, perm, pos, blk_hist, sched,
      x_perm, h_act, y_rows, x_stage, x_stage2, y_stage, down_part, grid_count, end;
  int nblk;           // dispatch blocks
  RouterPlan rplan;
};
Layout make_layout(const Ctx& c, int T, int num_sms);

constexpr int kDispatchChunk = 4096;   // slots per dispatch block
constexpr size_t kWsAlign = 1024;

// Per-device state, filled at the first launch on that device.
struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
  bool ready = false;
};
moe_status ensure_device(DeviceInfo** out);
// The layer shape a context was created with.
moe_status moe_internal_shape(moe_handle h, Ctx* out);

// ---- launchers (each returns cudaSuccess or the launch error) ----
cudaError_t launch_router(const Ctx& c, const RouterPlan& rp, const uint16_t* x, const float* Wr,
                          const float* bias, int T, float* part, uint16_t* wparts, int* status,
                          int num_sms, int32_t* topk_idx, float* topk_w, cudaStream_t st);
int router_tc_ksplit(const Ctx& c, int T, int num_sms);
cudaError_t launch_router_tc(const Ctx& c, int ksplit, const uint16_t* x, const float* Wr, int T,
                             uint16_t* wparts, float* part, int* status, int num_sms,
                             cudaStream_t st);
enum class GemmTiling { kSingle, kPair, kSwap, kSwapPair };
// Average routed rows per expert from which the 2-SM weight-major kernel is used.
constexpr int kSwapPairMinRowsPerExpert = 96;
GemmTiling gemm_tiling(const Ctx& c, int T);
// K ranges the dense layer's down projection is split into at small batches (1 = none): its
// d / 256 output tiles alone would leave most SMs idle.
constexpr int kDenseSplitMaxT = 128;
constexpr int kDenseSplitMax = 8;
int dense_down_ksplit(const Ctx& c, int T);

cudaError_t launch_dispatch(const Ctx& c, const int32_t* topk_idx, int T, int nblk,
                            int32_t* blk_hist, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* pos, int32_t* sched, int* status, cudaStream_t st);

cudaError_t launch_dense_schedule(int T, int32_t* offsets, int32_t* sched, cudaStream_t st);

cudaError_t launch_schedule_from_offsets(const Ctx& c, const int32_t* offsets, int T,
                                         int32_t* sched, cudaStream_t st);

cudaError_t launch_gather(const Ctx& c, const uint16_t* x, const int32_t* perm,
                          const int32_t* offsets, int T, uint16_t* x_perm, int num_sms,
                          cudaStream_t st);

cudaError_t launch_gather_tokens(const Ctx& c, const uint16_t* x, const int32_t* pos, int T,
                                 uint16_t* x_perm, int num_sms, cudaStream_t st);

cudaError_t launch_combine(const Ctx& c, const float* Y, const float* topk_w, const int32_t* pos,
                           int T, uint16_t* y, cudaStream_t st);
cudaError_t launch_combine_bf16(const Ctx& c, const uint16_t* Y, const float* topk_w,
                                const int32_t* pos, int T, uint16_t* y, cudaStream_t st);
cudaError_t launch_combine_partial(const Ctx& c, const uint16_t* Y, const float* topk_w,
                                   const int32_t* pos, int T, float* y_partial, cudaStream_t st);

// iHC: parallel residual streams per token (the pages' model uses 4).
constexpr int kMaxStreams = 8;
cudaError_t launch_ihc_mix(const Ctx& c, const uint16_t* H, const float* alpha, int n, int T,
                           uint16_t* x, cudaStream_t st);
cudaError_t launch_combine_ihc(const Ctx& c, const uint16_t* Y, const float* topk_w,
                               const int32_t* pos, int T, const uint16_t* H, const float* B,
                               const float* gamma, int n, uint16_t* H_out, cudaStream_t st);

// Up to this many fp32 partial outputs are added by one moe_reduce_partials call.
constexpr int kMaxPartials = 16;
struct PartialPtrs {
  const float* p[kMaxPartials];
};
cudaError_t launch_reduce_partials(const PartialPtrs& parts, int n, size_t elems, uint16_t* y,
                                   int num_sms, cudaStream_t st);

struct FfnArgs {
  const uint16_t* x;        // [T][d]
  const uint16_t* x_perm;   // [T*k][d]
  const int32_t* offsets;   // [E+1]
  const int32_t* sched;     // [2(E+S+1)]: 128-row then 256-row tile prefix sums
  const uint16_t *Wg, *Wu, *Wd, *Sg, *Su, *Sd;
  uint16_t* h_act;          // [T*k+S*T][F]
  void* Y;                  // [T*k+S*T][d], fp32 or (y_bf16) bf16
  bool y_bf16;
  int* status;
  int T;
  cudaEvent_t after_gate_up;  // recorded between the two GEMMs when non-null
  // FP8 weights (then Wg..Sd are unused): the routed set and the shared set
  // (nullptr when S == 0); both nullptr for bf16 weights.
  const moe_fp8_expert_weights* fp8_routed = nullptr;
  const moe_fp8_expert_weights* fp8_shared = nullptr;
  // Down projection split over K (1-SM weight-major tiling, bf16 Y): fp32 parts
  // [down_ksplit][rows][d] in the workspace, added in order into Y.
  int down_ksplit = 1;
  float* down_part = nullptr;
  // With split_count (zeroed, one counter per output tile) the down GEMM adds the parts
  // itself: the last K range to finish an output tile sums them, in range order.
  unsigned int* split_count = nullptr;
  // The dense layer: one group of dense_T rows and no shared group; the weight-major GEMMs
  // build that schedule themselves (offsets and sched are then not read).
  int dense_T = 0;
  // The combine fused into the down GEMM (weight-major tilings, bf16 Y rows): the down
  // kernel writes y itself after a grid-wide barrier on grid_count (workspace).
  bool fuse_combine = false;
  const float* topk_w = nullptr;
  const int32_t* pos = nullptr;
  uint16_t* y_out = nullptr;
  unsigned int* grid_count = nullptr;
};
moe_status launch_expert_ffn(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                             cudaStream_t st);
bool swap_down_all_resident(bool pair);
moe_status launch_expert_ffn_swap(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                                  bool pair, cudaStream_t st);
moe_status launch_expert_ffn_fp8(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                                 cudaStream_t st);
// FP8 expert FFNs on the CUDA cores (expert_gemv_fp8.cu), taken by launch_expert_ffn_fp8
// for batches of at most kGemvMaxT tokens unless a weight-major tiling is asked for.
constexpr int kGemvMaxT = 16;
moe_status launch_expert_ffn_gemv_fp8(const Ctx& c, const FfnArgs& a, const DeviceInfo& dev,
                                      cudaStream_t st);

}  // namespace moe
