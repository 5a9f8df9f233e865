// moe_api.cu -- the extern "C" entry points declared in include/moe.h.
//
// Host-side argument checks, the workspace carve-up, and the launch sequence
// of the layer: router -> dispatch -> gather -> gate/up GEMM (+SwiGLU) ->
// down GEMM -> combine, all on the caller's stream with no host
// synchronisation.  The carve-up does not depend on the device, so the
// workspace size and every result are the same on any sm_100 GPU.
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <new>

#include "common.cuh"
#include "internal.h"

// The input copies of moe_forward_host / moe_forward_fp8_host run on a helper stream
// (one per device, made at the context's first such call on it) into two staging slots
// used in turn, so that a call's copy can start while the previous call's layer runs.
struct HostPipe {
  bool ready = false;
  cudaStream_t copy = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr};   // the slot's input copy has landed
  cudaEvent_t freed[2] = {nullptr, nullptr};    // the layer that read the slot is done
  unsigned next = 0;                            // slot of the next call
};

struct moe_ctx {
  moe::Ctx c;
  cudaEvent_t stage_events[MOE_STAGE_EVENTS];
  int n_stage_events;
  HostPipe pipes[64];   // per device ordinal
  std::mutex pipe_mu;
};

namespace moe {
namespace {

constexpr int kPlanSms = 148;            // device-independent planning constant
constexpr long long kMaxRows = 1ll << 24;  // T*k + S*T upper bound
constexpr int kMaxDevices = 64;

DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mu;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint8_t* aligned_base(void* ws) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + kWsAlign - 1) &
                                    ~uintptr_t(kWsAlign - 1));
}

moe_status check_T(const Ctx& c, int T) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)T * (c.k + c.S) > kMaxRows) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ws(moe_handle h, int T, const void* ws, size_t ws_bytes) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size(h, T)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  cudaGetLastError();  // clear a non-sticky error so the caller's context stays usable
  return MOE_ERR_CUDA;
}

}  // namespace

Layout make_layout(const Ctx& c, int T, int num_sms) {
  Layout L;
  memset(&L, 0, sizeof L);
  L.rplan = router_plan(c, T, num_sms);
  const size_t nslots = size_t(T) * c.k;
  const size_t rows = nslots + size_t(c.S) * T;
  L.nblk = int(std::max<size_t>(1, (nslots + kDispatchChunk - 1) / kDispatchChunk));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + std::max<size_t>(bytes, 16), kWsAlign);
    return o;
  };
  L.status = take(2048);   // status word, grid counter, and the dense K split's counters
  L.part = take(size_t(L.rplan.ksplit) * T * c.E * sizeof(float));
  L.wparts = take(L.rplan.tc ? 3 * size_t(c.E) * c.d * sizeof(uint16_t) : 0);
  L.topk_idx = take(nslots * sizeof(int32_t));
  L.topk_w = take(nslots * sizeof(float));
  L.counts = take(size_t(c.E) * sizeof(int32_t));
  L.offsets = take(size_t(c.E + 1) * sizeof(int32_t));
  L.perm = take(nslots * sizeof(int32_t));
  L.pos = take(nslots * sizeof(int32_t));
  L.blk_hist = take(size_t(L.nblk) * c.E * sizeof(int32_t));
  L.sched = take(2 * size_t(c.E + c.S + 1) * sizeof(int32_t));  // 128- and 256-row tiles
  L.x_perm = take(nslots * c.d * sizeof(uint16_t));
  L.h_act = take(rows * c.F * sizeof(uint16_t));
  L.y_rows = take(rows * c.d * sizeof(uint16_t));  // bf16 rows of moe_forward
  L.x_stage = take(size_t(T) * c.d * sizeof(uint16_t));
  L.x_stage2 = take(size_t(T) * c.d * sizeof(uint16_t));
  L.y_stage = take(size_t(T) * c.d * sizeof(uint16_t));
  L.down_part = take(size_t(dense_down_ksplit(c, T) > 1 ? dense_down_ksplit(c, T) : 0) * T * c.d *
                     sizeof(float));
  L.grid_count = L.status + 64;   // inside the status block, cleared with the status word
  L.end = off;
  return L;
}

moe_status ensure_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& di = g_devices[dev];
  if (!di.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    // The kernels are built for sm_100a only (arch-specific tcgen05 / TMA).
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;
    di.device = dev;
    di.cc_major = major;
    di.cc_minor = minor;
    di.num_sms = sms;
    di.ready = true;
  }
  *out = &di;
  return MOE_OK;
}

moe_status moe_internal_shape(moe_handle h, Ctx* out) {
  if (!h || !out) return MOE_ERR_INVALID_ARG;
  *out = h->c;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_create(int d_model, int n_experts, int top_k, int d_ff, int n_shared,
                      moe_handle* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (d_model <= 0 || d_ff <= 0 || n_experts <= 0 || top_k < 1 || top_k > n_experts ||
      n_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (d_model % 64 || d_ff % 64 || d_model > 65536 || d_ff > 65536 || n_experts > 1024 ||
      top_k > 32 || n_shared > 8)
    return MOE_ERR_UNSUPPORTED;
  moe_ctx* h = new (std::nothrow) moe_ctx;
  if (!h) return MOE_ERR_INVALID_ARG;
  h->c = Ctx{d_model, n_experts, top_k, d_ff, n_shared};
  // Tuning overrides, fixed for the context's lifetime (unknown values are ignored).
  if (const char* v = getenv("MOE_ROUTER")) {
    if (strcmp(v, "tc") == 0) h->c.router = RouterMode::kTensorCore;
    if (strcmp(v, "ffma") == 0) h->c.router = RouterMode::kFfma;
  }
  if (const char* v = getenv("MOE_FUSED_COMBINE"))
    h->c.fused_combine = strcmp(v, "1") == 0;
  if (const char* v = getenv("MOE_GEMM_TILES")) {
    if (strcmp(v, "single") == 0) h->c.tiles = TilesMode::kSingle;
    if (strcmp(v, "pair") == 0) h->c.tiles = TilesMode::kPair;
    if (strcmp(v, "swap") == 0) h->c.tiles = TilesMode::kSwap;
    if (strcmp(v, "swap_pair") == 0) h->c.tiles = TilesMode::kSwapPair;
  }
  h->n_stage_events = 0;
  *out = h;
  return MOE_OK;
}

moe_status moe_destroy(moe_handle h) {
  if (!h) return MOE_OK;
  int cur = -1;
  const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
  for (int d = 0; d < 64; ++d) {
    HostPipe& hp = h->pipes[d];
    if (!hp.ready || cudaSetDevice(d) != cudaSuccess) continue;
    cudaStreamDestroy(hp.copy);
    for (int i = 0; i < 2; ++i) {
      cudaEventDestroy(hp.copied[i]);
      cudaEventDestroy(hp.freed[i]);
    }
  }
  if (have_cur) cudaSetDevice(cur);
  cudaGetLastError();
  delete h;
  return MOE_OK;
}

size_t moe_workspace_size(moe_handle h, int T) {
  if (!h || T < 0) return 0;
  if ((long long)T * (h->c.k + h->c.S) > kMaxRows) return 0;
  return make_layout(h->c, T, kPlanSms).end + kWsAlign;
}

moe_status moe_get_workspace_layout(moe_handle h, int T, uintptr_t workspace_addr,
                                    moe_workspace_layout* out) {
  if (!h || !out) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  const Layout L = make_layout(h->c, T, kPlanSms);
  const size_t base = ((workspace_addr + kWsAlign - 1) & ~uintptr_t(kWsAlign - 1)) - workspace_addr;
  out->status = base + L.status;
  out->router_partials = base + L.part;
  out->router_ksplit = size_t(L.rplan.ksplit);
  out->topk_idx = base + L.topk_idx;
  out->topk_w = base + L.topk_w;
  out->counts = base + L.counts;
  out->offsets = base + L.offsets;
  out->perm = base + L.perm;
  out->pos = base + L.pos;
  out->h_act = base + L.h_act;
  out->y_rows = base + L.y_rows;
  out->total = base + L.end;
  return MOE_OK;
}

moe_status moe_route(moe_handle h, const uint16_t* x, const float* W_router, const float* bias,
                     int T, int32_t* topk_idx, float* topk_w, void* workspace, size_t ws_bytes,
                     void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if (!x || !W_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_router)) return MOE_ERR_ALIGNMENT;
  if ((s = check_ws(h, T, workspace, ws_bytes))) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(h->c, T, kPlanSms);
  uint8_t* ws = aligned_base(workspace);
  if ((s = cuda_status(cudaMemsetAsync(ws + L.status, 0, sizeof(int), st)))) return s;
  return cuda_status(launch_router(h->c, L.rplan, x, W_router, bias, T,
                                   reinterpret_cast<float*>(ws + L.part),
                                   reinterpret_cast<uint16_t*>(ws + L.wparts),
                                   reinterpret_cast<int*>(ws + L.status), dev->num_sms, topk_idx,
                                   topk_w, st));
}

moe_status moe_dispatch(moe_handle h, const int32_t* topk_idx, int T, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* pos, void* workspace,
                        size_t ws_bytes, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if (!topk_idx || !counts || !offsets || !perm || !pos) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(h, T, workspace, ws_bytes))) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(h->c, T, kPlanSms);
  uint8_t* ws = aligned_base(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status);
  if ((s = cuda_status(cudaMemsetAsync(status, 0, sizeof(int), st)))) return s;
  return cuda_status(launch_dispatch(h->c, topk_idx, T, L.nblk,
                                     reinterpret_cast<int32_t*>(ws + L.blk_hist), counts, offsets,
                                     perm, pos, reinterpret_cast<int32_t*>(ws + L.sched), status,
                                     st));
}

// Expert weights of one call: bf16 (Wg..Sd) or FP8 (r8 / s8, the others null).
struct Weights {
  const uint16_t *Wg = nullptr, *Wu = nullptr, *Wd = nullptr;
  const uint16_t *Sg = nullptr, *Su = nullptr, *Sd = nullptr;
  const moe_fp8_expert_weights* r8 = nullptr;
  const moe_fp8_expert_weights* s8 = nullptr;
};

static Weights bf16_weights(const uint16_t* Wg, const uint16_t* Wu, const uint16_t* Wd,
                            const uint16_t* Sg, const uint16_t* Su, const uint16_t* Sd) {
  Weights w;
  w.Wg = Wg;
  w.Wu = Wu;
  w.Wd = Wd;
  w.Sg = Sg;
  w.Su = Su;
  w.Sd = Sd;
  return w;
}

static Weights fp8_weights(const moe_fp8_expert_weights* r8, const moe_fp8_expert_weights* s8) {
  Weights w;
  w.r8 = r8;
  w.s8 = s8;
  return w;
}

static moe_status check_fp8_set(const moe_fp8_expert_weights* w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  const uint8_t* ptrs[6] = {w->gate, w->gate_scale, w->up, w->up_scale, w->down, w->down_scale};
  for (const uint8_t* q : ptrs)
    if (!q) return MOE_ERR_INVALID_ARG;
  for (const uint8_t* q : ptrs)
    if (!aligned16(q)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

static moe_status check_weights(const Ctx& c, const Weights& w) {
  if (w.r8 || w.s8) {
    moe_status s = check_fp8_set(w.r8);
    if (s) return s;
    return c.S > 0 ? check_fp8_set(w.s8) : MOE_OK;
  }
  if (!w.Wg || !w.Wu || !w.Wd) return MOE_ERR_INVALID_ARG;
  if (c.S > 0 && (!w.Sg || !w.Su || !w.Sd)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w.Wg) || !aligned16(w.Wu) || !aligned16(w.Wd)) return MOE_ERR_ALIGNMENT;
  if (c.S > 0 && (!aligned16(w.Sg) || !aligned16(w.Su) || !aligned16(w.Sd)))
    return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

static void set_weights(FfnArgs& a, const Weights& w) {
  a.Wg = w.Wg;
  a.Wu = w.Wu;
  a.Wd = w.Wd;
  a.Sg = w.Sg;
  a.Su = w.Su;
  a.Sd = w.Sd;
  a.fp8_routed = w.r8;
  a.fp8_shared = w.s8;
}

static moe_status expert_ffn_impl(moe_handle h, const uint16_t* x, const int32_t* perm,
                                  const int32_t* offsets, int T, const Weights& w, float* Y,
                                  void* workspace, size_t ws_bytes, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  moe_status s = check_T(c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if (!x || !perm || !offsets || !Y) return MOE_ERR_INVALID_ARG;
  if ((s = check_weights(c, w))) return s;
  if (!aligned16(x) || !aligned16(Y)) return MOE_ERR_ALIGNMENT;
  if ((s = check_ws(h, T, workspace, ws_bytes))) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(c, T, kPlanSms);
  uint8_t* ws = aligned_base(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status);
  int32_t* sched = reinterpret_cast<int32_t*>(ws + L.sched);
  uint16_t* x_perm = reinterpret_cast<uint16_t*>(ws + L.x_perm);
  if ((s = cuda_status(cudaMemsetAsync(status, 0, sizeof(int), st)))) return s;
  if ((s = cuda_status(launch_schedule_from_offsets(c, offsets, T, sched, st)))) return s;
  if ((s = cuda_status(launch_gather(c, x, perm, offsets, T, x_perm, dev->num_sms, st)))) return s;
  FfnArgs a;
  a.x = x;
  a.x_perm = x_perm;
  a.offsets = offsets;
  a.sched = sched;
  set_weights(a, w);
  a.h_act = reinterpret_cast<uint16_t*>(ws + L.h_act);
  a.Y = Y;
  a.y_bf16 = false;
  a.status = status;
  a.T = T;
  a.after_gate_up = nullptr;
  return launch_expert_ffn(c, a, *dev, st);
}

moe_status moe_expert_ffn(moe_handle h, const uint16_t* x, const int32_t* perm,
                          const int32_t* offsets, int T, const uint16_t* W_gate,
                          const uint16_t* W_up, const uint16_t* W_down, const uint16_t* Ws_gate,
                          const uint16_t* Ws_up, const uint16_t* Ws_down, float* Y,
                          void* workspace, size_t ws_bytes, void* stream) {
  return expert_ffn_impl(h, x, perm, offsets, T,
                         bf16_weights(W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down), Y,
                         workspace, ws_bytes, stream);
}

moe_status moe_expert_ffn_fp8(moe_handle h, const uint16_t* x, const int32_t* perm,
                              const int32_t* offsets, int T, const moe_fp8_expert_weights* routed,
                              const moe_fp8_expert_weights* shared, float* Y, void* workspace,
                              size_t ws_bytes, void* stream) {
  if (!routed) return MOE_ERR_INVALID_ARG;
  return expert_ffn_impl(h, x, perm, offsets, T, fp8_weights(routed, shared), Y, workspace,
                         ws_bytes, stream);
}

moe_status moe_combine(moe_handle h, const float* Y, const float* topk_w, const int32_t* pos,
                       int T, uint16_t* y, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if (!Y || !topk_w || !pos || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(Y) || !aligned16(y)) return MOE_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  return cuda_status(
      launch_combine(h->c, Y, topk_w, pos, T, y, reinterpret_cast<cudaStream_t>(stream)));
}

// Whether moe_forward runs the combine inside the down GEMM (context option
// MOE_FUSED_COMBINE=1; only the weight-major tilings have the fused form).
static bool combine_fused(const Ctx& c, int T) {
  if (!c.fused_combine) return false;
  const GemmTiling t = gemm_tiling(c, T);
  if (t != GemmTiling::kSwap && t != GemmTiling::kSwapPair) return false;
  // its grid-wide barrier needs every CTA of the down GEMM resident at once
  return swap_down_all_resident(t == GemmTiling::kSwapPair);
}

// A shard of the layer for tensor or expert parallelism: the routed experts
// e_base .. e_base + n_local - 1 (the caller's weights hold just those), with or
// without the shared experts, and an unrounded fp32 output.
struct Shard {
  int e_base, n_local;
  bool shared;
  float* y_partial;
};

// The iHC wrapper's stream update, done by the combine (moe_forward_ihc).
struct IhcArgs {
  const uint16_t* H;     // [T][n][d] streams in
  const float* B;        // [n][n] exchange between streams
  const float* gamma;    // [n] weight of the layer output per stream
  int n;
  uint16_t* H_out;       // [T][n][d] streams out (may be H)
};

// The shape the expert stages see: the whole layer, or one shard of it.
static Ctx stage_shape(const Ctx& c, const Shard* sh) {
  Ctx cl = c;
  if (sh) {
    cl.e_base = sh->e_base;
    cl.E = sh->n_local;
    cl.E_all = c.E;
    if (!sh->shared) cl.S = 0;
  }
  return cl;
}

static moe_status forward_device(moe_handle h, const uint16_t* x, const float* W_router,
                                 const float* bias, const Weights& w, int T, uint16_t* y,
                                 uint8_t* ws, const Layout& L, DeviceInfo* dev, cudaStream_t st,
                                 const Shard* shard = nullptr, const IhcArgs* ihc = nullptr) {
  const Ctx& c = h->c;
  const Ctx cl = stage_shape(c, shard);   // dispatch, gather, GEMMs and combine
  moe_status s;
  int* status = reinterpret_cast<int*>(ws + L.status);
  int32_t* topk_idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  float* topk_w = reinterpret_cast<float*>(ws + L.topk_w);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
  int32_t* pos = reinterpret_cast<int32_t*>(ws + L.pos);
  int32_t* sched = reinterpret_cast<int32_t*>(ws + L.sched);
  uint16_t* x_perm = reinterpret_cast<uint16_t*>(ws + L.x_perm);
  uint16_t* Y = reinterpret_cast<uint16_t*>(ws + L.y_rows);  // bf16 rows
  const bool prof = h->n_stage_events == MOE_STAGE_EVENTS;
  auto mark = [&](int i) -> moe_status {
    return prof ? cuda_status(cudaEventRecord(h->stage_events[i], st)) : MOE_OK;
  };
  // the status word and the fused combine's grid counter (same 256-byte block)
  if ((s = cuda_status(cudaMemsetAsync(status, 0, 128, st)))) return s;
  if ((s = mark(0))) return s;
  if ((s = cuda_status(launch_router(c, L.rplan, x, W_router, bias, T,
                                     reinterpret_cast<float*>(ws + L.part),
                                     reinterpret_cast<uint16_t*>(ws + L.wparts), status,
                                     dev->num_sms, topk_idx, topk_w, st))))
    return s;
  if ((s = mark(1))) return s;
  if ((s = cuda_status(launch_dispatch(cl, topk_idx, T, L.nblk,
                                       reinterpret_cast<int32_t*>(ws + L.blk_hist), counts,
                                       offsets, perm, pos, sched, status, st))))
    return s;
  if ((s = mark(2))) return s;
  if ((s = cuda_status(launch_gather_tokens(cl, x, pos, T, x_perm, dev->num_sms, st)))) return s;
  if ((s = mark(3))) return s;
  FfnArgs a;
  a.x = x;
  a.x_perm = x_perm;
  a.offsets = offsets;
  a.sched = sched;
  set_weights(a, w);
  a.h_act = reinterpret_cast<uint16_t*>(ws + L.h_act);
  a.Y = Y;
  a.status = status;
  a.T = T;
  a.y_bf16 = true;
  a.after_gate_up = prof ? h->stage_events[4] : nullptr;
  const bool fuse = combine_fused(c, T) && !shard && !w.r8 && !ihc;
  a.fuse_combine = fuse;
  a.topk_w = topk_w;
  a.pos = pos;
  a.y_out = y;
  a.grid_count = reinterpret_cast<unsigned int*>(ws + L.grid_count);
  if ((s = launch_expert_ffn(cl, a, *dev, st))) return s;
  if ((s = mark(5))) return s;
  if (shard)
    s = cuda_status(launch_combine_partial(cl, Y, topk_w, pos, T, shard->y_partial, st));
  else if (ihc)
    s = cuda_status(launch_combine_ihc(c, Y, topk_w, pos, T, ihc->H, ihc->B, ihc->gamma, ihc->n,
                                       ihc->H_out, st));
  else if (!fuse)
    s = cuda_status(launch_combine_bf16(c, Y, topk_w, pos, T, y, st));
  if (s) return s;
  return mark(6);
}

static moe_status check_forward_args(moe_handle h, const uint16_t* x, const float* W_router,
                                     const Weights& w, int T, const uint16_t* y, bool host_io,
                                     const void* workspace, size_t ws_bytes) {
  if (!x || !W_router || !y) return MOE_ERR_INVALID_ARG;
  moe_status s;
  if ((s = check_weights(h->c, w))) return s;
  if (!aligned16(W_router)) return MOE_ERR_ALIGNMENT;
  if (!host_io && (!aligned16(x) || !aligned16(y))) return MOE_ERR_ALIGNMENT;
  return check_ws(h, T, workspace, ws_bytes);
}

static moe_status forward_impl(moe_handle h, const uint16_t* x, const float* W_router,
                               const float* bias, const Weights& w, int T, uint16_t* y,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if ((s = check_forward_args(h, x, W_router, w, T, y, false, workspace, ws_bytes))) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  const Layout L = make_layout(h->c, T, kPlanSms);
  return forward_device(h, x, W_router, bias, w, T, y, aligned_base(workspace), L, dev,
                        reinterpret_cast<cudaStream_t>(stream));
}

// The input copy of a host-activation call: on the device's helper stream, into the next of
// the two staging slots once the layer that last read that slot is done; the caller's stream
// then waits for it.  *slot receives the slot, *x_dev its device address.
static moe_status stage_host_input(moe_handle h, const DeviceInfo* dev, const Layout& L,
                                   uint8_t* ws, const uint16_t* x_host, size_t bytes,
                                   cudaStream_t st, unsigned* slot, uint16_t** x_dev) {
  HostPipe& hp = h->pipes[dev->device];
  {
    std::lock_guard<std::mutex> lock(h->pipe_mu);
    if (!hp.ready) {
      bool ok = cudaStreamCreateWithFlags(&hp.copy, cudaStreamNonBlocking) == cudaSuccess;
      for (int i = 0; i < 2 && ok; ++i)
        ok = cudaEventCreateWithFlags(&hp.copied[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.freed[i], cudaEventDisableTiming) == cudaSuccess;
      if (!ok) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      hp.ready = true;
    }
    *slot = hp.next++ & 1u;
  }
  *x_dev = reinterpret_cast<uint16_t*>(ws + (*slot ? L.x_stage2 : L.x_stage));
  moe_status s;
  if ((s = cuda_status(cudaStreamWaitEvent(hp.copy, hp.freed[*slot], 0)))) return s;
  if ((s = cuda_status(
           cudaMemcpyAsync(*x_dev, x_host, bytes, cudaMemcpyHostToDevice, hp.copy))))
    return s;
  if ((s = cuda_status(cudaEventRecord(hp.copied[*slot], hp.copy)))) return s;
  return cuda_status(cudaStreamWaitEvent(st, hp.copied[*slot], 0));
}

// After the layer that read a staging slot: the slot is free again once the stream gets
// here, and the output goes back to the host on the caller's stream.
static moe_status finish_host_output(moe_handle h, const DeviceInfo* dev, unsigned slot,
                                     uint16_t* y_host, const uint16_t* y_dev, size_t bytes,
                                     cudaStream_t st) {
  moe_status s;
  if ((s = cuda_status(cudaEventRecord(h->pipes[dev->device].freed[slot], st)))) return s;
  return cuda_status(cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, st));
}

static moe_status forward_host_impl(moe_handle h, const uint16_t* x_host, const float* W_router,
                                    const float* bias, const Weights& w, int T, uint16_t* y_host,
                                    void* workspace, size_t ws_bytes, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if ((s = check_forward_args(h, x_host, W_router, w, T, y_host, true, workspace, ws_bytes)))
    return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(h->c, T, kPlanSms);
  uint8_t* ws = aligned_base(workspace);
  const size_t bytes = size_t(T) * h->c.d * sizeof(uint16_t);
  unsigned slot;
  uint16_t* x_dev;
  if ((s = stage_host_input(h, dev, L, ws, x_host, bytes, st, &slot, &x_dev))) return s;
  uint16_t* y_dev = reinterpret_cast<uint16_t*>(ws + L.y_stage);
  if ((s = forward_device(h, x_dev, W_router, bias, w, T, y_dev, ws, L, dev, st))) return s;
  return finish_host_output(h, dev, slot, y_host, y_dev, bytes, st);
}

moe_status moe_forward(moe_handle h, const uint16_t* x, const float* W_router, const float* bias,
                       const uint16_t* W_gate, const uint16_t* W_up, const uint16_t* W_down,
                       const uint16_t* Ws_gate, const uint16_t* Ws_up, const uint16_t* Ws_down,
                       int T, uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
  return forward_impl(h, x, W_router, bias,
                      bf16_weights(W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down), T, y,
                      workspace, ws_bytes, stream);
}

moe_status moe_forward_host(moe_handle h, const uint16_t* x_host, const float* W_router,
                            const float* bias, const uint16_t* W_gate, const uint16_t* W_up,
                            const uint16_t* W_down, const uint16_t* Ws_gate,
                            const uint16_t* Ws_up, const uint16_t* Ws_down, int T,
                            uint16_t* y_host, void* workspace, size_t ws_bytes, void* stream) {
  return forward_host_impl(h, x_host, W_router, bias,
                           bf16_weights(W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down), T,
                           y_host, workspace, ws_bytes, stream);
}

moe_status moe_forward_fp8(moe_handle h, const uint16_t* x, const float* W_router,
                           const float* bias, const moe_fp8_expert_weights* routed,
                           const moe_fp8_expert_weights* shared, int T, uint16_t* y,
                           void* workspace, size_t ws_bytes, void* stream) {
  if (!routed) return MOE_ERR_INVALID_ARG;
  return forward_impl(h, x, W_router, bias, fp8_weights(routed, shared), T, y, workspace,
                      ws_bytes, stream);
}

moe_status moe_forward_fp8_host(moe_handle h, const uint16_t* x_host, const float* W_router,
                                const float* bias, const moe_fp8_expert_weights* routed,
                                const moe_fp8_expert_weights* shared, int T, uint16_t* y_host,
                                void* workspace, size_t ws_bytes, void* stream) {
  if (!routed) return MOE_ERR_INVALID_ARG;
  return forward_host_impl(h, x_host, W_router, bias, fp8_weights(routed, shared), T, y_host,
                           workspace, ws_bytes, stream);
}

moe_status moe_forward_partial(moe_handle h, const uint16_t* x, const float* W_router,
                               const float* bias, int expert_begin, int n_local_experts,
                               const uint16_t* W_gate, const uint16_t* W_up,
                               const uint16_t* W_down, const uint16_t* Ws_gate,
                               const uint16_t* Ws_up, const uint16_t* Ws_down, int T,
                               float* y_partial, void* workspace, size_t ws_bytes,
                               void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (expert_begin < 0 || n_local_experts < 1 ||
      (long long)expert_begin + n_local_experts > h->c.E)
    return MOE_ERR_INVALID_ARG;
  const int n_shared_ptrs = (Ws_gate != nullptr) + (Ws_up != nullptr) + (Ws_down != nullptr);
  if (n_shared_ptrs != 0 && n_shared_ptrs != 3) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const Shard shard{expert_begin, n_local_experts, n_shared_ptrs == 3 && h->c.S > 0, y_partial};
  const Ctx cl = stage_shape(h->c, &shard);
  const Weights w = bf16_weights(W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down);
  if (!x || !W_router || !y_partial) return MOE_ERR_INVALID_ARG;
  if ((s = check_weights(cl, w))) return s;
  if (!aligned16(x) || !aligned16(W_router) || !aligned16(y_partial)) return MOE_ERR_ALIGNMENT;
  if ((s = check_ws(h, T, workspace, ws_bytes))) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  const Layout L = make_layout(h->c, T, kPlanSms);
  return forward_device(h, x, W_router, bias, w, T, nullptr, aligned_base(workspace), L, dev,
                        reinterpret_cast<cudaStream_t>(stream), &shard);
}

// The checks of moe_dense_ffn and moe_dense_ffn_host (x and y device or host pointers).
static moe_status check_dense_args(moe_handle h, const uint16_t* x, const uint16_t* W_gate,
                                   const uint16_t* W_up, const uint16_t* W_down, int T,
                                   const uint16_t* y, void* workspace, size_t ws_bytes) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if (c.E != 1 || c.k != 1 || c.S != 0) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(c, T);
  if (s) return s;
  if (T == 0) return MOE_OK;
  if (!x || !W_gate || !W_up || !W_down || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) ||
      !aligned16(y))
    return MOE_ERR_ALIGNMENT;
  return check_ws(h, T, workspace, ws_bytes);
}

// The dense layer on device activations: the checks are done.
// The dense layer on the weight-major tilings: the GEMMs build the one-group schedule
// themselves, and the down GEMM's K ranges add their parts in the kernel when the counters
// (one per output tile and epilogue warp) fit the status block's last kilobyte.
static bool dense_weight_major(const Ctx& c, int T) {
  const GemmTiling t = gemm_tiling(c, T);
  return t == GemmTiling::kSwap || t == GemmTiling::kSwapPair;
}
constexpr size_t kSplitCountOffset = 1024;   // inside the 2 KB status block
constexpr int kMaxSplitCounters = 256;
static bool dense_split_summed_in_gemm(const Ctx& c, int T) {
  return dense_down_ksplit(c, T) > 1 &&
         ((T + 127) / 128) * ((c.d + 255) / 256) * 8 <= kMaxSplitCounters;
}

static moe_status dense_device(moe_handle h, const uint16_t* x, const uint16_t* W_gate,
                               const uint16_t* W_up, const uint16_t* W_down, int T, uint16_t* y,
                               uint8_t* ws, const Layout& L, const DeviceInfo* dev,
                               cudaStream_t st) {
  const Ctx& c = h->c;
  moe_status s;
  int* status = reinterpret_cast<int*>(ws + L.status);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* sched = reinterpret_cast<int32_t*>(ws + L.sched);
  const bool prof = h->n_stage_events == MOE_STAGE_EVENTS;
  auto mark = [&](int i) -> moe_status {
    return prof ? cuda_status(cudaEventRecord(h->stage_events[i], st)) : MOE_OK;
  };
  const bool wm = dense_weight_major(c, T);
  const bool split_in_gemm = wm && dense_split_summed_in_gemm(c, T);
  // the status word and the down GEMM's K-split counters (same 2 KB block)
  if ((s = cuda_status(cudaMemsetAsync(status, 0, 2048, st)))) return s;
  if ((s = mark(0))) return s;
  if ((s = mark(1))) return s;   // no router
  if (!wm && (s = cuda_status(launch_dense_schedule(T, offsets, sched, st)))) return s;
  if ((s = mark(2))) return s;   // the one-group schedule in place of dispatch
  if ((s = mark(3))) return s;   // no gather
  // One group holding every token in order: the GEMMs read x itself as the group's rows and
  // the down GEMM's rows are y (weight 1, nothing to combine).
  FfnArgs a;
  a.x = x;
  a.x_perm = x;
  a.offsets = offsets;
  a.sched = sched;
  set_weights(a, bf16_weights(W_gate, W_up, W_down, nullptr, nullptr, nullptr));
  a.h_act = reinterpret_cast<uint16_t*>(ws + L.h_act);
  a.Y = y;
  a.y_bf16 = true;
  a.status = status;
  a.T = T;
  a.after_gate_up = prof ? h->stage_events[4] : nullptr;
  a.down_ksplit = dense_down_ksplit(c, T);
  a.down_part = reinterpret_cast<float*>(ws + L.down_part);
  a.dense_T = wm ? T : 0;
  a.split_count =
      split_in_gemm ? reinterpret_cast<unsigned int*>(ws + L.status + kSplitCountOffset) : nullptr;
  if ((s = launch_expert_ffn(c, a, *dev, st))) return s;
  if ((s = mark(5))) return s;
  return mark(6);   // no combine
}

moe_status moe_dense_ffn(moe_handle h, const uint16_t* x, const uint16_t* W_gate,
                         const uint16_t* W_up, const uint16_t* W_down, int T, uint16_t* y,
                         void* workspace, size_t ws_bytes, void* stream) {
  moe_status s = check_dense_args(h, x, W_gate, W_up, W_down, T, y, workspace, ws_bytes);
  if (s || T == 0) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  const Layout L = make_layout(h->c, T, kPlanSms);
  return dense_device(h, x, W_gate, W_up, W_down, T, y, aligned_base(workspace), L, dev,
                      reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_dense_ffn_host(moe_handle h, const uint16_t* x_host, const uint16_t* W_gate,
                              const uint16_t* W_up, const uint16_t* W_down, int T,
                              uint16_t* y_host, void* workspace, size_t ws_bytes, void* stream) {
  moe_status s = check_dense_args(h, x_host, W_gate, W_up, W_down, T, y_host, workspace,
                                  ws_bytes);
  if (s || T == 0) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(h->c, T, kPlanSms);
  uint8_t* ws = aligned_base(workspace);
  const size_t bytes = size_t(T) * h->c.d * sizeof(uint16_t);
  unsigned slot;
  uint16_t* x_dev;
  if ((s = stage_host_input(h, dev, L, ws, x_host, bytes, st, &slot, &x_dev))) return s;
  uint16_t* y_dev = reinterpret_cast<uint16_t*>(ws + L.y_stage);
  if ((s = dense_device(h, x_dev, W_gate, W_up, W_down, T, y_dev, ws, L, dev, st))) return s;
  return finish_host_output(h, dev, slot, y_host, y_dev, bytes, st);
}

moe_status moe_ihc_mix(moe_handle h, const uint16_t* H, int n_streams, const float* alpha, int T,
                       uint16_t* x, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (n_streams < 1 || n_streams > kMaxStreams) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!H || !alpha || !x) return MOE_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(alpha) || !aligned16(x)) return MOE_ERR_ALIGNMENT;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  return cuda_status(
      launch_ihc_mix(h->c, H, alpha, n_streams, T, x, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_forward_ihc(moe_handle h, const uint16_t* H, int n_streams, const float* alpha,
                           const float* B, const float* gamma, const float* W_router,
                           const float* bias, const uint16_t* W_gate, const uint16_t* W_up,
                           const uint16_t* W_down, const uint16_t* Ws_gate,
                           const uint16_t* Ws_up, const uint16_t* Ws_down, int T,
                           uint16_t* H_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (n_streams < 1 || n_streams > kMaxStreams) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!H || !alpha || !B || !gamma || !H_out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(alpha) || !aligned16(B) || !aligned16(gamma) ||
      !aligned16(H_out))
    return MOE_ERR_ALIGNMENT;
  const Weights w = bf16_weights(W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down);
  // the layer input x is made by the mix below; H stands in for it in the checks
  if ((s = check_forward_args(h, H, W_router, w, T, H_out, false, workspace, ws_bytes))) return s;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(h->c, T, kPlanSms);
  uint8_t* ws = aligned_base(workspace);
  // x goes to the y staging area: the host-activation calls' helper stream writes only
  // the x staging slots, and everything on this stream is ordered
  uint16_t* x = reinterpret_cast<uint16_t*>(ws + L.y_stage);
  if ((s = cuda_status(launch_ihc_mix(h->c, H, alpha, n_streams, T, x, st)))) return s;
  const IhcArgs ihc{H, B, gamma, n_streams, H_out};
  return forward_device(h, x, W_router, bias, w, T, nullptr, ws, L, dev, st, nullptr, &ihc);
}

moe_status moe_reduce_partials(moe_handle h, const float* const* partials, int n_partials, int T,
                               uint16_t* y, void* stream) {
  if (!h || !partials || !y) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (n_partials < 1 || n_partials > kMaxPartials) return MOE_ERR_INVALID_ARG;
  PartialPtrs parts = {};
  for (int r = 0; r < n_partials; ++r) {
    if (!partials[r]) return MOE_ERR_INVALID_ARG;
    if (!aligned16(partials[r])) return MOE_ERR_ALIGNMENT;
    parts.p[r] = partials[r];
  }
  if (!aligned16(y)) return MOE_ERR_ALIGNMENT;
  if (T == 0) return MOE_OK;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  return cuda_status(launch_reduce_partials(parts, n_partials, size_t(T) * h->c.d, y,
                                            dev->num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_device_status(moe_handle h, int T, const void* workspace, void* stream,
                             int32_t* device_detail) {
  if (!h || !workspace) return MOE_ERR_INVALID_ARG;
  moe_status s = check_T(h->c, T);
  if (s) return s;
  if (device_detail) *device_detail = 0;
  DeviceInfo* dev;
  if ((s = ensure_device(&dev))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Layout L = make_layout(h->c, T, kPlanSms);
  const uint8_t* ws = aligned_base(const_cast<void*>(workspace));
  int32_t word = 0;
  if ((s = cuda_status(cudaMemcpyAsync(&word, ws + L.status, sizeof word, cudaMemcpyDeviceToHost,
                                       st))))
    return s;
  if ((s = cuda_status(cudaStreamSynchronize(st)))) return s;
  if (device_detail) *device_detail = word;
  if (word == 0) return MOE_OK;
  return (word >> 16) == kDevBadIndex ? MOE_ERR_BAD_INDEX : MOE_ERR_TIMEOUT;
}

int moe_forward_kernel_count(moe_handle h, int T) {
  if (!h || T < 0 || check_T(h->c, T) != MOE_OK) return -1;
  if (T == 0) return 0;
  const Ctx& c = h->c;
  const RouterPlan rp = router_plan(c, T, kPlanSms);
  const int router = rp.tc ? 3 : 2;  // [weight split +] score GEMM + top-k
  const int dispatch = (int64_t(T) * c.k <= kDispatchChunk && c.E <= 256) ? 1 : 3;
  const int combine = combine_fused(c, T) ? 0 : 1;
  return router + dispatch + 1 /*gather*/ + 2 /*GEMMs*/ + combine;
}

int moe_dense_ffn_kernel_count(moe_handle h, int T) {
  if (!h || T < 0 || check_T(h->c, T) != MOE_OK) return -1;
  const Ctx& c = h->c;
  if (c.E != 1 || c.k != 1 || c.S != 0) return -1;
  if (T == 0) return 0;
  if (!dense_weight_major(c, T)) return 3;   // schedule, GEMMs
  // the GEMMs [, the K ranges' sum when the kernel cannot add them itself]
  return 2 + (dense_down_ksplit(c, T) > 1 && !dense_split_summed_in_gemm(c, T) ? 1 : 0);
}

moe_status moe_set_stage_events(moe_handle h, void* const* events, int n_events) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!events || n_events == 0) {
    h->n_stage_events = 0;
    return MOE_OK;
  }
  if (n_events != MOE_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_STAGE_EVENTS; ++i) {
    if (!events[i]) return MOE_ERR_INVALID_ARG;
    h->stage_events[i] = reinterpret_cast<cudaEvent_t>(events[i]);
  }
  h->n_stage_events = MOE_STAGE_EVENTS;
  return MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or device";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "bounded device wait expired";
    case MOE_ERR_BAD_INDEX: return "expert index out of range";
    case MOE_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    default: return "unknown status";
  }
}

}  // extern "C"
