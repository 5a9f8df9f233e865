/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of one mixture-of-experts
 * FFN layer of the Hy4-preview shape.
 *
 * The layer, as the pages state it (m.xxqk.cn Hy4-preview MoE explainer,
 * section 2.1 "FFN split" and section 2.2 "router mechanism"; ZAKER Hy4 Preview
 * release news, MoE paragraph): a router scores every token against every
 * routed expert and keeps the top-k; the tokens are grouped per expert; every
 * chosen expert and every always-on shared expert runs its FFN on the token;
 * the results are merged with the gate weights into the layer output.
 * Readings where the pages are silent (applied identically by the CPU
 * oracle): softmax gate over the router logits, top-k gate values
 * renormalised to sum 1 (equal to a softmax over the k selected logits),
 * ties broken toward the lower expert index, SwiGLU experts without bias
 * y = W_down (silu(W_gate x) * (W_up x)), shared experts added with weight 1,
 * no capacity limit (dropless).
 *
 * Conventions for every call below.
 *  - Pointers named x, W_*, y, Y, topk_*, counts, offsets, perm, pos,
 *    workspace are DEVICE pointers on the current CUDA device, except where a
 *    parameter name ends in _host.  The caller allocates and owns all of
 *    them; the library keeps no pointer after a call returns.
 *  - bf16 tensors are passed as uint16_t bit patterns.  All matrices are
 *    row-major and C-contiguous.  Every device pointer must be 16-byte
 *    aligned.
 *  - stream is a cudaStream_t (NULL = the legacy default stream).  Every call
 *    is asynchronous on it: inputs must stay valid, and outputs must not be
 *    read, until the stream reaches the call.
 *  - Errors found on the host are returned before anything is enqueued.
 *    Errors found on the device (an expert index outside [0, E) given to
 *    moe_dispatch, a bounded wait inside a kernel that expired) are recorded
 *    in the workspace's status word; read it with moe_device_status().
 *    No call traps the GPU.
 *  - T == 0 is a no-op that returns MOE_OK.
 *  - Results are deterministic: the same inputs give bit-identical outputs
 *    (no floating-point atomics).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_ctx *moe_handle;
typedef int moe_status;

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1  /* null pointer, negative size, k < 1 or k > E, ...  */
#define MOE_ERR_UNSUPPORTED 2  /* shape outside the supported envelope, not sm_100  */
#define MOE_ERR_WORKSPACE 3    /* workspace too small                                */
#define MOE_ERR_CUDA 4         /* a CUDA runtime call or kernel launch failed        */
#define MOE_ERR_TIMEOUT 5      /* a bounded device wait expired (moe_device_status)  */
#define MOE_ERR_BAD_INDEX 6    /* an expert index outside [0, E) reached the device  */
#define MOE_ERR_ALIGNMENT 7    /* a device pointer is not 16-byte aligned            */

/* Device status words written into the workspace (see moe_device_status). */
#define MOE_DEVICE_OK 0

/*
 * Create a layer context.  d_model = hidden size, n_experts = E routed
 * experts, top_k = k experts per token, d_ff = F expert width, n_shared = S
 * always-on shared experts (Hy4 preview: 6144, 256, 8, 2048 assumed, 1).
 * Supported envelope: d_model and d_ff multiples of 64 in [64, 65536];
 * 1 <= E <= 1024; 1 <= k <= min(E, 32); 0 <= S <= 8.  Shapes outside it give
 * MOE_ERR_UNSUPPORTED, impossible ones MOE_ERR_INVALID_ARG.  No CUDA call is
 * made here; the device is checked (sm_100 required) at the first launch.
 * Three tuning overrides are read from the environment here, once, and fixed
 * for the context's lifetime: MOE_ROUTER=tc|ffma (router path),
 * MOE_GEMM_TILES=single|pair|swap|swap_pair (expert GEMM tiling; with FP8
 * weights any of them picks the tcgen05 kernel at every batch size --
 * swap_pair its 2-SM form, the others its 1-SM form -- where the default
 * takes the warp-MMA form up to 16 tokens) and MOE_FUSED_COMBINE=1
 * (moe_forward merges the experts'
 * rows into y inside the down GEMM kernel, after a grid-wide barrier,
 * instead of in a separate kernel; weight-major tilings only, the same
 * order of additions, so the same bits).  All choices compute the same
 * result up to the order of fp32 additions.
 */
moe_status moe_create(int d_model, int n_experts, int top_k, int d_ff, int n_shared,
                      moe_handle *out);

/* Release a context (NULL is allowed).  Does not synchronise any stream. */
moe_status moe_destroy(moe_handle h);

/*
 * Bytes of device workspace that any call below needs for T tokens
 * (0 when h is NULL or T < 0).  One workspace of this size serves every
 * call; it holds intermediates only and may be reused across calls that the
 * stream orders.  At the Hy4 shape it is about 2.3 GB at T = 8192 and about
 * 6 MB at T = 16.
 */
size_t moe_workspace_size(moe_handle h, int T);

/* Offsets (bytes from the workspace pointer) of the intermediates that
 * moe_forward leaves in the workspace, for inspection after the stream has
 * reached the call.  The workspace pointer itself need not be aligned: the
 * library aligns it up to 1024 bytes and 'base' is that adjustment's offset
 * for a pointer with the given low bits. */
typedef struct {
    size_t status;    /* int32 device status word                            */
    size_t topk_idx;  /* int32 [T][k]                                        */
    size_t topk_w;    /* fp32  [T][k]                                        */
    size_t counts;    /* int32 [E]                                           */
    size_t offsets;   /* int32 [E+1]                                         */
    size_t perm;      /* int32 [T*k]                                         */
    size_t pos;       /* int32 [T*k]                                         */
    size_t h_act;     /* bf16  [T*k + S*T][F]  SwiGLU activations            */
    size_t y_rows;    /* bf16  [T*k + S*T][d]  per-(slot, expert) outputs    */
    size_t total;     /* bytes used, including the alignment slack           */
    size_t router_partials; /* fp32 [router_ksplit][T][E] partial logits     */
    size_t router_ksplit;   /* their count; the logits are their in-order sum */
} moe_workspace_layout;
moe_status moe_get_workspace_layout(moe_handle h, int T, uintptr_t workspace_addr,
                                    moe_workspace_layout *out);

/*
 * Router: score, top-k select and gate (explainer section 2.2).
 *   logits[t][e] = sum_j x[t][j] * W_router[e][j] + bias[e]     (fp32-accurate:
 *                  on the tensor cores with W_router split exactly into three
 *                  bf16 parts and every 128-wide K chunk accumulated separately
 *                  and added in fp32 (T > 32), or with fp32 FMA on the CUDA
 *                  cores (T <= 32); MOE_ROUTER=tc|ffma in the environment when
 *                  the context is created forces one for that context; split-K
 *                  partial sums added in a fixed order)
 *   topk_idx[t][i] = the i-th largest logit's expert (ties: lower index)
 *   topk_w[t][i]   = exp(l_i - l_0) / sum_{j<k} exp(l_j - l_0)
 * x: bf16 [T][d]; W_router: fp32 [E][d]; bias: fp32 [E] or NULL;
 * topk_idx: int32 [T][k]; topk_w: fp32 [T][k] (outputs).
 */
moe_status moe_route(moe_handle h, const uint16_t *x, const float *W_router, const float *bias,
                     int T, int32_t *topk_idx, float *topk_w, void *workspace,
                     size_t ws_bytes, void *stream);

/*
 * Dispatch: group the T*k (token, choice) slots s = t*k + i by expert with a
 * stable counting sort (per-expert histogram, exclusive scan, permutation).
 *   counts[e]  = #{s : topk_idx[s] == e}                     int32 [E]
 *   offsets[e] = sum_{e' < e} counts[e'], offsets[E] = T*k   int32 [E+1]
 *   perm[p]    = slot at position p; ascending slots within each expert
 *   pos[s]     = position of slot s (perm[pos[s]] == s)      int32 [T*k] each
 * Indices outside [0, E) are skipped and flagged MOE_ERR_BAD_INDEX in the
 * workspace status word: such a slot gets pos[s] = -1 and belongs to no
 * segment, offsets[E] is then the number of valid slots (less than T*k), and
 * perm[p] for p >= offsets[E] is left unwritten.  moe_combine and
 * moe_forward leave slots with pos = -1 out of the sum.
 */
moe_status moe_dispatch(moe_handle h, const int32_t *topk_idx, int T, int32_t *counts,
                        int32_t *offsets, int32_t *perm, int32_t *pos, void *workspace,
                        size_t ws_bytes, void *stream);

/*
 * Expert FFNs (explainer section 2.1: each expert is one FFN sub-network;
 * ZAKER release news: the shared expert runs on every token).  Rows of Y:
 *   Y[p]           = FFN_e(x[perm[p] / k])  for p in expert e's segment
 *                    [offsets[e], offsets[e+1]),
 *   Y[T*k + s*T+t] = FFN_shared_s(x[t]),
 *   FFN(x) = W_down (silu(W_gate x) * (W_up x)); bf16 tensor-core GEMMs
 *   (tcgen05, fp32 accumulation), the activation rounded to bf16 before the
 *   down projection, Y in fp32.
 * W_gate, W_up: bf16 [E][F][d]; W_down: bf16 [E][d][F];
 * Ws_gate, Ws_up: bf16 [S][F][d]; Ws_down: bf16 [S][d][F] (NULL when S == 0);
 * Y: fp32 [T*k + S*T][d] (output).
 */
moe_status moe_expert_ffn(moe_handle h, const uint16_t *x, const int32_t *perm,
                          const int32_t *offsets, int T, const uint16_t *W_gate,
                          const uint16_t *W_up, const uint16_t *W_down, const uint16_t *Ws_gate,
                          const uint16_t *Ws_up, const uint16_t *Ws_down, float *Y,
                          void *workspace, size_t ws_bytes, void *stream);

/*
 * Combine (explainer section 2.2: the chosen experts' results are merged into
 * the layer output):
 *   y[t] = sum_{s<S} Y[T*k + s*T + t] + sum_{i<k} topk_w[t][i] * Y[pos[t*k+i]]
 * in fp32, in exactly that order, rounded once to bf16.
 * Y: fp32 [T*k + S*T][d]; topk_w: fp32 [T][k]; pos: int32 [T*k];
 * y: bf16 [T][d] (output).
 */
moe_status moe_combine(moe_handle h, const float *Y, const float *topk_w, const int32_t *pos,
                       int T, uint16_t *y, void *stream);

/*
 * The whole layer: moe_route, moe_dispatch, moe_expert_ffn and moe_combine
 * in one call, intermediates kept in the workspace (moe_get_workspace_layout).
 * Arguments as in those calls; y: bf16 [T][d] (output).  One difference from
 * chaining the four calls: the per-(slot, expert) rows Y are kept in bf16
 * (rounded once from the fp32 accumulator) instead of fp32, halving their
 * write and read; the combine still sums in fp32.
 */
moe_status moe_forward(moe_handle h, const uint16_t *x, const float *W_router, const float *bias,
                       const uint16_t *W_gate, const uint16_t *W_up, const uint16_t *W_down,
                       const uint16_t *Ws_gate, const uint16_t *Ws_up, const uint16_t *Ws_down,
                       int T, uint16_t *y, void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_forward with the activations in HOST memory: copies x_host (bf16
 * [T][d]) to the device, runs the layer, copies y back to y_host (bf16
 * [T][d]); returns once everything is enqueued.  y_host holds the result
 * when the stream has reached the end of the call (the caller synchronises
 * the stream before reading it).  The input copy runs on a helper stream of
 * the context (made at its first host-activation call on a device) into one
 * of two staging slots of the workspace used in turn, so it can start before
 * the stream reaches the call -- while the previous call's layer still runs;
 * x_host must therefore stay unchanged from the call until the stream has
 * passed it.  Host buffers should be page-locked for the copies to be
 * asynchronous.  Weights and the workspace are device memory as in
 * moe_forward.  Calls may run on several streams at once when each stream has
 * its own workspace and output buffer: a serving loop that alternates two
 * streams lets one call's output copy overlap the next call's layer.
 */
moe_status moe_forward_host(moe_handle h, const uint16_t *x_host, const float *W_router,
                            const float *bias, const uint16_t *W_gate, const uint16_t *W_up,
                            const uint16_t *W_down, const uint16_t *Ws_gate,
                            const uint16_t *Ws_up, const uint16_t *Ws_down, int T,
                            uint16_t *y_host, void *workspace, size_t ws_bytes, void *stream);

/*
 * FP8 expert weights.  The Hy4 pages mention an FP8 checkpoint of the model
 * (ZAKER Hy4 Preview release news; gpuvram.cloud "Tencent Hy4 preview" model
 * card) but print no scaling scheme; this library takes the OCP microscaling
 * layout.  Every expert weight is an FP8 E4M3 code (1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest
 * finite value 448), and each run of 32 consecutive K elements of a weight
 * row shares one power-of-two scale stored as a biased exponent byte e
 * (scale 2^(e - 127)).  Scales are stored K-block-major: scale[n][K/32][rows],
 * so the scales of consecutive rows for one 32-element K block are adjacent.
 * Each set holds n = E (routed) or n = S (shared) experts:
 */
typedef struct moe_fp8_expert_weights {
  const uint8_t *gate;        /* [n][F][d]    E4M3 codes          */
  const uint8_t *gate_scale;  /* [n][d/32][F] biased exponents    */
  const uint8_t *up;          /* [n][F][d]                        */
  const uint8_t *up_scale;    /* [n][d/32][F]                     */
  const uint8_t *down;        /* [n][d][F]                        */
  const uint8_t *down_scale;  /* [n][F/32][d]                     */
} moe_fp8_expert_weights;

/*
 * moe_expert_ffn with FP8 expert weights.  The GEMMs decode codes and scales
 * to bf16 and run the same bf16 tensor-core contractions (fp32 accumulation,
 * activation rounded to bf16, Y in fp32), so Y equals moe_expert_ffn's Y
 * given the decoded weights.  At up to 16 tokens (unless MOE_GEMM_TILES is
 * set) the codes are decoded in registers and multiplied by warp-level
 * m16n8k16 MMAs: the same exact bf16 x bf16 products, added in fp32 in
 * another order, so there the activations and Y equal the tcgen05 path's up
 * to that order.  The decoding is exact for
 * every finite code whose scaled value is zero or at least 2^-133 in
 * magnitude (bf16's smallest subnormal), which holds for scale bytes >= 7,
 * and for scale bytes up to 134 (scales up to 2^7, weights up to 57344 in
 * magnitude).  The E4M3 NaN codes (0x7F, 0xFF) and scale bytes above 134 are
 * outside the accepted input: they decode to unspecified values.
 * routed: the E routed experts' set (all six pointers required);
 * shared: the S shared experts' set (NULL when S == 0).  Every pointer must be
 * 16-byte aligned.  Other arguments as in moe_expert_ffn.
 */
moe_status moe_expert_ffn_fp8(moe_handle h, const uint16_t *x, const int32_t *perm,
                              const int32_t *offsets, int T, const moe_fp8_expert_weights *routed,
                              const moe_fp8_expert_weights *shared, float *Y, void *workspace,
                              size_t ws_bytes, void *stream);

/*
 * moe_forward with FP8 expert weights (as in moe_expert_ffn_fp8); the router,
 * dispatch and combine are those of moe_forward.
 */
moe_status moe_forward_fp8(moe_handle h, const uint16_t *x, const float *W_router,
                           const float *bias, const moe_fp8_expert_weights *routed,
                           const moe_fp8_expert_weights *shared, int T, uint16_t *y,
                           void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_forward_fp8 with the activations in host memory, as moe_forward_host.
 */
moe_status moe_forward_fp8_host(moe_handle h, const uint16_t *x_host, const float *W_router,
                                const float *bias, const moe_fp8_expert_weights *routed,
                                const moe_fp8_expert_weights *shared, int T, uint16_t *y_host,
                                void *workspace, size_t ws_bytes, void *stream);

/*
 * Sharded layer, for tensor parallelism over d_ff and expert parallelism.
 * The pages deploy the model on eight GPUs with vLLM's tensor-parallel
 * recipe (gpuvram.cloud "Tencent Hy4 preview" model card, hardware row: vLLM
 * TP8 on 8 x H200-class GPUs) and name vLLM's expert parallelism for MoE
 * (pgsm.cn Hy4 preview hands-on, vLLM deployment section).  Both shard the
 * expert FFNs so that each GPU computes part of every token's output y, and
 * y is the sum of the parts:
 *  - over d_ff: SwiGLU acts on each feature alone, so a GPU holding rows
 *    [f0, f1) of every W_gate and W_up and the matching columns of every
 *    W_down computes W_down[:, f0:f1] h[f0:f1] of every expert, and the sum
 *    over the slices is the layer;
 *  - over experts: a GPU holding experts [e0, e0 + n) computes the terms of
 *    the slots routed to them, and the sum over GPUs is the layer.
 *
 * moe_forward_partial runs the whole router (every routed expert scores, so
 * W_router is the full [E][d]) and computes one shard's part of y:
 *   y_partial[t] = sum_s FFN_s(x_t) + sum_{i : e0 <= idx[t][i] < e0 + n}
 *                  topk_w[t][i] * FFN_{idx[t][i]}(x_t)
 * with FFN restricted to this GPU's slice of d_ff, in fp32 and unrounded.
 * The context gives the slice: create it with d_ff = the slice's width (a
 * multiple of 64) and E, k, S of the whole layer.
 * expert_begin, n_local_experts: the routed experts this GPU holds,
 *   0 <= expert_begin, 1 <= n_local_experts, expert_begin + n_local_experts <= E;
 * W_gate, W_up: bf16 [n_local_experts][F][d] and W_down: bf16
 *   [n_local_experts][d][F] for those experts' slices (F = the context's d_ff);
 * Ws_gate, Ws_up, Ws_down: the shared experts' slices as in moe_forward, or
 *   all three NULL when this GPU computes no shared-expert term (expert
 *   parallelism: one GPU adds them; tensor parallelism: every GPU adds its
 *   slice);
 * y_partial: fp32 [T][d] (output).
 * Slots routed to experts outside the local range are skipped like an
 * out-of-range index in moe_dispatch but are not flagged.  Workspace: as
 * moe_forward with the same context.  Other arguments as in moe_forward.
 */
moe_status moe_forward_partial(moe_handle h, const uint16_t *x, const float *W_router,
                               const float *bias, int expert_begin, int n_local_experts,
                               const uint16_t *W_gate, const uint16_t *W_up,
                               const uint16_t *W_down, const uint16_t *Ws_gate,
                               const uint16_t *Ws_up, const uint16_t *Ws_down, int T,
                               float *y_partial, void *workspace, size_t ws_bytes, void *stream);

/*
 * The layer output from the shards' parts:
 *   y[t][j] = bf16( sum_{r < n_partials} partials[r][t][j] )
 * added in fp32 in the order r = 0, 1, ..., then rounded once.
 * partials: a HOST array of n_partials (1..16) device pointers, each fp32
 * [T][d] and 16-byte aligned; they may point to another GPU's memory where
 * peer access is enabled, and the caller orders their writers before this
 * call.  y: bf16 [T][d] (output); d is the context's d_model.
 */
moe_status moe_reduce_partials(moe_handle h, const float *const *partials, int n_partials, int T,
                               uint16_t *y, void *stream);

/*
 * iHC wrapper: the layer inside n parallel residual streams.  The pages'
 * model widens the residual stream to 4 parallel streams that are
 * recombined at every layer and keeps a stable identity path under the
 * learned exchange between them (ZAKER Hy4 Preview release news, iHC
 * paragraphs: identity Hyper-Connections); they give no formula.  Reading:
 *   layer input   x[t]     = sum_j alpha[j] * H[t][j]
 *   stream update H'[t][i] = H[t][i] + sum_j B[i][j] * H[t][j] + gamma[i] * y[t]
 * with y the MoE layer on x (as in moe_forward), alpha [n], B [n][n] and
 * gamma [n] the learned coefficients.  Arithmetic: fp32, in the order written
 * (identity term, exchange terms in j order, layer output); x is rounded to
 * bf16 as the layer's input, y stays in fp32 (the combine's sum) and each
 * H' element is rounded once to bf16.
 *
 * moe_ihc_mix: x only.  H: bf16 [T][n][d]; alpha: fp32 [n] (device);
 * x: bf16 [T][d] (output); 1 <= n_streams <= 8.
 */
moe_status moe_ihc_mix(moe_handle h, const uint16_t *H, int n_streams, const float *alpha, int T,
                       uint16_t *x, void *stream);

/*
 * moe_forward_ihc: the whole wrapped layer: the mix, then moe_forward on x
 * (x kept in the workspace), with the combine writing the updated streams
 * H_out instead of y (y never leaves the combine's registers).  B: fp32
 * [n][n] row-major (B[i][j] is stream j's share in stream i); gamma: fp32 [n]
 * (device pointers); H_out: bf16 [T][n][d], may be H itself.  Other
 * arguments and the workspace as in moe_forward.
 */
moe_status moe_forward_ihc(moe_handle h, const uint16_t *H, int n_streams, const float *alpha,
                           const float *B, const float *gamma, const float *W_router,
                           const float *bias, const uint16_t *W_gate, const uint16_t *W_up,
                           const uint16_t *W_down, const uint16_t *Ws_gate,
                           const uint16_t *Ws_up, const uint16_t *Ws_down, int T,
                           uint16_t *H_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * The dense FFN layer.  Of the model's 78 layers the first uses a standard
 * dense FFN and the other 77 the MoE FFN (ZAKER Hy4 Preview release news,
 * architecture paragraph); the pages give the dense layer no width.  Reading:
 * the SwiGLU form of the experts,
 *   y[t] = W_down (silu(W_gate x[t]) * (W_up x[t]))
 * which is the MoE layer with one routed expert chosen with weight 1 and no
 * shared expert, and is computed as that layer without its router, dispatch,
 * gather and combine (the expert GEMMs read x and write y directly).
 * h: a context created with n_experts = 1, top_k = 1, n_shared = 0 and the
 * dense layer's d_model and d_ff (others give MOE_ERR_INVALID_ARG);
 * x: bf16 [T][d]; W_gate, W_up: bf16 [F][d]; W_down: bf16 [d][F];
 * y: bf16 [T][d] (output); workspace: moe_workspace_size(h, T) bytes.
 * The activation is rounded to bf16 before the down projection, and the
 * output rows once from the fp32 accumulator.  At up to 128 tokens the down
 * projection's K is split into ranges whose fp32 parts are added in range
 * order (deterministic) before that rounding, so that enough SMs stream the
 * weights; the down GEMM adds them itself (d up to 8192), or a separate kernel
 * does.  The workspace's status block (its first 2 KB) holds the counters of
 * that sum and is cleared by every call.
 */
moe_status moe_dense_ffn(moe_handle h, const uint16_t *x, const uint16_t *W_gate,
                         const uint16_t *W_up, const uint16_t *W_down, int T, uint16_t *y,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * moe_dense_ffn with the activations in host memory, as moe_forward_host:
 * x_host [T][d] and y_host [T][d] bf16 in host memory (pinned for the copies
 * to be asynchronous).  The input copy runs on the same per-device helper
 * stream and the same two workspace staging slots as moe_forward_host, so a
 * call's copy overlaps the previous call's layer; the output copy runs on
 * `stream` after the layer.  y_host is complete when `stream` reaches the end
 * of the call.  Checks and errors as in moe_dense_ffn.
 */
moe_status moe_dense_ffn_host(moe_handle h, const uint16_t *x_host, const uint16_t *W_gate,
                              const uint16_t *W_up, const uint16_t *W_down, int T,
                              uint16_t *y_host, void *workspace, size_t ws_bytes, void *stream);

/*
 * Synchronise the stream and read the workspace's device status word, which
 * the last call on this workspace wrote: MOE_OK, MOE_ERR_TIMEOUT or
 * MOE_ERR_BAD_INDEX.  *device_detail receives the raw word (0 if none).
 */
moe_status moe_device_status(moe_handle h, int T, const void *workspace, void *stream,
                             int32_t *device_detail);

/*
 * Profiling hook.  With n_events == MOE_STAGE_EVENTS and events non-NULL,
 * every later moe_forward / moe_forward_host / moe_dense_ffn(_host) call on this
 * context records events[0..6] (cudaEvent_t handles the caller created) on
 * its stream at the stage boundaries: before the router, after the router,
 * after dispatch, after the gather, after the gate/up GEMM, after the down
 * GEMM, after the combine.  The elapsed time between consecutive events is
 * then the device time of one stage (moe_dense_ffn: its one-group schedule,
 * where a kernel builds it, counts as dispatch; router, gather and combine
 * are empty).  events == NULL
 * (n_events == 0) switches it off.  The
 * context keeps the handles only; the caller keeps the events alive.
 */
#define MOE_STAGE_EVENTS 7
moe_status moe_set_stage_events(moe_handle h, void *const *events, int n_events);

/*
 * moe_dispatch without a workspace, for callers that cannot allocate device
 * memory -- for example a plug-in inside a host application that owns every
 * device allocation through its own pool, or a latency-critical loop where a
 * cudaMalloc (which can synchronise the device) is not allowed.  (The pages
 * describe the layer only; they have no counterpart to this entry point.)
 * Same arguments and results as moe_dispatch, minus the workspace: the
 * scratch it needs (per-block histograms, the GEMM tile schedule, a status
 * word) lives in a fixed array of about 74 KB compiled into the library,
 * which every CUDA context that loads the library's kernels keeps until the
 * context ends (for a device's primary context: process exit or
 * cudaDeviceReset).
 * Limits: T * k <= 65536 slots and E <= 1024; larger calls return
 * MOE_ERR_WORKSPACE and enqueue nothing.  It allocates nothing: no
 * cudaMalloc / cudaFree or allocating library routine.
 * Every call looks up the array's device address in the calling thread's
 * current CUDA context (cudaGetSymbolAddress, a lookup that allocates
 * nothing), so the array used is the one of the context current at the call,
 * also under a context the host application created itself and after a
 * cudaDeviceReset.  The first call in a context also loads the library's
 * kernels into it; make that first call before any stream capture.  All
 * calls in one context share the one array and it keeps the last
 * call's contents (each call clears what must start at zero), so calls that
 * overlap on the GPU -- on different streams without ordering between them
 * -- race and corrupt each other's results.  Out-of-range expert indices are
 * skipped as in moe_dispatch (pos = -1, offsets[E] = the number of valid
 * slots), but the status word is not readable through this entry point.
 */
moe_status moe_dispatch_noalloc(moe_handle h, const int32_t *topk_idx, int T, int32_t *counts,
                                int32_t *offsets, int32_t *perm, int32_t *pos, void *stream);

/*
 * Self-test of the failure path.  Every wait inside the library's kernels is
 * bounded: when it expires the kernel records MOE_ERR_TIMEOUT in the
 * workspace's status word and returns instead of hanging.  This call runs a
 * one-CTA kernel that waits, through the same bounded wait, on a barrier that
 * nothing completes, so the wait expires after timeout_ns (1 ns .. 2 s).
 * Afterwards moe_device_status on this workspace (with any handle and
 * T >= 0 whose layout starts at the same status word -- every layout does)
 * reports MOE_ERR_TIMEOUT, and the device stays usable.  workspace: at least
 * 1028 bytes of device memory.  Asynchronous on the stream.
 */
moe_status moe_selftest_wait_timeout(void *workspace, size_t ws_bytes,
                                     unsigned long long timeout_ns, void *stream);

/* Number of kernels one moe_forward call with T tokens launches (for launch
 * accounting), or -1 for invalid arguments. */
int moe_forward_kernel_count(moe_handle h, int T);

/* Number of kernels one moe_dense_ffn call with T tokens launches, or -1 for
 * invalid arguments (including a context that is not the dense E=1, k=1, S=0
 * layer). */
int moe_dense_ffn_kernel_count(moe_handle h, int T);

/* Static text for a status code. */
const char *moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
