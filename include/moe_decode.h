/*
 * moe_decode.h -- C ABI of libmoe_decode.so: the batch-1 MXFP4 mixture-of-experts
 * decode step on NVIDIA B200 (sm_100a).
 *
 * What is computed (sources):
 *  - "知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的三种方法" (DGX Spark MoE
 *    knowledge card), section 事件概述或研究问题 ("overview"): decode at batch 1 is
 *    bound by reading weights, the MoE and the LM head dominate; every MoE layer
 *    routes a token to 8 of 512 routed experts plus 1 shared expert.
 *  - same card, section 方法/产品要点 ("methods"), item 1: the routed experts are
 *    MXFP4 with moe_intermediate_size = 768; item 2: the LM head (vocabulary GEMM
 *    157,184 x 2,560, BF16 in the checkpoint) is quantised online to FP8 when the
 *    head is built, halving its bytes; item 3: a 4-token verify window can fire up
 *    to 32 distinct experts.
 *  - "英伟达称不换芯片也能提速：DGX Spark靠软件优化多吐42.5%的token", section
 *    不换卡，快在哪: the three optimisations and the 157,184 x 2,560 output layer.
 *  Formats: OCP Microscaling (MX) v1.0 -- MXFP4 = FP4 E2M1 codes with one E8M0
 *  scale 2^(e-127) per 32 consecutive elements; FP8 E4M3 (bias 7, max 448).
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers (cudaMalloc'd or equivalent) unless
 *    stated; the caller owns every buffer.  The library never allocates, frees or
 *    synchronises (moe_workspace_status and moe_selfcheck excepted, as they say);
 *    every other call is asynchronous and ordered on `stream`.
 *  - Arguments are validated on the host before anything is enqueued; a non-OK
 *    status means nothing was launched.  No C++ exception crosses the ABI.
 *  - Pointers must be 16-byte aligned (MOE_ERR_ALIGNMENT otherwise).
 *  - Layouts are row-major, "[out][in]" for weights (the Linear convention).
 *    BF16 tensors are raw uint16 bit patterns.  MXFP4 codes: two per byte along
 *    the input dimension, element 2j in the LOW nibble of byte j; the scale byte
 *    b of a row covers input elements [32b, 32b+32).  E2M1 bit 3 = sign, bits 2..1
 *    exponent (bias 1), bit 0 mantissa.
 *  - W13 stacks the gate projection (rows [0, I)) over the up projection (rows
 *    [I, 2I)); SwiGLU a = silu(gate) * up, kept in fp32.
 *  - Routing: l = x . Wr^T in fp32; the top_k largest logits (ties to the lower
 *    expert index); weights = softmax over the selected logits (= the softmax
 *    over all experts renormalised over the selected).
 *  - Workspaces are caller-owned scratch of at least the *_workspace_bytes()
 *    size; their contents on entry do not matter and are clobbered.
 *  - A CUDA error while enqueuing returns MOE_ERR_CUDA; moe_last_cuda_error()
 *    then gives the cudaError_t value (per calling thread).
 *  - Thread safety: stateless apart from the caller's buffers and the per-thread
 *    last-error value; concurrent calls on different workspaces are safe.
 *  - Contexts: the first call on a device reads its attributes and raises the
 *    kernels' shared-memory limits once, for the process; this assumes every call
 *    runs in the device's primary context (the CUDA runtime's).  After
 *    cudaDeviceReset those limits are gone and large launches fail (MOE_ERR_CUDA):
 *    reload the library in a new process instead.
 */
#ifndef MOE_DECODE_H
#define MOE_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Layout-compatible with cudaStream_t / CUstream; NULL = the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* NULL where a buffer is required, negative size, ... */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside the limits listed per entry point */
  MOE_ERR_ALIGNMENT = 3,         /* a pointer not 16-byte aligned */
  MOE_ERR_WORKSPACE = 4,         /* workspace NULL or smaller than required */
  MOE_ERR_DTYPE = 5,             /* a model buffer tagged with the wrong format */
  MOE_ERR_CUDA = 6,              /* the CUDA runtime refused a launch */
  MOE_ERR_TIMEOUT = 7,           /* a bounded device-side wait gave up */
  MOE_ERR_SELFCHECK = 8          /* moe_selfcheck: a result differs from the expected one */
} moe_status_t;

/* Human-readable name of a status value (static storage). */
MOE_API const char* moe_status_string(int status);
/* ABI version of this header: MOE_ABI_VERSION. */
#define MOE_ABI_VERSION 2
MOE_API int moe_abi_version(void);
/* cudaError_t of the last MOE_ERR_CUDA returned on the calling thread (0 if none). */
MOE_API int moe_last_cuda_error(void);
/* Device-side status of the last call that used workspace `ws`: synchronises
 * `stream`, then reads the status word every call clears on entry.  MOE_OK, or
 * MOE_ERR_TIMEOUT when a bounded device wait gave up (the kernel returned early
 * instead of hanging; its outputs are then incomplete).  Host-blocking: meant for
 * checks and tests, not for the hot path. */
MOE_API moe_status_t moe_workspace_status(const void* ws, moe_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Router (knowledge card, overview: 8 of 512 routed experts per token)       */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace moe_route needs for M tokens and E experts. */
MOE_API size_t moe_route_workspace_bytes(int M, int E);

/* Router logits, top-k selection and renormalised weights for M tokens.
 *   x_bf16        [M][H]  bf16 activations
 *   w_router_bf16 [E][H]  bf16 router weight
 *   topk_ids      [M][top_k] int32 out: selected experts, descending logit,
 *                 ties broken toward the lower index
 *   topk_w        [M][top_k] fp32 out: softmax over the selected logits (sums to 1)
 *   logits_opt    [M][E] fp32 out, or NULL
 * Limits: 1 <= M <= 8; H % 64 == 0, 64 <= H <= 4096; E % 16 == 0, 16 <= E <= 1024;
 *         1 <= top_k <= min(8, E). */
MOE_API moe_status_t moe_route(const void* x_bf16, int M, int H, const void* w_router_bf16, int E,
                       int top_k, int32_t* topk_ids, float* topk_w, float* logits_opt,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Routed MXFP4 experts + BF16 shared expert (knowledge card, methods item 1)  */
/* ------------------------------------------------------------------------- */

/* Bytes of workspace moe_mxfp4_experts needs (0 for an unsupported shape). */
MOE_API size_t moe_experts_workspace_bytes(int M, int H, int I, int E, int top_k, int Is);

/* One MoE layer for M tokens under a given routing:
 *   y[t] = sum_j topk_w[t][j] * W2_e (silu(Wg_e x_t) * Wu_e x_t),  e = topk_ids[t][j]
 *        + Ws2 (silu(Wsg x_t) * Wsu x_t)                  (when the shared expert is given)
 *   x_bf16       [M][H] bf16
 *   topk_ids     [M][top_k] int32 expert ids in [0, E)   (device)
 *   topk_w       [M][top_k] fp32 weights                  (device)
 *   w13_codes    [E][2I][H/2]  u8   MXFP4 codes of gate (rows < I) and up (rows >= I)
 *   w13_scales   [E][2I][H/32] u8   E8M0
 *   w2_codes     [E][H][I/2]   u8
 *   w2_scales    [E][H][I/32]  u8
 *   shared_w13_bf16 [2Is][H] bf16 (gate rows then up rows) and shared_w2_bf16 [H][Is]
 *                 bf16, both NULL (with Is = 0) when the layer has no shared expert
 *   y            [M][H] fp32 out (overwritten)
 * Every distinct expert among the M*top_k selections is streamed from HBM once
 * per call, whatever the number of tokens that chose it.  Activations stay BF16
 * (the products are formed exactly and accumulated in fp32).
 * Ids outside [0, E) contribute nothing (they are dropped on the device, never read
 * out of bounds).  A token listing the same expert twice gives it both weights.
 * Limits: 1 <= M <= 8 (decode / verify windows); H % 64 == 0, 64 <= H <= 4096;
 *         I % 32 == 0, 32 <= I <= 1024; Is % 32 == 0, 0 <= Is <= 1024;
 *         E % 16 == 0, 16 <= E <= 1024; 1 <= top_k <= min(8, E).
 * A chunk -- M a multiple of 128, 128 <= M <= 16384 -- takes the prefill chunk's
 * block-scaled tcgen05 path under the given routing instead: the activations x and
 * silu(g)*u are quantised to MXFP8 (E4M3 with an E8M0 scale per 32: scale exponent
 * floor(log2 amax) - 8, clamped to [-127, 127]) before the E2M1 x E4M3 products; shapes
 * as moe_prefill_layer (H, I multiples of 128 up to 4096; E a multiple of 128 up to 512;
 * Is a multiple of 64), w13_codes and w2_codes 32-byte aligned, workspace from
 * moe_experts_workspace_bytes with the same M. */
MOE_API moe_status_t moe_mxfp4_experts(const void* x_bf16, int M, int H, int I, int E, int top_k,
                               const int32_t* topk_ids, const float* topk_w,
                               const uint8_t* w13_codes, const uint8_t* w13_scales,
                               const uint8_t* w2_codes, const uint8_t* w2_scales,
                               const void* shared_w13_bf16, const void* shared_w2_bf16, int Is,
                               float* y, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ------------------------------------------------------------------------- */
/* FP8 LM head (knowledge card, methods item 2; retelling, 不换卡，快在哪)        */
/* ------------------------------------------------------------------------- */

/* Online FP8 quantisation of a BF16 LM head, done once when the head is built:
 *   amax_v = max_h |W[v][h]|;  s_v = amax_v / 448 (fp32 division; 1.0 if amax_v == 0)
 *   w_e4m3[v][h] = e4m3 round-to-nearest-even of W[v][h] / s_v (fp32 division),
 *                  saturating at +-448.
 *   w_bf16 [V][H] bf16 in; w_e4m3 [V][H] u8 out; row_scale [V] fp32 out.
 * Limits: 1 <= V; H % 16 == 0, 16 <= H <= 16384. */
MOE_API moe_status_t lm_head_fp8_quantize(const void* w_bf16, int V, int H, uint8_t* w_e4m3,
                                  float* row_scale, moe_stream_t stream);

/* Bytes of workspace lm_head_fp8_gemv needs. */
MOE_API size_t lm_head_workspace_bytes(int M, int V, int H);

/* logits[t][v] = row_scale[v] * sum_h e4m3(w_e4m3[v][h]) * x[t][h]  (fp32 accumulation)
 * argmax[t]    = the index of the largest logit of row t, lowest index on ties.
 *   x_bf16 [M][H] bf16; logits [M][V] fp32 out (may be NULL: argmax only);
 *   argmax [M] int32 out.
 * Limits: 1 <= M <= 8; 1 <= V <= 2^26; H % 64 == 0, 64 <= H <= 2560. */
MOE_API moe_status_t lm_head_fp8_gemv(const void* x_bf16, int M, int V, int H, const uint8_t* w_e4m3,
                              const float* row_scale, float* logits, int32_t* argmax,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/* Verify window of multi-token prediction, fused into the head's argmax tail (source:
 * the DGX Spark MoE knowledge card, 方法/产品要点 item 2 -- the window of the last
 * accepted token and M-1 draft tokens goes through the step at once).  As
 * lm_head_fp8_gemv for the M window positions, then draft t+1 is accepted while it
 * equals argmax[t], and argmax at the first mismatch (or after the last draft) is
 * accepted too:
 *   drafts [M-1] int32 in; accept [1+M] int32 out: accept[0] = accepted count (1..M),
 *   accept[1..count] = the accepted tokens.  2 <= M <= 8; other limits as the GEMV. */
MOE_API moe_status_t lm_head_fp8_verify(const void* x_bf16, int M, int V, int H, const uint8_t* w_e4m3,
                                        const float* row_scale, const int32_t* drafts, float* logits,
                                        int32_t* argmax, int32_t* accept, void* ws, size_t ws_bytes,
                                        moe_stream_t stream);

/* The same head on the BF16 weights it is quantised from (the comparison the FP8
 * head halves the bytes against; same knowledge card, 方法/产品要点 item 2):
 *   logits[t][v] = sum_h w_bf16[v][h] * x[t][h] (fp32 accumulation), argmax as above.
 *   w_bf16 [V][H] bf16; workspace as lm_head_workspace_bytes; limits as the FP8 GEMV. */
MOE_API moe_status_t lm_head_bf16_gemv(const void* x_bf16, int M, int V, int H, const void* w_bf16,
                                       float* logits, int32_t* argmax, void* ws, size_t ws_bytes,
                                       moe_stream_t stream);

/* Sampling of one token per row of fp32 logits [M][V] (the knowledge card's serving
 * settings: temperature, top-k 29, top-p 0.95), the uniform draw u [M] in [0,1) given:
 * z = logits / T over the top_k largest logits (ties to the lower index), p = softmax
 * of z, nucleus = the shortest prefix (in that order) with sum p >= top_p, sample =
 * the first nucleus token whose cumulative p / sum_nucleus p exceeds u.
 *   ids [M] int32 out.  1 <= top_k <= 32 (and <= V); T > 0; 0 < top_p <= 1.
 *   At most 1024 logits may tie at or above the top_k-th value. */
MOE_API moe_status_t moe_sample(const float* logits, int M, int V, float temperature, int top_k, float top_p,
                                const float* u, int32_t* ids, moe_stream_t stream);

/* Start-up self-check (the DGX Spark MoE knowledge card, 局限与不确定性: with the FP8
 * head and the verify window both on, a module mismatch made the framework fall back
 * silently -- FP8 bytes read as BF16, accept length 1.00 -- visible in no throughput
 * figure, and the advice is to confirm at start-up that every optimisation is really
 * active).  On inputs it generates in `ws` from a counter-based generator, runs
 *   1 moe_route on one token (expert ids compared bit for bit),
 *   2 moe_mxfp4_experts on that routing (y: relative L2 <= 5e-3),
 *   3 lm_head_fp8_gemv on a 4-token window (argmaxes bit for bit),
 *   4 lm_head_fp8_verify with the head's own argmaxes as drafts (accept length 4),
 *   5 decode_step, two layers, one token, and 6 the same on the 4-token window
 *     (argmaxes bit for bit, logits relative L2 <= 5e-3 per row),
 *   7 whether decode_step took its single persistent kernel at M = 1 and M = 4,
 * against results computed once by the CPU oracle and compiled into the library.
 *   ws: device workspace of moe_selfcheck_workspace_bytes() bytes, 16-byte aligned.
 *   failed_check (HOST, may be NULL): 0, or the number of the first check that failed.
 *   max_rel_l2 (HOST, may be NULL): the largest relative L2 seen in checks 2, 5, 6.
 * Returns MOE_OK, MOE_ERR_SELFCHECK when a check failed, or the error of the entry
 * point that refused (MOE_ERR_TIMEOUT included).  Synchronises `stream` (host-blocking):
 * call it once at start-up, not in the decode loop. */
MOE_API size_t moe_selfcheck_workspace_bytes(void);
MOE_API moe_status_t moe_selfcheck(void* ws, size_t ws_bytes, moe_stream_t stream, int* failed_check,
                                   float* max_rel_l2);

/* Allocation-free variant of lm_head_fp8_gemv (no counterpart on the pages; it
 * exists for integration).  Some callers cannot hand this library any scratch
 * memory: an operator slot that passes only input and output tensors and has no
 * workspace argument, a runtime whose device memory is fixed at start-up and may
 * not grow, or code that must not call cudaMalloc because it synchronises the
 * device.  This entry point takes inputs and outputs only and allocates nothing;
 * the 256-byte control block the GEMV needs (argmax keys of up to 8 tokens, a
 * completion counter, the status word) is a static device array inside the library,
 * one per device that loads it, held until the process exits.
 *   Arguments, layouts, results and errors: as lm_head_fp8_gemv.  M above 8 (the
 *   keys the static block holds) returns MOE_ERR_UNSUPPORTED_SHAPE.
 *   Each call looks up the array's device address in the current context (host-side,
 *   no device work); the first call in a process may load the module, so make it
 *   before any stream capture.
 *   Every call shares the one array and clears it on entry, so calls whose GPU
 *   work overlaps (other streams, other host threads, the same device) race and
 *   corrupt each other's argmax; serialise them. */
MOE_API moe_status_t lm_head_fp8_gemv_noalloc(const void* x_bf16, int M, int V, int H,
                                              const uint8_t* w_e4m3, const float* row_scale,
                                              float* logits, int32_t* argmax, moe_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Whole decode step: L MoE layers + FP8 LM head                              */
/* ------------------------------------------------------------------------- */

/* Format tags carried by every model buffer, checked by decode_step.  A buffer
 * whose tag disagrees with its role is rejected (MOE_ERR_DTYPE) instead of being
 * silently reinterpreted -- e.g. FP8 LM-head bytes read as BF16. */
enum {
  MOE_FMT_NONE = 0,
  MOE_FMT_BF16 = 1,
  MOE_FMT_MXFP4_CODES = 2,
  MOE_FMT_E8M0_SCALES = 3,
  MOE_FMT_E4M3 = 4,
  MOE_FMT_F32 = 5
};

typedef struct {
  const void* ptr; /* device pointer */
  int fmt;         /* MOE_FMT_* */
} moe_buf_t;

typedef struct {
  moe_buf_t router;      /* [E][H]   bf16 */
  moe_buf_t w13_codes;   /* [E][2I][H/2]  MXFP4 codes */
  moe_buf_t w13_scales;  /* [E][2I][H/32] E8M0 */
  moe_buf_t w2_codes;    /* [E][H][I/2]   MXFP4 codes */
  moe_buf_t w2_scales;   /* [E][H][I/32]  E8M0 */
  moe_buf_t shared_w13;  /* [2Is][H] bf16, or ptr NULL when Is == 0 */
  moe_buf_t shared_w2;   /* [H][Is]  bf16, or ptr NULL when Is == 0 */
} moe_layer_t;

typedef struct {
  int n_layers;               /* L >= 1 */
  int H, I, E, top_k, Is, V;  /* shapes shared by all layers (limits as above) */
  float rms_eps;              /* RMSNorm epsilon of the layer-chaining stand-in (1e-6) */
  const moe_layer_t* layers;  /* HOST array of n_layers entries */
  moe_buf_t lm_head;          /* [V][H] e4m3 codes (from lm_head_fp8_quantize) */
  moe_buf_t lm_scale;         /* [V] fp32 row scales */
  int step_path;              /* MOE_STEP_AUTO or MOE_STEP_PER_LAYER */
} moe_model_t;

/* How decode_step runs the layers.  AUTO: one persistent kernel for all layers
 * (cooperative launch, one block per SM) followed by the LM-head kernel, when the
 * model fits it (n_layers <= 64, H % 128 == 0); otherwise three kernels per layer.
 * PER_LAYER: always three kernels per layer (router + shared W13, routed W13,
 * W2 + combine), a final RMSNorm kernel and the LM head. */
enum { MOE_STEP_AUTO = 0, MOE_STEP_PER_LAYER = 1 };

/* Optional debug trace of a decode step (device buffers, any may be NULL):
 *   x  [L+1][M][H] bf16: each layer's input and the LM head's input
 *   h  [L+1][M][H] fp32: the residual stream entering each layer, and the final one
 *   ids [L][M][top_k] int32, w [L][M][top_k] fp32: each layer's routing
 *   events: NULL or an array of n_events cudaEvent_t handles (host array, created by
 *     the caller) recorded on the step's stream around every kernel: events[2i] before
 *     and events[2i+1] after launch i, in the order decode_step_launch_names gives: the
 *     persistent kernel then the LM head (2 launches), or on the per-layer path (router +
 *     shared W13, routed W13, W2 + combine) per layer, the final RMSNorm and the LM head
 *     (3L+2 launches).  Fewer events than 2 x (launch count) record the first
 *     n_events/2 launches only.
 *   timeline: NULL or [2*L*16 + 4*4096 + G*L*16] uint64 %globaltimer stamps (ns), G the
 *     device's SM count, for profiling the persistent path: [2][L][16] phase boundaries of
 *     blocks 0 and G-1, then block 0's first 2048 weight items, 8 stamps each (window
 *     acquired, data ready, done, wait started, producer entered, copies issued, 2 unused),
 *     then [G][L][16] phase ends of every block (residual seen, input staged, router item
 *     published, router/shared-W13 items done, plan built, shared W2 done, routed W13
 *     done, routed W2 done, then finer marks inside the top-k and data arrivals).
 *   wait_limit_ns: 0, or a shorter limit for every bounded device wait of the step (the
 *     default is 2 s): for testing the timeout path only.
 *   hold_layer: 0, or l + 1 to make the persistent step never publish layer l's residual,
 *     so the next wait on it can only time out: with a short wait_limit_ns this drives
 *     the step's timeout path (MOE_ERR_TIMEOUT from moe_workspace_status; the kernels
 *     return early, every output is then undefined).  Ignored on the per-layer path. */
typedef struct {
  void* x;
  float* h;
  int32_t* ids;
  float* w;
  void** events;
  int n_events;
  unsigned long long* timeline;
  unsigned long long wait_limit_ns;
  int hold_layer;
} moe_trace_t;

MOE_API size_t decode_step_workspace_bytes(const moe_model_t* model, int M);

/* The kernels one decode_step call launches, in order (the order of the trace's
 * event pairs): writes up to max_names static name strings into names (may be NULL)
 * and returns the count, or -1 for an invalid model / M.  Needs the CUDA device
 * (the choice of path depends on it). */
MOE_API int decode_step_launch_names(const moe_model_t* model, int M, const char** names, int max_names);

/* One decode step for an M-token window (M = 1 decode, M = 4 verify window):
 *   h_0 = fp32(x);  for l < L:  x_l = (l == 0 ? x : bf16(RMSNorm(h_l))),
 *                               h_{l+1} = h_l + MoE_l(x_l)       (route + experts + shared)
 *   x_L = bf16(RMSNorm(h_L));   logits = FP8 LM head(x_L);  argmax per row.
 * RMSNorm has unit weight: h / sqrt(mean(h^2) + rms_eps).  It stands in for the
 * attention blocks between MoE layers, which are not part of this library.
 *   model  HOST pointer; its buffers are device pointers with format tags
 *   x_bf16 [M][H] bf16; logits [M][V] fp32 out (may be NULL); argmax [M] int32 out
 *   trace_opt HOST pointer or NULL.
 * Limits: as moe_mxfp4_experts (1 <= M <= 8) and lm_head_fp8_gemv (H <= 2560). */
MOE_API moe_status_t decode_step(const moe_model_t* model, const void* x_bf16, int M, float* logits,
                         int32_t* argmax, const moe_trace_t* trace_opt, void* ws,
                         size_t ws_bytes, moe_stream_t stream);

/* A whole decode step captured once as a CUDA graph (the workspace clear and the
 * step's kernels: 2 on the persistent path, 3L+2 on the per-layer one), replayed with
 * a single launch.  The graph binds the given x, logits, argmax and
 * workspace pointers: refill x in place between launches.  The handle is a small
 * host object owned by the caller (decode_step_graph_destroy); no device memory is
 * allocated.  The model's buffers must stay valid while the handle lives. */
typedef struct moe_graph_s* moe_graph_t;
MOE_API moe_status_t decode_step_graph_create(const moe_model_t* model, const void* x_bf16, int M, float* logits,
                                      int32_t* argmax, const moe_trace_t* trace_opt, void* ws,
                                      size_t ws_bytes, moe_graph_t* out);
MOE_API moe_status_t decode_step_graph_launch(moe_graph_t graph, moe_stream_t stream);
MOE_API void decode_step_graph_destroy(moe_graph_t graph);

/* ---------------------------------------------------------------------------
 * Prefill chunk: one MoE layer for M tokens on the block-scaled tensor cores.
 * Source: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
 * 三种方法), 方法/产品要点 items 1 and 3: MXFP4 expert weights, 8 of 512 routed experts
 * plus one shared BF16 expert.  The pages fix no prefill activation format; the
 * block-scaled MMA needs MX operands on both sides, so the routed experts take
 * their activations as MXFP8 (per token, per 32 elements of K: s = clamp(floor(log2
 * amax) - 8, -127, 127), codes e4m3 RNE-saturating of v * 2^-s; amax = 0 gives
 * s = -127 and zero codes) -- both x and the SwiGLU output a.  Router and shared
 * expert run on BF16 operands with fp32 accumulation; the shared activation is
 * rounded to BF16.
 * ------------------------------------------------------------------------- */

/* Bytes of workspace moe_prefill_layer needs (0: unsupported shape). */
MOE_API size_t moe_prefill_workspace_bytes(int M, int H, int I, int E, int top_k, int Is);

/* y[t] = sum_j w[t][j] * W2_e (MXFP8(silu(Wg_e xq) * Wu_e xq)) + Ws2 bf16(silu(Wsg x) * Wsu x),
 * e = ids[t][j], xq = MXFP8(x[t]); ids/w = top-k of the router logits x Wr^T (largest,
 * lowest index on ties) and the softmax over the k selected logits.
 *   x_bf16 [M][H] bf16; w_router_bf16 [E][H]; w13_codes [E][2I][H/2] MXFP4 (rows 0..I-1
 *   gate, I..2I-1 up; low nibble = even element), w13_scales [E][2I][H/32] E8M0;
 *   w2_codes [E][H][I/2], w2_scales [E][H][I/32]; shared_w13_bf16 [2Is][H],
 *   shared_w2_bf16 [H][Is] (both NULL when Is == 0);
 *   topk_ids_opt [M][k] int32, topk_w_opt [M][k] fp32, logits_opt [M][E] fp32: optional
 *   outputs (NULL: not written); y [M][H] fp32 out (overwritten).
 * Limits: M % 128 == 0, 128 <= M <= 16384; H, I multiples of 128 in [128, 4096];
 *   E % 128 == 0, 128 <= E <= 512; 1 <= top_k <= 8; Is % 64 == 0, 0 <= Is <= 4096.
 * Pointers 16-byte aligned; w13_codes and w2_codes 32-byte aligned (MOE_ERR_ALIGNMENT).
 * Asynchronous on `stream`; device-side bounded waits report MOE_ERR_TIMEOUT through
 * moe_workspace_status.  Caller owns every buffer; nothing is allocated. */
MOE_API moe_status_t moe_prefill_layer(const void* x_bf16, int M, int H, int I, int E, int top_k,
                                       const void* w_router_bf16, const uint8_t* w13_codes,
                                       const uint8_t* w13_scales, const uint8_t* w2_codes,
                                       const uint8_t* w2_scales, const void* shared_w13_bf16,
                                       const void* shared_w2_bf16, int Is, int32_t* topk_ids_opt,
                                       float* topk_w_opt, float* logits_opt, float* y, void* ws,
                                       size_t ws_bytes, moe_stream_t stream);

/* MXFP8 quantiser of the prefill path on its own: v [M][K] fp32 -> q [M][K] e4m3 codes,
 * scales [M][K/32] E8M0, by the rule above.  K % 32 == 0; M * K <= 2^31. */
MOE_API moe_status_t moe_mxfp8_quantize(const float* v, int M, int K, uint8_t* q, uint8_t* scales,
                                        moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H */
