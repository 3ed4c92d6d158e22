// api.cu -- the C ABI of libmoe_decode.so (declared in include/moe_decode.h).
//
// Host side only: argument validation (before anything is enqueued), workspace
// carving, launch configuration (one block per SM for the streamed kernels,
// shared-memory stage counts from the device's opt-in limit) and the per-layer
// launch sequence of the decode step.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/moe_decode.h"
#include "decode_kernels.cuh"
#include "lmhead_kernels.cuh"
#include "step_kernel.cuh"
#include "prefill_kernels.cuh"
#include "sample_kernels.cuh"
#include "selfcheck.cuh"

using namespace moe;

namespace {

thread_local int g_last_cuda_error = 0;

moe_status_t cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return MOE_ERR_CUDA;
}

#define MOE_CUDA(call)                          \
  do {                                          \
    cudaError_t e_ = (call);                    \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t b) { return (b + 255) / 256 * 256; }

struct DevInfo {
  int sms = 0;
  int smem_optin = 0;
  // largest dynamic shared memory per kernel family: the opt-in limit minus the
  // kernel's own static shared memory
  int dyn_dense = 0, dyn_e13 = 0, dyn_e2 = 0, dyn_lm = 0, dyn_lmb = 0, dyn_step = 0, dyn_pf = 0;
  int coop = 0;
};

template <class K>
cudaError_t allow_dyn_smem(K kernel, int optin, int* dyn) {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return e;
  const int lim = optin - static_cast<int>(a.sharedSizeBytes);
  *dyn = (*dyn == 0 || lim < *dyn) ? lim : *dyn;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
}

// Per-device launch facts and one-time kernel attributes (opt-in shared memory).
moe_status_t dev_info(DevInfo* out) {
  static std::mutex mu;
  static DevInfo cache[64];
  static bool ready[64] = {};
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (!ready[dev]) {
    DevInfo d;
    MOE_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    MOE_CUDA(cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    const int lim = d.smem_optin;
    MOE_CUDA(allow_dyn_smem(k_dense, lim, &d.dyn_dense));
    MOE_CUDA(allow_dyn_smem(k_experts13, lim, &d.dyn_e13));
    MOE_CUDA(allow_dyn_smem(k_experts2, lim, &d.dyn_e2));
    MOE_CUDA(allow_dyn_smem(k_lm_gemv, lim, &d.dyn_lm));
    MOE_CUDA(allow_dyn_smem(k_lm_gemv_bf16, lim, &d.dyn_lmb));
    MOE_CUDA(allow_dyn_smem(k_step<false, false>, lim, &d.dyn_step));
    MOE_CUDA(allow_dyn_smem(k_step<true, false>, lim, &d.dyn_step));
    MOE_CUDA(allow_dyn_smem(k_step<false, true>, lim, &d.dyn_step));
    MOE_CUDA(allow_dyn_smem(k_step<true, true>, lim, &d.dyn_step));
    MOE_CUDA(allow_dyn_smem(k_umma<PF_ROUTER>, lim, &d.dyn_pf));
    MOE_CUDA(allow_dyn_smem(k_umma<PF_SH13>, lim, &d.dyn_pf));
    MOE_CUDA(allow_dyn_smem(k_umma<PF_SH2>, lim, &d.dyn_pf));
    MOE_CUDA(allow_dyn_smem(k_umma<PF_R13>, lim, &d.dyn_pf));
    MOE_CUDA(allow_dyn_smem(k_umma<PF_R2>, lim, &d.dyn_pf));
    MOE_CUDA(cudaDeviceGetAttribute(&d.coop, cudaDevAttrCooperativeLaunch, dev));
    cache[dev] = d;
    ready[dev] = true;
  }
  *out = cache[dev];
  return MOE_OK;
}

// ---- shape checks -----------------------------------------------------------
bool ok_M(int M) { return M >= 1 && M <= MAX_M; }
bool ok_H(int H) { return H >= 64 && H <= 4096 && H % 64 == 0; }
bool ok_I(int I) { return I >= 32 && I <= 1024 && I % 32 == 0; }
bool ok_Is(int Is) { return Is >= 0 && Is <= 1024 && Is % 32 == 0; }
bool ok_E(int E) { return E >= 16 && E <= 1024 && E % 16 == 0; }
bool ok_k(int k, int E) { return k >= 1 && k <= 8 && k <= E; }
bool ok_H_lm(int H) { return H >= 64 && H <= 2560 && H % 64 == 0; }

// ---- workspace layouts ------------------------------------------------------
constexpr size_t CTRL_BYTES = 256;  // status (int @0), counters (@4, @8), argmax keys (@64)

struct Ctrl {
  int* status;
  unsigned* route_counter;
  unsigned* lm_counter;
  unsigned long long* keys;
};
Ctrl ctrl_of(void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  return Ctrl{reinterpret_cast<int*>(b), reinterpret_cast<unsigned*>(b + 4), reinterpret_cast<unsigned*>(b + 8),
              reinterpret_cast<unsigned long long*>(b + 64)};
}

size_t slots_of(int M, int E, int k) { return static_cast<size_t>(M * k < E ? M * k : E); }

struct ExpertsWs {
  float* a_shared;
  float* a_routed;
  size_t bytes;
};
ExpertsWs experts_ws(void* ws, int M, int H, int I, int E, int k, int Is) {
  (void)H;
  size_t off = CTRL_BYTES;
  ExpertsWs w{};
  uint8_t* b = static_cast<uint8_t*>(ws);
  w.a_shared = reinterpret_cast<float*>(b + off);
  off += up256((size_t)M * Is * 4);
  w.a_routed = reinterpret_cast<float*>(b + off);
  off += up256(slots_of(M, E, k) * M * I * 4);
  w.bytes = off;
  return w;
}

struct StepWs {
  unsigned* ctr;
  unsigned long long* tlogits;  // persistent step: tagged router logits [M][E]
  unsigned long long* tshared;  // persistent step: tagged shared activation [M][Is]
  size_t ctrl_bytes;  // control block, per-layer counters and the tagged buffers, cleared every step
  float* logits;
  int32_t* ids;
  float* w;
  __nv_bfloat16* x_cur;
  float* h;
  float* a_shared;
  float* a_routed;
  __nv_bfloat16* x_final;
  size_t bytes;
};
StepWs step_ws(void* ws, int L, int M, int H, int I, int E, int k, int Is) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  size_t off = CTRL_BYTES;
  StepWs s{};
  s.ctr = reinterpret_cast<unsigned*>(b + off);
  off += up256((size_t)L * CTR_PER_LAYER * sizeof(unsigned));
  s.tlogits = reinterpret_cast<unsigned long long*>(b + off);
  off += up256((size_t)M * E * 8);
  s.tshared = reinterpret_cast<unsigned long long*>(b + off);
  off += up256((size_t)M * Is * 8);
  s.ctrl_bytes = off;
  s.logits = reinterpret_cast<float*>(b + off);
  off += up256((size_t)M * E * 4);
  s.ids = reinterpret_cast<int32_t*>(b + off);
  off += up256((size_t)M * k * 4);
  s.w = reinterpret_cast<float*>(b + off);
  off += up256((size_t)M * k * 4);
  s.x_cur = reinterpret_cast<__nv_bfloat16*>(b + off);
  off += up256((size_t)M * H * 2);
  s.h = reinterpret_cast<float*>(b + off);  // [2][M][H]: the persistent step alternates by layer
  off += up256((size_t)2 * M * H * 4);
  s.a_shared = reinterpret_cast<float*>(b + off);
  off += up256((size_t)M * Is * 4);
  s.a_routed = reinterpret_cast<float*>(b + off);
  off += up256((size_t)MAX_SLOTS * M * I * 4);
  s.x_final = reinterpret_cast<__nv_bfloat16*>(b + off);
  off += up256((size_t)M * H * 2);
  s.bytes = off;
  return s;
}

// ---- launchers ----------------------------------------------------------------
moe_status_t launch_dense(const DenseParams& p, cudaStream_t st) {
  const int grid = p.n_rtiles + p.n_stiles;
  if (grid == 0) return MOE_OK;
  k_dense<<<grid, DENSE_THREADS, dense_smem_bytes(p.H), st>>>(p);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// Stage count of a streamed kernel: as many as fit, at most MAX_STAGES, and a
// multiple of the consumer-warp count.  Consumer warp w takes items w, w+NC, ...
// and item i uses stage i % S, so with S % NC == 0 the warp waiting on a stage's
// next phase is the warp that consumed its previous phase -- the mbarrier parity
// it waits on can never alias a phase that has not completed yet.
int stages_for(int dyn_limit, size_t fixed, size_t stage) {
  if ((size_t)dyn_limit <= fixed) return 0;
  size_t s = ((size_t)dyn_limit - fixed) / stage;
  if (s > (size_t)MAX_STAGES) s = MAX_STAGES;
  return (int)(s / N_CONSUMERS * N_CONSUMERS);
}

moe_status_t launch_e13(E13Params p, const DevInfo& d, cudaStream_t st) {
  const size_t fixed = e13_fixed_bytes(p.H), stage = e13_stage_bytes(p.H);
  p.stages = stages_for(d.dyn_e13, fixed, stage);
  if (p.stages < N_CONSUMERS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t smem = fixed + (size_t)p.stages * stage;
  const int grid = d.sms;
  k_experts13<<<grid, EXPERT_THREADS, smem, st>>>(p);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status_t launch_e2(E2Params p, const DevInfo& d, cudaStream_t st) {
  const size_t fixed = e2_fixed_bytes(p.M, p.I, p.Is), stage = e2_stage_bytes(p.I, p.Is);
  p.stages = stages_for(d.dyn_e2, fixed, stage);
  if (p.stages < N_CONSUMERS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t smem = fixed + (size_t)p.stages * stage;
  // Each block's contiguous item range must touch at most E2_MAX_LOCAL_SLOTS experts.
  const long long htiles = p.H / 16;
  const long long nch = p.Is > 0 ? (p.Is + SHARED_CHUNK - 1) / SHARED_CHUNK : 0;
  const long long Tmax = (long long)slots_of(p.M, p.E, p.top_k) * htiles + htiles * nch;
  long long grid = d.sms;
  while ((Tmax + grid - 1) / grid > (E2_MAX_LOCAL_SLOTS - 1) * htiles + 1) grid *= 2;
  k_experts2<<<(int)grid, EXPERT_THREADS, smem, st>>>(p);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status_t launch_lm(LMParams p, const DevInfo& d, cudaStream_t st) {
  const size_t fixed = lm_fixed_bytes(p.H), stage = lm_stage_bytes(p.H);
  p.stages = stages_for(d.dyn_lm, fixed, stage);
  // every consumer warp needs a stage of its own in flight (LM_STAGES == LM_CONSUMERS)
  if (p.stages < LM_CONSUMERS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t smem = fixed + (size_t)p.stages * stage;
  const long long T = (p.V + 7) / 8;
  const int grid = (int)(T < d.sms ? T : d.sms);
  k_lm_gemv<<<grid, LM_THREADS, smem, st>>>(p);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// The whole-step persistent kernel serves the model when it fits: at most
// STEP_MAX_LAYERS layers, H a multiple of 128 (router/shared tiles split into four
// 32-column-aligned quarters), cooperative launch available, and a shared-memory
// ring next to the activation region that holds at least N_CONSUMERS of the
// largest items (one per consumer warp in flight).
bool use_persistent(const moe_model_t& m, int M, const DevInfo& d, uint32_t* ring_bytes) {
  if (m.step_path == MOE_STEP_PER_LAYER) return false;
  if (m.n_layers > STEP_MAX_LAYERS || m.H % 128 != 0 || !d.coop) return false;
  const size_t fixed = STEP_FIXED + step_act_bytes(M, m.H, m.I, m.Is);
  if ((size_t)d.dyn_step <= fixed) return false;
  const size_t ring = ((size_t)d.dyn_step - fixed) / 128 * 128;
  *ring_bytes = (uint32_t)ring;
  // a block's contiguous routed-W2 range of n items (H/16 per expert) touches at most
  // (n - 2) / (H/16) + 2 experts; their activations must fit the block's cache
  const long long T = m.H / 16;
  const long long n = ((long long)slots_of(M, m.E, m.top_k) * T + d.sms - 1) / d.sms;
  const long long span = n <= 1 ? 1 : (n - 2) / T + 2;
  if (span > CR_CACHE) return false;
  return ring >= (size_t)N_CONSUMERS * step_max_item_bytes(m.H, m.I, m.Is);
}

moe_status_t launch_step(const StepParams& sp, const DevInfo& d, cudaStream_t st) {
  const size_t smem = STEP_FIXED + (size_t)sp.ring_bytes + sp.act_bytes;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(d.sms);
  cfg.blockDim = dim3(STEP_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all blocks co-resident: the grid-wide waits need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the profiling and trace code only in the instantiation a timeline or trace asks for
  const bool dbg = sp.timeline || sp.x_trace || sp.h_trace || sp.ids_trace || sp.w_trace;
  if (sp.M == 1)
    MOE_CUDA(cudaLaunchKernelEx(&cfg, dbg ? k_step<true, true> : k_step<true, false>, sp));
  else
    MOE_CUDA(cudaLaunchKernelEx(&cfg, dbg ? k_step<false, true> : k_step<false, false>, sp));
  return MOE_OK;
}

// One 64-bit word written on the stream (capturable): the test wait limit of a control block.
__global__ void k_set_u64(unsigned long long* p, unsigned long long v) { *p = v; }

// Records events[2i] / events[2i+1] around launch i when the caller asked for them.
struct EventHook {
  cudaEvent_t* ev = nullptr;
  int n = 0;
  int i = 0;
  // External records: under stream capture they become event-record graph nodes
  // (a plain record would only mark a capture dependency); outside capture they are
  // ordinary records.
  moe_status_t record(cudaEvent_t e, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    MOE_CUDA(cudaStreamIsCapturing(st, &cs));
    if (cs == cudaStreamCaptureStatusActive)
      MOE_CUDA(cudaEventRecordWithFlags(e, st, cudaEventRecordExternal));
    else
      MOE_CUDA(cudaEventRecord(e, st));
    return MOE_OK;
  }
  moe_status_t before(cudaStream_t st) {
    if (ev && 2 * i + 1 < n) return record(ev[2 * i], st);
    return MOE_OK;
  }
  moe_status_t after(cudaStream_t st) {
    moe_status_t s = MOE_OK;
    if (ev && 2 * i + 1 < n) s = record(ev[2 * i + 1], st);
    ++i;
    return s;
  }
};

// ---- validation helpers ---------------------------------------------------------
#define REQ(cond, code) \
  do {                  \
    if (!(cond)) return (code); \
  } while (0)

moe_status_t check_ptrs_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

moe_status_t check_layer_buf(const moe_buf_t& b, int fmt, bool required) {
  if (!b.ptr) return required ? MOE_ERR_INVALID_ARG : MOE_OK;
  if (b.fmt != fmt) return MOE_ERR_DTYPE;
  if (!aligned16(b.ptr)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}


// The chunk path (M > MAX_M) of moe_mxfp4_experts, with the prefill machinery below.
bool ok_pf(int M, int H, int I, int E, int k, int Is);
size_t pf_ws_bytes(int M, int H, int I, int E, int k, int Is);
moe_status_t experts_chunk(const void* x_bf16, int M, int H, int I, int E, int top_k, const int32_t* topk_ids,
                           const float* topk_w, const uint8_t* w13_codes, const uint8_t* w13_scales,
                           const uint8_t* w2_codes, const uint8_t* w2_scales, const void* shared_w13_bf16,
                           const void* shared_w2_bf16, int Is, float* y, void* ws, size_t ws_bytes,
                           moe_stream_t stream);

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_DTYPE: return "MOE_ERR_DTYPE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_SELFCHECK: return "MOE_ERR_SELFCHECK";
    default: return "MOE_ERR_UNKNOWN";
  }
}

int moe_abi_version(void) { return MOE_ABI_VERSION; }
int moe_last_cuda_error(void) { return g_last_cuda_error; }

moe_status_t moe_workspace_status(const void* ws, moe_stream_t stream) {
  REQ(ws, MOE_ERR_INVALID_ARG);
  MOE_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int st = 0;
  MOE_CUDA(cudaMemcpy(&st, ws, sizeof st, cudaMemcpyDeviceToHost));
  return st == 0 ? MOE_OK : (moe_status_t)st;
}

size_t moe_route_workspace_bytes(int M, int E) {
  if (!ok_M(M) || !ok_E(E)) return 0;
  return CTRL_BYTES + up256((size_t)M * E * 4);
}

moe_status_t moe_route(const void* x_bf16, int M, int H, const void* w_router_bf16, int E, int top_k,
                       int32_t* topk_ids, float* topk_w, float* logits_opt, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  REQ(x_bf16 && w_router_bf16 && topk_ids && topk_w, MOE_ERR_INVALID_ARG);
  REQ(ok_M(M) && ok_H(H) && ok_E(E) && ok_k(top_k, E), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({x_bf16, w_router_bf16, topk_ids, topk_w, logits_opt, ws});
  if (s != MOE_OK) return s;
  REQ(ws && ws_bytes >= moe_route_workspace_bytes(M, E), MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(ws);
  MOE_CUDA(cudaMemsetAsync(ws, 0, CTRL_BYTES, st));
  DenseParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.mode = 0;
  p.M = M;
  p.H = H;
  p.wr = static_cast<const __nv_bfloat16*>(w_router_bf16);
  p.E = E;
  p.top_k = top_k;
  p.n_rtiles = E / 16;
  p.logits_ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + CTRL_BYTES);
  p.logits_out = logits_opt;
  p.ids = topk_ids;
  p.w = topk_w;
  p.counter = c.route_counter;
  return launch_dense(p, st);
}

size_t moe_experts_workspace_bytes(int M, int H, int I, int E, int top_k, int Is) {
  if (M > MAX_M) return ok_pf(M, H, I, E, top_k, Is) ? pf_ws_bytes(M, H, I, E, top_k, Is) : 0;
  if (!ok_M(M) || !ok_H(H) || !ok_I(I) || !ok_E(E) || !ok_k(top_k, E) || !ok_Is(Is)) return 0;
  return experts_ws(nullptr, M, H, I, E, top_k, Is).bytes;
}

moe_status_t moe_mxfp4_experts(const void* x_bf16, int M, int H, int I, int E, int top_k,
                               const int32_t* topk_ids, const float* topk_w, const uint8_t* w13_codes,
                               const uint8_t* w13_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                               const void* shared_w13_bf16, const void* shared_w2_bf16, int Is, float* y,
                               void* ws, size_t ws_bytes, moe_stream_t stream) {
  REQ(x_bf16 && topk_ids && topk_w && w13_codes && w13_scales && w2_codes && w2_scales && y, MOE_ERR_INVALID_ARG);
  REQ((Is == 0) == (shared_w13_bf16 == nullptr) && (Is == 0) == (shared_w2_bf16 == nullptr), MOE_ERR_INVALID_ARG);
  moe_status_t s = check_ptrs_aligned({x_bf16, topk_ids, topk_w, w13_codes, w13_scales, w2_codes, w2_scales,
                                       shared_w13_bf16, shared_w2_bf16, y, ws});
  if (s != MOE_OK) return s;
  if (M > MAX_M)  // a chunk: block-scaled tcgen05 GEMMs on MXFP8 activations
    return experts_chunk(x_bf16, M, H, I, E, top_k, topk_ids, topk_w, w13_codes, w13_scales, w2_codes, w2_scales,
                         shared_w13_bf16, shared_w2_bf16, Is, y, ws, ws_bytes, stream);
  REQ(ok_M(M) && ok_H(H) && ok_I(I) && ok_E(E) && ok_k(top_k, E) && ok_Is(Is), MOE_ERR_UNSUPPORTED_SHAPE);
  const size_t need = moe_experts_workspace_bytes(M, H, I, E, top_k, Is);
  REQ(ws && ws_bytes >= need, MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(ws);
  ExpertsWs w = experts_ws(ws, M, H, I, E, top_k, Is);
  MOE_CUDA(cudaMemsetAsync(ws, 0, CTRL_BYTES, st));
  MOE_CUDA(cudaMemsetAsync(y, 0, (size_t)M * H * sizeof(float), st));
  if (Is > 0) {
    DenseParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x_bf16);
    p.mode = 0;
    p.M = M;
    p.H = H;
    p.E = E;
    p.top_k = top_k;
    p.n_rtiles = 0;
    p.sw13 = static_cast<const __nv_bfloat16*>(shared_w13_bf16);
    p.Is = Is;
    p.n_stiles = Is / 8;
    p.a_shared = w.a_shared;
    p.counter = c.route_counter;
    if ((s = launch_dense(p, st)) != MOE_OK) return s;
  }
  E13Params a{};
  a.x = static_cast<const __nv_bfloat16*>(x_bf16);
  a.M = M;
  a.H = H;
  a.I = I;
  a.E = E;
  a.top_k = top_k;
  a.ids = topk_ids;
  a.w = topk_w;
  a.w13c = w13_codes;
  a.w13s = w13_scales;
  a.a_routed = w.a_routed;
  a.status = c.status;
  if ((s = launch_e13(a, d, st)) != MOE_OK) return s;
  E2Params b{};
  b.M = M;
  b.H = H;
  b.I = I;
  b.E = E;
  b.top_k = top_k;
  b.Is = Is;
  b.ids = topk_ids;
  b.w = topk_w;
  b.w2c = w2_codes;
  b.w2s = w2_scales;
  b.sw2 = static_cast<const __nv_bfloat16*>(shared_w2_bf16);
  b.a_routed = w.a_routed;
  b.a_shared = w.a_shared;
  b.out = y;
  b.status = c.status;
  return launch_e2(b, d, st);
}

moe_status_t lm_head_fp8_quantize(const void* w_bf16, int V, int H, uint8_t* w_e4m3, float* row_scale,
                                  moe_stream_t stream) {
  REQ(w_bf16 && w_e4m3 && row_scale, MOE_ERR_INVALID_ARG);
  REQ(V >= 1 && H >= 16 && H <= 16384 && H % 16 == 0, MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({w_bf16, w_e4m3, row_scale});
  if (s != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long blocks = ((long long)V + 7) / 8;
  k_lm_quantize<<<(unsigned)blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w_bf16), V, H, w_e4m3,
                                                   row_scale);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

size_t lm_head_workspace_bytes(int M, int V, int H) {
  if (!ok_M(M) || V < 1 || !ok_H_lm(H)) return 0;
  return CTRL_BYTES;
}

moe_status_t lm_head_fp8_gemv(const void* x_bf16, int M, int V, int H, const uint8_t* w_e4m3,
                              const float* row_scale, float* logits, int32_t* argmax, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  REQ(x_bf16 && w_e4m3 && row_scale && argmax, MOE_ERR_INVALID_ARG);
  REQ(ok_M(M) && V >= 1 && V <= (1 << 26) && ok_H_lm(H), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({x_bf16, w_e4m3, row_scale, logits, argmax, ws});
  if (s != MOE_OK) return s;
  REQ(ws && ws_bytes >= lm_head_workspace_bytes(M, V, H), MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(ws);
  MOE_CUDA(cudaMemsetAsync(ws, 0, CTRL_BYTES, st));
  LMParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.M = M;
  p.V = V;
  p.H = H;
  p.w = w_e4m3;
  p.rs = row_scale;
  p.logits = logits;
  p.argmax = argmax;
  p.keys = c.keys;
  p.counter = c.lm_counter;
  p.status = c.status;
  return launch_lm(p, d, st);
}

moe_status_t lm_head_fp8_verify(const void* x_bf16, int M, int V, int H, const uint8_t* w_e4m3,
                                const float* row_scale, const int32_t* drafts, float* logits, int32_t* argmax,
                                int32_t* accept, void* ws, size_t ws_bytes, moe_stream_t stream) {
  REQ(x_bf16 && w_e4m3 && row_scale && argmax && drafts && accept, MOE_ERR_INVALID_ARG);
  REQ(M >= 2 && ok_M(M) && V >= 1 && V <= (1 << 26) && ok_H_lm(H), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({x_bf16, w_e4m3, row_scale, logits, argmax, ws});
  if (s != MOE_OK) return s;
  REQ(ws && ws_bytes >= lm_head_workspace_bytes(M, V, H), MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(ws);
  MOE_CUDA(cudaMemsetAsync(ws, 0, CTRL_BYTES, st));
  LMParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.M = M;
  p.V = V;
  p.H = H;
  p.w = w_e4m3;
  p.rs = row_scale;
  p.logits = logits;
  p.argmax = argmax;
  p.keys = c.keys;
  p.counter = c.lm_counter;
  p.status = c.status;
  p.drafts = drafts;
  p.accept = accept;
  return launch_lm(p, d, st);
}

moe_status_t lm_head_bf16_gemv(const void* x_bf16, int M, int V, int H, const void* w_bf16, float* logits,
                               int32_t* argmax, void* ws, size_t ws_bytes, moe_stream_t stream) {
  REQ(x_bf16 && w_bf16 && argmax, MOE_ERR_INVALID_ARG);
  REQ(ok_M(M) && V >= 1 && V <= (1 << 26) && ok_H_lm(H), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({x_bf16, w_bf16, logits, argmax, ws});
  if (s != MOE_OK) return s;
  REQ(ws && ws_bytes >= lm_head_workspace_bytes(M, V, H), MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(ws);
  MOE_CUDA(cudaMemsetAsync(ws, 0, CTRL_BYTES, st));
  LMParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.M = M;
  p.V = V;
  p.H = H;
  p.w = static_cast<const uint8_t*>(w_bf16);
  p.logits = logits;
  p.argmax = argmax;
  p.keys = c.keys;
  p.counter = c.lm_counter;
  p.status = c.status;
  const size_t fixed = lmb_fixed_bytes(H), stage = lmb_stage_bytes(H);
  p.stages = stages_for(d.dyn_lmb, fixed, stage);
  if (p.stages < N_CONSUMERS) return MOE_ERR_UNSUPPORTED_SHAPE;
  const long long T = (V + 7) / 8;
  const int grid = (int)(T < d.sms ? T : d.sms);
  k_lm_gemv_bf16<<<grid, EXPERT_THREADS, fixed + (size_t)p.stages * stage, st>>>(p);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status_t moe_sample(const float* logits, int M, int V, float temperature, int top_k, float top_p,
                        const float* u, int32_t* ids, moe_stream_t stream) {
  REQ(logits && u && ids, MOE_ERR_INVALID_ARG);
  REQ(M >= 1 && M <= 65535 && V >= 1 && V <= (1 << 26) && top_k >= 1 && top_k <= SAMPLE_MAX_K && top_k <= V,
      MOE_ERR_UNSUPPORTED_SHAPE);
  REQ(temperature > 0.0f && top_p > 0.0f && top_p <= 1.0f, MOE_ERR_INVALID_ARG);
  moe_status_t s = check_ptrs_aligned({logits, u, ids});
  if (s != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  k_sample<<<M, SAMPLE_THREADS, 0, st>>>(logits, V, temperature, top_k, top_p, u, ids);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

static moe_status_t check_model(const moe_model_t* m) {
  REQ(m && m->layers, MOE_ERR_INVALID_ARG);
  REQ(m->n_layers >= 1 && m->n_layers <= 4096, MOE_ERR_UNSUPPORTED_SHAPE);
  REQ(ok_H_lm(m->H) && ok_I(m->I) && ok_E(m->E) && ok_k(m->top_k, m->E) && ok_Is(m->Is), MOE_ERR_UNSUPPORTED_SHAPE);
  REQ(m->V >= 1 && m->V <= (1 << 26), MOE_ERR_UNSUPPORTED_SHAPE);
  REQ(m->rms_eps >= 0.0f, MOE_ERR_INVALID_ARG);
  moe_status_t s;
  for (int l = 0; l < m->n_layers; ++l) {
    const moe_layer_t& L = m->layers[l];
    if ((s = check_layer_buf(L.router, MOE_FMT_BF16, true)) != MOE_OK) return s;
    if ((s = check_layer_buf(L.w13_codes, MOE_FMT_MXFP4_CODES, true)) != MOE_OK) return s;
    if ((s = check_layer_buf(L.w13_scales, MOE_FMT_E8M0_SCALES, true)) != MOE_OK) return s;
    if ((s = check_layer_buf(L.w2_codes, MOE_FMT_MXFP4_CODES, true)) != MOE_OK) return s;
    if ((s = check_layer_buf(L.w2_scales, MOE_FMT_E8M0_SCALES, true)) != MOE_OK) return s;
    if ((s = check_layer_buf(L.shared_w13, MOE_FMT_BF16, m->Is > 0)) != MOE_OK) return s;
    if ((s = check_layer_buf(L.shared_w2, MOE_FMT_BF16, m->Is > 0)) != MOE_OK) return s;
  }
  if ((s = check_layer_buf(m->lm_head, MOE_FMT_E4M3, true)) != MOE_OK) return s;
  if ((s = check_layer_buf(m->lm_scale, MOE_FMT_F32, true)) != MOE_OK) return s;
  return MOE_OK;
}

int decode_step_launch_names(const moe_model_t* model, int M, const char** names, int max_names) {
  if (check_model(model) != MOE_OK || !ok_M(M)) return -1;
  DevInfo d;
  if (dev_info(&d) != MOE_OK) return -1;
  int n = 0;
  auto put = [&](const char* nm) {
    if (names && n < max_names) names[n] = nm;
    ++n;
  };
  uint32_t ring_bytes = 0;
  if (use_persistent(*model, M, d, &ring_bytes)) {
    put("k_step");
  } else {
    for (int l = 0; l < model->n_layers; ++l) {
      put("k_dense");
      put("k_experts13");
      put("k_experts2");
    }
    put("k_final_norm");
  }
  put("k_lm_gemv");
  return n;
}

size_t decode_step_workspace_bytes(const moe_model_t* model, int M) {
  if (check_model(model) != MOE_OK || !ok_M(M)) return 0;
  return step_ws(nullptr, model->n_layers, M, model->H, model->I, model->E, model->top_k, model->Is).bytes;
}

moe_status_t decode_step(const moe_model_t* model, const void* x_bf16, int M, float* logits, int32_t* argmax,
                         const moe_trace_t* trace_opt, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status_t s = check_model(model);
  if (s != MOE_OK) return s;
  REQ(x_bf16 && argmax, MOE_ERR_INVALID_ARG);
  REQ(ok_M(M), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_trace_t tr{};
  if (trace_opt) tr = *trace_opt;
  if ((s = check_ptrs_aligned({x_bf16, logits, argmax, ws, tr.x, tr.h, tr.ids, tr.w, tr.timeline})) != MOE_OK) return s;
  const int H = model->H, I = model->I, E = model->E, k = model->top_k, Is = model->Is, L = model->n_layers;
  REQ(ws && ws_bytes >= decode_step_workspace_bytes(model, M), MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(ws);
  StepWs w = step_ws(ws, L, M, H, I, E, k, Is);
  MOE_CUDA(cudaMemsetAsync(ws, 0, w.ctrl_bytes, st));
  if (tr.wait_limit_ns) {
    k_set_u64<<<1, 1, 0, st>>>(reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + 16), tr.wait_limit_ns);
    MOE_CUDA(cudaGetLastError());
  }
  const __nv_bfloat16* x_in = static_cast<const __nv_bfloat16*>(x_bf16);
  __nv_bfloat16* xt = static_cast<__nv_bfloat16*>(tr.x);
  EventHook hook;
  hook.ev = reinterpret_cast<cudaEvent_t*>(tr.events);
  hook.n = tr.events ? tr.n_events : 0;
  uint32_t ring_bytes = 0;
  if (use_persistent(*model, M, d, &ring_bytes)) {
    StepParams sp{};
    sp.L = L;
    sp.M = M;
    sp.H = H;
    sp.I = I;
    sp.E = E;
    sp.k = k;
    sp.Is = Is;
    sp.eps = model->rms_eps;
    sp.ring_bytes = ring_bytes;
    sp.act_bytes = step_act_bytes(M, H, I, Is);
    sp.x_in = x_in;
    sp.h = w.h;
    sp.x_final = w.x_final;
    sp.logits = w.tlogits;
    sp.a_shared = w.tshared;
    sp.a_routed = w.a_routed;
    sp.ctr = w.ctr;
    sp.status = c.status;
    sp.x_trace = xt;
    sp.h_trace = tr.h;
    sp.ids_trace = tr.ids;
    sp.w_trace = tr.w;
    sp.timeline = tr.timeline;
    sp.hold_layer = tr.hold_layer - 1;
    for (int l = 0; l < L; ++l) {
      const moe_layer_t& Ly = model->layers[l];
      sp.layer[l] = LayerPtrs{static_cast<const __nv_bfloat16*>(Ly.router.ptr),
                              static_cast<const uint8_t*>(Ly.w13_codes.ptr),
                              static_cast<const uint8_t*>(Ly.w13_scales.ptr),
                              static_cast<const uint8_t*>(Ly.w2_codes.ptr),
                              static_cast<const uint8_t*>(Ly.w2_scales.ptr),
                              static_cast<const __nv_bfloat16*>(Ly.shared_w13.ptr),
                              static_cast<const __nv_bfloat16*>(Ly.shared_w2.ptr)};
    }
    if ((s = hook.before(st)) != MOE_OK || (s = launch_step(sp, d, st)) != MOE_OK || (s = hook.after(st)) != MOE_OK)
      return s;
  } else {
  for (int l = 0; l < L; ++l) {
    const moe_layer_t& Ly = model->layers[l];
    const size_t mh = (size_t)M * H, mk = (size_t)M * k;
    DenseParams p{};
    p.x = x_in;
    p.h = w.h;
    p.mode = l == 0 ? 0 : 1;
    p.eps = model->rms_eps;
    p.x_out = w.x_cur;
    p.x_trace = xt ? xt + l * mh : nullptr;
    p.h_trace = tr.h ? tr.h + l * mh : nullptr;
    p.M = M;
    p.H = H;
    p.wr = static_cast<const __nv_bfloat16*>(Ly.router.ptr);
    p.E = E;
    p.top_k = k;
    p.n_rtiles = E / 16;
    p.logits_ws = w.logits;
    p.ids = w.ids;
    p.w = w.w;
    p.ids_trace = tr.ids ? tr.ids + l * mk : nullptr;
    p.w_trace = tr.w ? tr.w + l * mk : nullptr;
    p.counter = c.route_counter;
    p.sw13 = static_cast<const __nv_bfloat16*>(Ly.shared_w13.ptr);
    p.Is = Is;
    p.n_stiles = Is / 8;
    p.a_shared = w.a_shared;
    if ((s = hook.before(st)) != MOE_OK || (s = launch_dense(p, st)) != MOE_OK || (s = hook.after(st)) != MOE_OK)
      return s;
    E13Params a{};
    a.x = l == 0 ? x_in : w.x_cur;
    a.M = M;
    a.H = H;
    a.I = I;
    a.E = E;
    a.top_k = k;
    a.ids = w.ids;
    a.w = w.w;
    a.w13c = static_cast<const uint8_t*>(Ly.w13_codes.ptr);
    a.w13s = static_cast<const uint8_t*>(Ly.w13_scales.ptr);
    a.a_routed = w.a_routed;
    a.status = c.status;
    if ((s = hook.before(st)) != MOE_OK || (s = launch_e13(a, d, st)) != MOE_OK || (s = hook.after(st)) != MOE_OK)
      return s;
    E2Params b{};
    b.M = M;
    b.H = H;
    b.I = I;
    b.E = E;
    b.top_k = k;
    b.Is = Is;
    b.ids = w.ids;
    b.w = w.w;
    b.w2c = static_cast<const uint8_t*>(Ly.w2_codes.ptr);
    b.w2s = static_cast<const uint8_t*>(Ly.w2_scales.ptr);
    b.sw2 = static_cast<const __nv_bfloat16*>(Ly.shared_w2.ptr);
    b.a_routed = w.a_routed;
    b.a_shared = w.a_shared;
    b.out = w.h;
    b.status = c.status;
    if ((s = hook.before(st)) != MOE_OK || (s = launch_e2(b, d, st)) != MOE_OK || (s = hook.after(st)) != MOE_OK)
      return s;
  }
  if ((s = hook.before(st)) != MOE_OK) return s;
  k_final_norm<<<1, 256, 0, st>>>(w.h, M, H, model->rms_eps, w.x_final, xt ? xt + (size_t)L * M * H : nullptr,
                                  tr.h ? tr.h + (size_t)L * M * H : nullptr);
  MOE_CUDA(cudaGetLastError());
  if ((s = hook.after(st)) != MOE_OK) return s;
  }
  LMParams q{};
  q.x = w.x_final;
  q.M = M;
  q.V = model->V;
  q.H = H;
  q.w = static_cast<const uint8_t*>(model->lm_head.ptr);
  q.rs = static_cast<const float*>(model->lm_scale.ptr);
  q.logits = logits;
  q.argmax = argmax;
  q.keys = c.keys;
  q.counter = c.lm_counter;
  q.status = c.status;
  if ((s = hook.before(st)) != MOE_OK || (s = launch_lm(q, d, st)) != MOE_OK) return s;
  return hook.after(st);
}

// ---- graph capture of a whole step -------------------------------------------
struct moe_graph_s {
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

moe_status_t decode_step_graph_create(const moe_model_t* model, const void* x_bf16, int M, float* logits,
                                      int32_t* argmax, const moe_trace_t* trace_opt, void* ws, size_t ws_bytes,
                                      moe_graph_t* out) {
  REQ(out, MOE_ERR_INVALID_ARG);
  *out = nullptr;
  DevInfo d;
  moe_status_t s = dev_info(&d);  // kernel attributes are set before capture begins
  if (s != MOE_OK) return s;
  cudaStream_t cs;
  MOE_CUDA(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
  cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) {
    cudaStreamDestroy(cs);
    return cuda_fail(e);
  }
  s = decode_step(model, x_bf16, M, logits, argmax, trace_opt, ws, ws_bytes, reinterpret_cast<moe_stream_t>(cs));
  cudaGraph_t g = nullptr;
  e = cudaStreamEndCapture(cs, &g);
  cudaStreamDestroy(cs);
  if (s != MOE_OK) {
    if (g) cudaGraphDestroy(g);
    return s;
  }
  if (e != cudaSuccess) return cuda_fail(e);
  cudaGraphExec_t ex;
  e = cudaGraphInstantiate(&ex, g, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(g);
    return cuda_fail(e);
  }
  moe_graph_s* h = new (std::nothrow) moe_graph_s{g, ex};
  if (!h) {
    cudaGraphExecDestroy(ex);
    cudaGraphDestroy(g);
    return MOE_ERR_INVALID_ARG;
  }
  *out = h;
  return MOE_OK;
}

moe_status_t decode_step_graph_launch(moe_graph_t g, moe_stream_t stream) {
  REQ(g, MOE_ERR_INVALID_ARG);
  MOE_CUDA(cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

void decode_step_graph_destroy(moe_graph_t g) {
  if (!g) return;
  cudaGraphExecDestroy(g->exec);
  cudaGraphDestroy(g->graph);
  delete g;
}

}  // extern "C"

// ---- allocation-free LM head ---------------------------------------------------
// The control block lm_head_fp8_gemv keeps in the caller's workspace (status word,
// completion counter, argmax keys of up to MAX_M tokens) lives here instead: one
// 256-byte copy per device that loads the library, kept until the process exits.
static __device__ __align__(256) unsigned char g_lm_noalloc_scratch[CTRL_BYTES];

namespace {
// Device address of g_lm_noalloc_scratch in the current context.  The name is only a
// host-side stand-in for the array; the address is looked up on every call (a host
// table lookup), so a context created after a device reset never sees a stale one.
moe_status_t lm_noalloc_scratch(void** out) {
  void* p = nullptr;
  MOE_CUDA(cudaGetSymbolAddress(&p, g_lm_noalloc_scratch));
  *out = p;
  return MOE_OK;
}
}  // namespace

extern "C" moe_status_t lm_head_fp8_gemv_noalloc(const void* x_bf16, int M, int V, int H, const uint8_t* w_e4m3,
                                                 const float* row_scale, float* logits, int32_t* argmax,
                                                 moe_stream_t stream) {
  REQ(x_bf16 && w_e4m3 && row_scale && argmax, MOE_ERR_INVALID_ARG);
  // the static control block holds argmax keys for at most MAX_M (8) tokens
  REQ(ok_M(M) && V >= 1 && V <= (1 << 26) && ok_H_lm(H), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({x_bf16, w_e4m3, row_scale, logits, argmax});
  if (s != MOE_OK) return s;
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  void* scratch = nullptr;
  if ((s = lm_noalloc_scratch(&scratch)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ctrl c = ctrl_of(scratch);
  MOE_CUDA(cudaMemsetAsync(scratch, 0, CTRL_BYTES, st));  // counters and keys start at zero
  LMParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.M = M;
  p.V = V;
  p.H = H;
  p.w = w_e4m3;
  p.rs = row_scale;
  p.logits = logits;
  p.argmax = argmax;
  p.keys = c.keys;
  p.counter = c.lm_counter;
  p.status = c.status;
  return launch_lm(p, d, st);
}

// =============================================================================
// prefill chunk: one MoE layer for M tokens on tcgen05 (router, shared expert,
// routed experts with MXFP8 activations)
// =============================================================================
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn f = [] {
    void* fp = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(fp);
  }();
  return f;
}

// Activation operand, K-major in chunks of box_inner elements (chunk_bytes in HBM):
// dims {chunk, rows, K / chunk}, box {chunk, 64 rows, kc}, 128-byte swizzle.  The chunk
// index is the outermost dimension although its stride is the smallest, so kc chunks
// arrive as kc consecutive swizzled tiles.
bool make_map(CUtensorMap* m, CUtensorMapDataType t, const void* base, uint64_t inner, uint64_t rows,
              uint64_t row_bytes, uint32_t box_inner, uint64_t chunk_bytes, int kc, uint32_t box_rows = 64) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[3] = {box_inner, rows, inner / box_inner};
  cuuint64_t strides[2] = {row_bytes, chunk_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, (cuuint32_t)kc};
  cuuint32_t es[3] = {1, 1, 1};
  return f(m, t, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Bytes per activation-scale row: K/32 rounded up to 16 (rows are bulk-copied).
int pf_sf_ld(int K) { return (K / 32 + 15) / 16 * 16; }

// Weight operand as {chunk, rows, 2 halves, K / chunk}: one box of {chunk, 64, 2, kc}
// brings 64 rows and the 64 rows half_bytes further on (gate and up rows, or the next
// 64) for kc consecutive K chunks.  Fewer, larger copies: each tensor copy costs the copy
// engine a fixed fraction of a microsecond besides its bytes.
bool make_map_halves(CUtensorMap* m, CUtensorMapDataType t, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t row_bytes, uint64_t half_bytes, uint32_t box_inner, uint64_t chunk_bytes, int kc) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[4] = {box_inner, rows, 2, inner / box_inner};
  cuuint64_t strides[3] = {row_bytes, half_bytes, chunk_bytes};
  cuuint32_t box[4] = {box_inner, 64, 2, (cuuint32_t)kc};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return f(m, t, 4, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}
// K chunks per stage of a dense (bf16) k_umma launch: as many (4, 2, 1) as divide the
// chunk count and still leave two stages -- each stage costs a fixed hand-off (copy
// issue, barrier waits, commit) besides its bytes, so fewer, larger stages go faster.
int pf_kc(int K, int kbox, const DevInfo& d) {
  const int nch = K / kbox;
  for (int kc = 4; kc > 1; kc /= 2)
    if (nch % kc == 0 && 1024 + 2LL * PF_STAGE_BYTES * kc <= (long long)d.dyn_pf) return kc;
  return 1;
}
// Routed launches: as many K chunks per stage (4, 3, 2, 1) as divide K / 128 and still
// leave two stages beside the scale buffer -- each stage costs the SM's copy engine two
// copies whatever their size, so fewer, larger stages move the weights faster.
int pf_kc_routed(int K, int sf_ld, const DevInfo& d) {
  const int nch = K / 128;
  for (int kc = 4; kc > 1; --kc)
    if (nch % kc == 0 &&
        1024 + 2LL * PF_STAGE_BYTES * kc + (long long)pf_sf_buf_bytes(K, sf_ld) <= (long long)d.dyn_pf)
      return kc;
  return 1;
}

bool ok_pf(int M, int H, int I, int E, int k, int Is) {
  return M >= 128 && M % 128 == 0 && M <= 16384 && H >= 128 && H % 128 == 0 && H <= 4096 && I >= 128 &&
         I % 128 == 0 && I <= 4096 && E >= 128 && E % 128 == 0 && E <= 512 && k >= 1 && k <= 8 && Is >= 0 &&
         Is % 64 == 0 && Is <= 4096;
}

struct PfWs {
  int* status;
  int* counts;  // [E]
  int* fill;    // [E]
  int* goff;    // [E+1]
  int* ntp;     // [E+1]
  uint16_t* te; // [M k / 64 + E] expert of each routed token tile
  size_t clear_bytes;
  float* logits;  // [M][E]
  int32_t* ids;   // [M][k]
  float* w;       // [M][k]
  int32_t* g_tok; // [G]
  float* g_w;     // [G]
  int32_t* pos;   // [M][k]
  uint8_t* xq;    // [G][H]
  uint8_t* xs;    // [G][H/32]
  __nv_bfloat16* as;  // [M][Is]
  uint8_t* aq;    // [G][I]
  uint8_t* aqs;   // [G][I/32]
  size_t bytes;
};
// own_routing: the chunk routes itself (moe_prefill_layer) and needs buffers for its
// router logits, ids and weights; under a caller's routing they are left out.
PfWs pf_ws(void* ws, int M, int H, int I, int E, int k, int Is, bool own_routing = true) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  PfWs s{};
  const size_t G = (size_t)M * k;
  size_t off = 0;
  s.status = reinterpret_cast<int*>(b);
  off += CTRL_BYTES;
  s.counts = reinterpret_cast<int*>(b + off);
  off += up256((size_t)E * 4);
  s.clear_bytes = off;
  s.fill = reinterpret_cast<int*>(b + off);
  off += up256((size_t)E * 4);
  s.goff = reinterpret_cast<int*>(b + off);
  off += up256((size_t)(E + 1) * 4);
  s.ntp = reinterpret_cast<int*>(b + off);
  off += up256((size_t)(E + 1) * 4);
  s.te = reinterpret_cast<uint16_t*>(b + off);
  off += up256((G / PF_BN + (size_t)E) * 2);
  if (own_routing) {
    s.logits = reinterpret_cast<float*>(b + off);
    off += up256((size_t)M * E * 4);
    s.ids = reinterpret_cast<int32_t*>(b + off);
    off += up256(G * 4);
    s.w = reinterpret_cast<float*>(b + off);
    off += up256(G * 4);
  }
  s.g_tok = reinterpret_cast<int32_t*>(b + off);
  off += up256(G * 4);
  s.g_w = reinterpret_cast<float*>(b + off);
  off += up256(G * 4);
  s.pos = reinterpret_cast<int32_t*>(b + off);
  off += up256(G * 4);
  s.xq = b + off;
  off += up256(G * H);
  s.xs = b + off;
  off += up256(G * pf_sf_ld(H));
  s.as = reinterpret_cast<__nv_bfloat16*>(b + off);
  off += up256((size_t)M * (Is > 0 ? Is : 1) * 2);
  s.aq = b + off;
  off += up256(G * I);
  s.aqs = b + off;
  off += up256(G * pf_sf_ld(I));
  s.bytes = off;
  return s;
}

moe_status_t launch_umma(PrefillParams& p, const DevInfo& d, cudaStream_t st) {
  // the MMA issuer unrolls at most four K chunks per stage, whole stages per tile
  const int kbox = (p.mode == PF_R13 || p.mode == PF_R2) ? 128 : 64;
  if (p.kc < 1 || p.kc > 4 || (p.K / kbox) % p.kc != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const bool mx = p.mode == PF_R13 || p.mode == PF_R2;
  const long long stage = (long long)PF_STAGE_BYTES * p.kc;
  const long long sf1 = mx ? (long long)pf_sf_buf_bytes(p.K, p.sf_ld) : 0;
  // a second scale buffer when it costs no stage
  const long long room1 = (long long)d.dyn_pf - 1024 - sf1;
  const long long cap = PF_MAX_STAGES;
  p.sf_bufs = (mx && room1 > 0 && std::min((room1 - sf1) / stage, cap) >= std::min(room1 / stage, cap)) ? 2 : 1;
  const size_t sf = (size_t)(p.sf_bufs * sf1);
  const long long room = (long long)d.dyn_pf - 1024 - (long long)sf;
  const int stages = room > 0 ? (int)(room / stage) : 0;
  p.stages = stages > PF_MAX_STAGES ? PF_MAX_STAGES : stages;
  if (p.stages < 2) return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t smem = 1024 + (size_t)p.stages * stage + sf;
  switch (p.mode) {
    case PF_ROUTER: k_umma<PF_ROUTER><<<d.sms, PF_THREADS, smem, st>>>(p); break;
    case PF_SH13: k_umma<PF_SH13><<<d.sms, PF_THREADS, smem, st>>>(p); break;
    case PF_SH2: k_umma<PF_SH2><<<d.sms, PF_THREADS, smem, st>>>(p); break;
    case PF_R13: k_umma<PF_R13><<<d.sms, PF_THREADS, smem, st>>>(p); break;
    case PF_R2: k_umma<PF_R2><<<d.sms, PF_THREADS, smem, st>>>(p); break;
    default: return MOE_ERR_INVALID_ARG;
  }
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// workspace of a chunk under the caller's routing (moe_mxfp4_experts with M > 8)
size_t pf_ws_bytes(int M, int H, int I, int E, int k, int Is) {
  return pf_ws(nullptr, M, H, I, E, k, Is, false).bytes;
}

// a2-a5 of a chunk whose routing (ids, wts [M][top_k], per-expert counts in w.counts) is
// known: grouped rows per expert, MXFP8 activations, shared expert, routed W13 + SwiGLU,
// routed W2 into y.  Ids outside [0, E) contribute nothing.
moe_status_t pf_experts(const __nv_bfloat16* x, int M, int H, int I, int E, int top_k, const int32_t* ids,
                        const float* wts, const uint8_t* w13_codes, const uint8_t* w13_scales,
                        const uint8_t* w2_codes, const uint8_t* w2_scales, const void* shared_w13_bf16,
                        const void* shared_w2_bf16, int Is, float* y, const PfWs& w, const DevInfo& d,
                        cudaStream_t st) {
  moe_status_t s = MOE_OK;
  const int G = M * top_k;
  // a2: grouped rows per expert
  k_pf_scan<<<1, 1024, 0, st>>>(w.counts, E, w.goff, w.ntp, w.fill, w.te);
  MOE_CUDA(cudaGetLastError());
  k_pf_scatter<<<(G + 255) / 256, 256, 0, st>>>(ids, wts, M, top_k, E, w.goff, w.fill, w.g_tok, w.g_w, w.pos);
  MOE_CUDA(cudaGetLastError());
  k_pf_quant_x<<<(int)(((long long)M * (H / 32) + 255) / 256), 256, 0, st>>>(x, M, H, top_k, w.pos, w.xq, w.xs,
                                                                          pf_sf_ld(H));
  MOE_CUDA(cudaGetLastError());

  // a5: shared expert (bf16): a_s = bf16(silu(Wg x) * Wu x), y = Ws2 a_s
  if (Is > 0) {
    PrefillParams q{};
    q.status = w.status;
    q.kc = pf_kc(H, 64, d);
    REQ(make_map_halves(&q.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, shared_w13_bf16, H, 2 * (uint64_t)Is,
                        (uint64_t)H * 2, (uint64_t)Is * H * 2, 64, 128, q.kc),
        MOE_ERR_INVALID_ARG);
    REQ(make_map(&q.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, M, (uint64_t)H * 2, 64, 128, q.kc),
        MOE_ERR_INVALID_ARG);
    q.mode = PF_SH13;
    q.K = H;
    q.m_tiles = Is / 64;
    q.up_off = Is;
    q.M = M;
    q.out_bf16 = w.as;
    q.out_ld = Is;
    if ((s = launch_umma(q, d, st)) != MOE_OK) return s;
    PrefillParams r{};
    r.status = w.status;
    r.kc = pf_kc(Is, 64, d);
    REQ(make_map_halves(&r.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, shared_w2_bf16, Is, H, (uint64_t)Is * 2,
                        (uint64_t)64 * Is * 2, 64, 128, r.kc),
        MOE_ERR_INVALID_ARG);
    REQ(make_map(&r.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w.as, Is, M, (uint64_t)Is * 2, 64, 128, r.kc),
        MOE_ERR_INVALID_ARG);
    r.mode = PF_SH2;
    r.K = Is;
    r.m_tiles = H / 128;
    r.M = M;
    r.out_f32 = y;
    r.out_ld = H;
    if ((s = launch_umma(r, d, st)) != MOE_OK) return s;
  } else {
    MOE_CUDA(cudaMemsetAsync(y, 0, (size_t)M * H * 4, st));
  }

  // a3: routed W13 + SwiGLU, activation re-quantised to MXFP8 (E2M1 x E4M3 block-scaled)
  PrefillParams a{};
  a.status = w.status;
  a.kc = pf_kc_routed(H, pf_sf_ld(H), d);
  REQ(make_map_halves(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w13_codes, H, (uint64_t)E * 2 * I,
                      (uint64_t)H / 2, (uint64_t)I * (H / 2), 128, 64, a.kc),
      MOE_ERR_INVALID_ARG);
  REQ(make_map(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.xq, H, G, H, 128, 128, a.kc), MOE_ERR_INVALID_ARG);
  REQ(make_map(&a.tmB32, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.xq, H, G, H, 128, 128, a.kc, 32), MOE_ERR_INVALID_ARG);
  a.mode = PF_R13;
  a.K = H;
  a.m_tiles = I / 64;
  a.up_off = I;
  a.prob_rows = 2 * I;
  a.E = E;
  a.ntile_prefix = w.ntp;
  a.goff = w.goff;
  a.tile_e = w.te;
  a.sfa = w13_scales;
  a.sfb = w.xs;
  a.sf_ld = pf_sf_ld(H);
  a.out_q = w.aq;
  a.out_qs = w.aqs;
  a.out_qs_ld = pf_sf_ld(I);
  a.out_ld = I;
  if ((s = launch_umma(a, d, st)) != MOE_OK) return s;

  // a4: routed W2, weighted by the routing weight and added into y
  PrefillParams b{};
  b.status = w.status;
  b.kc = pf_kc_routed(I, pf_sf_ld(I), d);
  REQ(make_map_halves(&b.tmA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w2_codes, I, (uint64_t)E * H, (uint64_t)I / 2,
                      (uint64_t)64 * (I / 2), 128, 64, b.kc),
      MOE_ERR_INVALID_ARG);
  REQ(make_map(&b.tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.aq, I, G, I, 128, 128, b.kc), MOE_ERR_INVALID_ARG);
  REQ(make_map(&b.tmB32, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.aq, I, G, I, 128, 128, b.kc, 32), MOE_ERR_INVALID_ARG);
  b.mode = PF_R2;
  b.K = I;
  b.m_tiles = H / 128;
  b.prob_rows = H;
  b.E = E;
  b.ntile_prefix = w.ntp;
  b.goff = w.goff;
  b.tile_e = w.te;
  b.g_tok = w.g_tok;
  b.g_w = w.g_w;
  b.sfa = w2_scales;
  b.sfb = w.aqs;
  b.sf_ld = pf_sf_ld(I);
  b.out_f32 = y;
  b.out_ld = H;
  if ((s = launch_umma(b, d, st)) != MOE_OK) return s;

  return MOE_OK;
}

// Chunk path of moe_mxfp4_experts: the routing is the caller's.
moe_status_t experts_chunk(const void* x_bf16, int M, int H, int I, int E, int top_k, const int32_t* topk_ids,
                           const float* topk_w, const uint8_t* w13_codes, const uint8_t* w13_scales,
                           const uint8_t* w2_codes, const uint8_t* w2_scales, const void* shared_w13_bf16,
                           const void* shared_w2_bf16, int Is, float* y, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  REQ(ok_pf(M, H, I, E, top_k, Is), MOE_ERR_UNSUPPORTED_SHAPE);
  REQ((reinterpret_cast<uintptr_t>(w13_codes) & 31u) == 0 && (reinterpret_cast<uintptr_t>(w2_codes) & 31u) == 0,
      MOE_ERR_ALIGNMENT);
  REQ(ws && ws_bytes >= pf_ws_bytes(M, H, I, E, top_k, Is), MOE_ERR_WORKSPACE);
  DevInfo d;
  moe_status_t s;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const PfWs w = pf_ws(ws, M, H, I, E, top_k, Is, false);
  MOE_CUDA(cudaMemsetAsync(ws, 0, w.clear_bytes, st));
  const int G = M * top_k;
  k_pf_count<<<(G + 255) / 256, 256, 0, st>>>(topk_ids, G, E, w.counts);
  MOE_CUDA(cudaGetLastError());
  return pf_experts(static_cast<const __nv_bfloat16*>(x_bf16), M, H, I, E, top_k, topk_ids, topk_w, w13_codes,
                    w13_scales, w2_codes, w2_scales, shared_w13_bf16, shared_w2_bf16, Is, y, w, d, st);
}

}  // namespace

extern "C" {

size_t moe_prefill_workspace_bytes(int M, int H, int I, int E, int top_k, int Is) {
  if (!ok_pf(M, H, I, E, top_k, Is)) return 0;
  return pf_ws(nullptr, M, H, I, E, top_k, Is).bytes;
}

moe_status_t moe_prefill_layer(const void* x_bf16, int M, int H, int I, int E, int top_k, const void* w_router_bf16,
                               const uint8_t* w13_codes, const uint8_t* w13_scales, const uint8_t* w2_codes,
                               const uint8_t* w2_scales, const void* shared_w13_bf16, const void* shared_w2_bf16,
                               int Is, int32_t* topk_ids_opt, float* topk_w_opt, float* logits_opt, float* y,
                               void* ws, size_t ws_bytes, moe_stream_t stream) {
  REQ(x_bf16 && w_router_bf16 && w13_codes && w13_scales && w2_codes && w2_scales && y, MOE_ERR_INVALID_ARG);
  REQ(ok_pf(M, H, I, E, top_k, Is), MOE_ERR_UNSUPPORTED_SHAPE);
  REQ(Is == 0 || (shared_w13_bf16 && shared_w2_bf16), MOE_ERR_INVALID_ARG);
  moe_status_t s = check_ptrs_aligned({x_bf16, w_router_bf16, w13_codes, w13_scales, w2_codes, w2_scales,
                                       shared_w13_bf16, shared_w2_bf16, topk_ids_opt, topk_w_opt, logits_opt, y, ws});
  if (s != MOE_OK) return s;
  // the 4-bit tensor-map form reads from 32-byte aligned bases
  REQ((reinterpret_cast<uintptr_t>(w13_codes) & 31u) == 0 && (reinterpret_cast<uintptr_t>(w2_codes) & 31u) == 0,
      MOE_ERR_ALIGNMENT);
  REQ(ws && ws_bytes >= moe_prefill_workspace_bytes(M, H, I, E, top_k, Is), MOE_ERR_WORKSPACE);
  DevInfo d;
  if ((s = dev_info(&d)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const PfWs w = pf_ws(ws, M, H, I, E, top_k, Is);
  const int G = M * top_k;
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(x_bf16);
  MOE_CUDA(cudaMemsetAsync(ws, 0, w.clear_bytes, st));

  // a1: router logits (bf16 x bf16 on tcgen05), top-k, softmax over the selected
  PrefillParams p{};
  p.status = w.status;
  p.E = E;
  p.kc = pf_kc(H, 64, d);
  REQ(make_map_halves(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_router_bf16, H, E, (uint64_t)H * 2,
                      (uint64_t)64 * H * 2, 64, 128, p.kc),
      MOE_ERR_INVALID_ARG);
  REQ(make_map(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, M, (uint64_t)H * 2, 64, 128, p.kc),
      MOE_ERR_INVALID_ARG);
  p.mode = PF_ROUTER;
  p.K = H;
  p.m_tiles = E / 128;
  p.M = M;
  p.out_f32 = w.logits;
  p.out_ld = E;
  if ((s = launch_umma(p, d, st)) != MOE_OK) return s;
  k_pf_topk<<<(M + 7) / 8, 256, 0, st>>>(w.logits, M, E, top_k, w.ids, w.w, w.counts);
  MOE_CUDA(cudaGetLastError());
  if ((s = pf_experts(x, M, H, I, E, top_k, w.ids, w.w, w13_codes, w13_scales, w2_codes, w2_scales,
                      shared_w13_bf16, shared_w2_bf16, Is, y, w, d, st)) != MOE_OK)
    return s;

  if (topk_ids_opt) MOE_CUDA(cudaMemcpyAsync(topk_ids_opt, w.ids, (size_t)G * 4, cudaMemcpyDeviceToDevice, st));
  if (topk_w_opt) MOE_CUDA(cudaMemcpyAsync(topk_w_opt, w.w, (size_t)G * 4, cudaMemcpyDeviceToDevice, st));
  if (logits_opt) MOE_CUDA(cudaMemcpyAsync(logits_opt, w.logits, (size_t)M * E * 4, cudaMemcpyDeviceToDevice, st));
  return MOE_OK;
}

moe_status_t moe_mxfp8_quantize(const float* v, int M, int K, uint8_t* q, uint8_t* scales, moe_stream_t stream) {
  REQ(v && q && scales, MOE_ERR_INVALID_ARG);
  REQ(M >= 1 && K >= 32 && K % 32 == 0 && (long long)M * K <= (1LL << 31), MOE_ERR_UNSUPPORTED_SHAPE);
  moe_status_t s = check_ptrs_aligned({v, q, scales});
  if (s != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  k_mxfp8_quantize<<<(int)(((long long)M * (K / 32) + 7) / 8), 256, 0, st>>>(v, M, K, q, scales);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // extern "C"

// =============================================================================
// start-up self-check
// =============================================================================
namespace {

#include "selfcheck_expected.inc"

constexpr int SC_H = 256, SC_I = 64, SC_E = 16, SC_K = 2, SC_IS = 64, SC_V = 256, SC_M = 4, SC_L = 2;
constexpr float SC_TOL = 5e-3f;  // relative L2 per row, as the parity tests

struct ScBufs {
  uint8_t *x, *wr, *w13c, *w13s, *w2c, *w2s, *sw13, *sw2, *lmq, *lms;
  int32_t *ids, *am, *accept, *drafts;
  float *w, *y, *logits;
  uint8_t* scratch;
  size_t bytes;
};

size_t sc_scratch_bytes(const moe_model_t& m) {
  size_t b = moe_route_workspace_bytes(1, SC_E);
  b = std::max(b, moe_experts_workspace_bytes(1, SC_H, SC_I, SC_E, SC_K, SC_IS));
  b = std::max(b, lm_head_workspace_bytes(SC_M, SC_V, SC_H));
  b = std::max(b, decode_step_workspace_bytes(&m, 1));
  b = std::max(b, decode_step_workspace_bytes(&m, SC_M));
  return b;
}

ScBufs sc_carve(uint8_t* base, const moe_model_t* m) {
  ScBufs b{};
  size_t off = 0;
  auto take = [&](size_t n) {
    uint8_t* p = base ? base + off : nullptr;
    off += up256(n);
    return p;
  };
  b.x = take(SC_M * SC_H * 2);
  b.wr = take(SC_E * SC_H * 2);
  b.w13c = take(SC_E * 2 * SC_I * SC_H / 2);
  b.w13s = take(SC_E * 2 * SC_I * SC_H / 32);
  b.w2c = take(SC_E * SC_H * SC_I / 2);
  b.w2s = take(SC_E * SC_H * SC_I / 32);
  b.sw13 = take(2 * SC_IS * SC_H * 2);
  b.sw2 = take(SC_H * SC_IS * 2);
  b.lmq = take(SC_V * SC_H);
  b.lms = take(SC_V * 4);
  b.ids = reinterpret_cast<int32_t*>(take(SC_K * 4));
  b.w = reinterpret_cast<float*>(take(SC_K * 4));
  b.y = reinterpret_cast<float*>(take(SC_H * 4));
  b.am = reinterpret_cast<int32_t*>(take(SC_M * 4));
  b.accept = reinterpret_cast<int32_t*>(take((1 + SC_M) * 4));
  b.drafts = reinterpret_cast<int32_t*>(take((SC_M - 1) * 4));
  b.logits = reinterpret_cast<float*>(take(SC_M * SC_V * 4));
  b.scratch = take(m ? sc_scratch_bytes(*m) : 0);
  b.bytes = off;
  return b;
}

void sc_model(const ScBufs& b, moe_layer_t* layers, moe_model_t* m) {
  for (int l = 0; l < SC_L; ++l) {
    layers[l].router = {b.wr, MOE_FMT_BF16};
    layers[l].w13_codes = {b.w13c, MOE_FMT_MXFP4_CODES};
    layers[l].w13_scales = {b.w13s, MOE_FMT_E8M0_SCALES};
    layers[l].w2_codes = {b.w2c, MOE_FMT_MXFP4_CODES};
    layers[l].w2_scales = {b.w2s, MOE_FMT_E8M0_SCALES};
    layers[l].shared_w13 = {b.sw13, MOE_FMT_BF16};
    layers[l].shared_w2 = {b.sw2, MOE_FMT_BF16};
  }
  *m = moe_model_t{};
  m->n_layers = SC_L;
  m->H = SC_H;
  m->I = SC_I;
  m->E = SC_E;
  m->top_k = SC_K;
  m->Is = SC_IS;
  m->V = SC_V;
  m->rms_eps = 1e-6f;
  m->layers = layers;
  m->lm_head = {b.lmq, MOE_FMT_E4M3};
  m->lm_scale = {b.lms, MOE_FMT_F32};
  m->step_path = MOE_STEP_AUTO;
}

double sc_rel_l2(const float* got, const float* ref, int n) {
  double num = 0, den = 0;
  for (int i = 0; i < n; ++i) {
    const double dlt = static_cast<double>(got[i]) - ref[i];
    num += dlt * dlt;
    den += static_cast<double>(ref[i]) * ref[i];
  }
  return (num == num) ? std::sqrt(num / (den > 0 ? den : 1e-300)) : 1e300;
}

}  // namespace

extern "C" size_t moe_selfcheck_workspace_bytes(void) {
  moe_layer_t layers[SC_L];
  moe_model_t m;
  ScBufs dummy = sc_carve(reinterpret_cast<uint8_t*>(256), nullptr);  // any aligned base: only pointers
  sc_model(dummy, layers, &m);
  return sc_carve(nullptr, &m).bytes;
}

extern "C" moe_status_t moe_selfcheck(void* ws, size_t ws_bytes, moe_stream_t stream, int* failed_check,
                                      float* max_rel_l2) {
  if (failed_check) *failed_check = 0;
  if (max_rel_l2) *max_rel_l2 = 0.0f;
  REQ(ws, MOE_ERR_INVALID_ARG);
  moe_status_t s = check_ptrs_aligned({ws});
  if (s != MOE_OK) return s;
  REQ(ws_bytes >= moe_selfcheck_workspace_bytes(), MOE_ERR_WORKSPACE);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  moe_layer_t layers[SC_L];
  moe_model_t m;
  ScBufs b = sc_carve(static_cast<uint8_t*>(ws), nullptr);
  sc_model(b, layers, &m);
  b = sc_carve(static_cast<uint8_t*>(ws), &m);
  const size_t scratch = sc_scratch_bytes(m);

  struct Fill {
    void* dst;
    uint32_t n;
    int kind, tid, e0;
  } fills[] = {{b.x, SC_M * SC_H, SC_BF16, 1, 125},
               {b.wr, SC_E * SC_H, SC_BF16, 2, 119},
               {b.w13c, SC_E * 2 * SC_I * SC_H / 2, SC_BYTE, 3, 0},
               {b.w13s, SC_E * 2 * SC_I * SC_H / 32, SC_E8M0, 4, 0},
               {b.w2c, SC_E * SC_H * SC_I / 2, SC_BYTE, 5, 0},
               {b.w2s, SC_E * SC_H * SC_I / 32, SC_E8M0, 6, 0},
               {b.sw13, 2 * SC_IS * SC_H, SC_BF16, 7, 119},
               {b.sw2, SC_H * SC_IS, SC_BF16, 8, 119},
               {b.lmq, SC_V * SC_H, SC_E4M3, 9, 0},
               {b.lms, SC_V, SC_POW2, 10, 0}};
  for (const Fill& f : fills) {
    k_selfcheck_fill<<<(f.n + 255) / 256, 256, 0, st>>>(f.dst, f.n, f.kind, static_cast<uint32_t>(f.tid), f.e0);
    MOE_CUDA(cudaGetLastError());
  }
  MOE_CUDA(cudaMemcpyAsync(b.drafts, kSelfcheckHeadArgmax, (SC_M - 1) * 4, cudaMemcpyHostToDevice, st));

  int fail = 0;
  double worst = 0;
  auto note = [&](int check, bool ok) {
    if (!ok && !fail) fail = check;
  };
  auto device_ok = [&]() -> moe_status_t { return moe_workspace_status(b.scratch, stream); };

  // 1, 2: router and expert layer on token 0
  int32_t ids[SC_K];
  float y[SC_H];
  if ((s = moe_route(b.x, 1, SC_H, b.wr, SC_E, SC_K, b.ids, b.w, nullptr, b.scratch, scratch, stream)) != MOE_OK)
    return s;
  if ((s = moe_mxfp4_experts(b.x, 1, SC_H, SC_I, SC_E, SC_K, b.ids, b.w, b.w13c, b.w13s, b.w2c, b.w2s, b.sw13,
                             b.sw2, SC_IS, b.y, b.scratch, scratch, stream)) != MOE_OK)
    return s;
  if ((s = device_ok()) != MOE_OK) return s;
  MOE_CUDA(cudaMemcpyAsync(ids, b.ids, sizeof ids, cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaMemcpyAsync(y, b.y, sizeof y, cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  note(1, std::equal(ids, ids + SC_K, kSelfcheckIds));
  double r = sc_rel_l2(y, kSelfcheckY, SC_H);
  worst = std::max(worst, r);
  note(2, r <= SC_TOL);

  // 3, 4: FP8 head on the 4 tokens, and its verify window with drafts equal to the
  // head's own argmaxes (every draft must be accepted: accept length 4, not 1)
  int32_t am[SC_M], accept[1 + SC_M];
  if ((s = lm_head_fp8_gemv(b.x, SC_M, SC_V, SC_H, b.lmq, reinterpret_cast<const float*>(b.lms), nullptr, b.am,
                            b.scratch, scratch, stream)) != MOE_OK)
    return s;
  if ((s = device_ok()) != MOE_OK) return s;
  MOE_CUDA(cudaMemcpyAsync(am, b.am, sizeof am, cudaMemcpyDeviceToHost, st));
  if ((s = lm_head_fp8_verify(b.x, SC_M, SC_V, SC_H, b.lmq, reinterpret_cast<const float*>(b.lms), b.drafts,
                              nullptr, b.am, b.accept, b.scratch, scratch, stream)) != MOE_OK)
    return s;
  if ((s = device_ok()) != MOE_OK) return s;
  MOE_CUDA(cudaMemcpyAsync(accept, b.accept, sizeof accept, cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  note(3, std::equal(am, am + SC_M, kSelfcheckHeadArgmax));
  note(4, accept[0] == SC_M && std::equal(accept + 1, accept + 1 + SC_M, kSelfcheckHeadArgmax));

  // 5, 6: two-layer decode step on token 0 alone and on the 4-token window
  float lg[SC_M * SC_V];
  for (int M : {1, SC_M}) {
    const int check = M == 1 ? 5 : 6;
    if ((s = decode_step(&m, b.x, M, b.logits, b.am, nullptr, b.scratch, scratch, stream)) != MOE_OK) return s;
    if ((s = device_ok()) != MOE_OK) return s;
    MOE_CUDA(cudaMemcpyAsync(am, b.am, M * 4, cudaMemcpyDeviceToHost, st));
    MOE_CUDA(cudaMemcpyAsync(lg, b.logits, (size_t)M * SC_V * 4, cudaMemcpyDeviceToHost, st));
    MOE_CUDA(cudaStreamSynchronize(st));
    bool ok = std::equal(am, am + M, kSelfcheckStepArgmax);
    for (int t = 0; t < M; ++t) {
      r = sc_rel_l2(lg + t * SC_V, kSelfcheckStepLogits + t * SC_V, SC_V);
      worst = std::max(worst, r);
      ok = ok && r <= SC_TOL;
    }
    note(check, ok);
  }

  // 7: the step took the single persistent kernel, not the per-layer launches
  note(7, decode_step_launch_names(&m, 1, nullptr, 0) == 2 && decode_step_launch_names(&m, SC_M, nullptr, 0) == 2);

  if (failed_check) *failed_check = fail;
  if (max_rel_l2) *max_rel_l2 = static_cast<float>(worst);
  return fail ? MOE_ERR_SELFCHECK : MOE_OK;
}

#ifdef PF_TIMELINE
// Profiling builds only: copies the routed-W13 prefill timeline (see prefill_kernels.cuh).
extern "C" __attribute__((visibility("default"))) int moe_debug_pf_timeline(unsigned long long* out, int n) {
  return (int)cudaMemcpyFromSymbol(out, pf_tl, (size_t)n * sizeof(unsigned long long));
}
#endif
