// decode_kernels.cuh -- one MoE layer of the batch-1 decode step, M <= 8 tokens.
//
// Three kernels per layer, each a stream over HBM-resident weights:
//   k_dense      router logits (BF16 Wr) + top-k + renormalised weights, and the
//                shared expert's W13 + SwiGLU (BF16); optional RMSNorm prologue
//                that chains layers.
//   k_experts13  routed experts' MXFP4 W13 + SwiGLU, one pass per *distinct*
//                expert of the M-token window (each expert's bytes read once).
//   k_experts2   routed MXFP4 W2 weighted by the routing weights + shared W2,
//                accumulated into the output (or the residual stream).
//
// Dataflow of the expert kernels: a producer warp moves whole weight tiles
// (16 rows) from HBM into a ring of shared-memory stages with bulk copies
// (TMA engine, mbarrier completion, L2 evict-first); four consumer warps turn
// the tiles into warp tensor-core products.  MXFP4 codes are widened to f16 by
// the hardware e2m1x2 conversion, products accumulate in fp32 per 32-element
// scale block and are scaled by the block's E8M0 factor in fp32 -- the same
// arithmetic as the definition, reassociated only across the sum.
//
// Sources: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理
// 吞吐的三种方法), sections 事件概述或研究问题 (8 of 512 experts + 1 shared, weight
// reads dominate at batch 1) and 方法/产品要点 items 1 and 3 (MXFP4 experts,
// moe_intermediate_size 768, up to 32 experts in a 4-token verify window).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int MAX_M = 8;
constexpr int MAX_SLOTS = 64;  // distinct experts of a window: <= MAX_M * 8
constexpr int N_CONSUMERS = 4;
constexpr int MAX_STAGES = 8;

// ---------------------------------------------------------------------------
// Union plan: the distinct experts of the window, ascending, with the weight
// each token gives them (0 when the token did not select the expert).
// ---------------------------------------------------------------------------
struct Plan {
  int n_unique;
  int ids[MAX_SLOTS];
  float w[MAX_SLOTS][MAX_M];
  unsigned bits[32];  // membership bitmap over expert ids (E <= 1024)
  int pref[32];       // exclusive prefix popcount of bits[]
};

// Built by one warp.  Ids outside [0, E) are dropped.  A token that lists the same
// expert twice gives it the sum of both weights.
__device__ __forceinline__ void build_plan(Plan& P, const int32_t* ids, const float* w, int M, int k,
                                           int E) {
  const int lane = threadIdx.x & 31;
  const int n = M * k;
  P.bits[lane] = 0u;
  for (int i = lane; i < MAX_SLOTS * MAX_M; i += 32) (&P.w[0][0])[i] = 0.0f;
  __syncwarp();
  int my_id[2];
  float my_w[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int i = lane + 32 * r;
    my_id[r] = -1;
    my_w[r] = 0.0f;
    if (i < n) {
      const int e = ids[i];
      if (e >= 0 && e < E) {
        my_id[r] = e;
        my_w[r] = w[i];
        atomicOr(&P.bits[e >> 5], 1u << (e & 31));
      }
    }
  }
  __syncwarp();
  const unsigned word = P.bits[lane];
  const int cnt = __popc(word);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int excl = incl - cnt;
  P.pref[lane] = excl;
  if (lane == 31) P.n_unique = incl;
  {
    unsigned wb = word;
    int j = excl;
    while (wb) {
      const int b = __ffs(wb) - 1;
      wb &= wb - 1u;
      P.ids[j++] = 32 * lane + b;
    }
  }
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int i = lane + 32 * r;
    if (my_id[r] >= 0) {
      const int e = my_id[r];
      const int slot = P.pref[e >> 5] + __popc(P.bits[e >> 5] & ((1u << (e & 31)) - 1u));
      atomicAdd(&P.w[slot][i / k], my_w[r]);
    }
  }
  __syncwarp();
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// k_dense: router (+ top-k tail) and shared-expert W13 + SwiGLU
// ---------------------------------------------------------------------------
struct DenseParams {
  const __nv_bfloat16* x;  // mode 0: layer input [M][H]
  float* h;                // residual stream [M][H]: mode 1 reads it; mode 0 writes fp32(x) if non-null
  int mode;                // 0: x given; 1: x = bf16(RMSNorm(h))
  float eps;
  __nv_bfloat16* x_out;    // mode 1: block 0 stores the computed x here
  __nv_bfloat16* x_trace;  // optional [M][H]
  float* h_trace;          // optional [M][H]
  int M, H;
  const __nv_bfloat16* wr;  // router [E][H]
  int E, top_k, n_rtiles;   // n_rtiles = E/16 router tiles (0: no router)
  float* logits_ws;         // [M][E]
  float* logits_out;        // optional [M][E]
  int32_t* ids;             // [M][top_k]
  float* w;                 // [M][top_k]
  int32_t* ids_trace;
  float* w_trace;
  unsigned* counter;        // zero on entry; last router block resets it
  const __nv_bfloat16* sw13;  // shared W13 [2Is][H]
  int Is, n_stiles;           // n_stiles = Is/8 shared tiles
  float* a_shared;            // [M][Is]
};

constexpr int DENSE_THREADS = 256;

__host__ __device__ inline size_t dense_smem_bytes(int H) {
  return 8 * (size_t)padded_stride(2u * H) + 8 * 32 * 4 * sizeof(float);
}

// Row r of bf16 x (token-major) scaled by 1/rms: the layer-chaining stand-in.
__device__ __forceinline__ void rms_rows(const float* h, int M, int H, float eps, float* rscale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  for (int t = warp; t < M; t += nw) {
    float ss = 0.0f;
    for (int i = lane; i < H; i += 32) {
      const float v = h[(size_t)t * H + i];
      ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) rscale[t] = 1.0f / sqrtf(ss / (float)H + eps);
  }
}

__global__ void __launch_bounds__(DENSE_THREADS) k_dense(DenseParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_r[MAX_M];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, H = p.H;
  const uint32_t xss = padded_stride(2u * H);
  uint8_t* xs = smem;                                        // bf16 [8][xss/2]
  float* red = reinterpret_cast<float*>(smem + 8 * xss);     // [8][32][4]

  // 1. Stage this layer's input x (bf16) in shared memory, tokens >= M zero.
  if (p.mode == 1) {
    rms_rows(p.h, M, H, p.eps, s_r);
    __syncthreads();
  }
  for (int i = tid; i < MAX_M * (H / 2); i += DENSE_THREADS) {
    const int tok = i / (H / 2), c = i % (H / 2);
    __nv_bfloat162 v = __floats2bfloat162_rn(0.0f, 0.0f);
    if (tok < M) {
      if (p.mode == 1) {
        const float2 hv = *reinterpret_cast<const float2*>(p.h + (size_t)tok * H + 2 * c);
        v = __floats2bfloat162_rn(hv.x * s_r[tok], hv.y * s_r[tok]);
      } else {
        v = *reinterpret_cast<const __nv_bfloat162*>(p.x + (size_t)tok * H + 2 * c);
      }
    }
    *reinterpret_cast<__nv_bfloat162*>(xs + tok * xss + 4 * c) = v;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int i = tid; i < M * H; i += DENSE_THREADS) {
      const int tok = i / H, c = i % H;
      const __nv_bfloat16 xv = *reinterpret_cast<const __nv_bfloat16*>(xs + tok * xss + 2 * c);
      if (p.mode == 1) {
        if (p.x_out) p.x_out[i] = xv;
        if (p.h_trace) p.h_trace[i] = p.h[i];
      } else {
        const float hv = __bfloat162float(xv);
        if (p.h) p.h[i] = hv;
        if (p.h_trace) p.h_trace[i] = hv;
      }
      if (p.x_trace) p.x_trace[i] = xv;
    }
  }

  // 2. This block's 16-row tile, K split across the 8 warps (interleaved 32-column spans).
  const int tile = blockIdx.x;
  const bool is_router = tile < p.n_rtiles;
  const __nv_bfloat16* W;
  int R0, R1, st = 0;
  if (is_router) {
    W = p.wr;
    R0 = 16 * tile + g;
    R1 = R0 + 8;
  } else {
    st = tile - p.n_rtiles;
    W = p.sw13;
    R0 = 8 * st + g;       // gate row
    R1 = p.Is + 8 * st + g;  // up row
  }
  const uint8_t* rowA = reinterpret_cast<const uint8_t*>(W + (size_t)R0 * H);
  const uint8_t* rowB = reinterpret_cast<const uint8_t*>(W + (size_t)R1 * H);
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  const int nspan = H / 32;
  constexpr int U = 4;
  for (int j0 = warp; j0 < nspan; j0 += 8 * U) {
    uint4 A[U], B[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + 8 * u;
      if (j < nspan) {
        A[u] = ldg128_stream(rowA + 64 * j + 16 * t);
        B[u] = ldg128_stream(rowB + 64 * j + 16 * t);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + 8 * u;
      if (j < nspan) {
        const uint4 X = lds128(xs + g * xss + 64 * j + 16 * t);
        mma_bf16(c, A[u].x, B[u].x, A[u].y, B[u].y, X.x, X.y);
        mma_bf16(c, A[u].z, B[u].z, A[u].w, B[u].w, X.z, X.w);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) red[(warp * 32 + lane) * 4 + i] = c[i];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float s = 0.0f;
      for (int ww = 0; ww < 8; ++ww) s += red[(ww * 32 + lane) * 4 + i];
      c[i] = s;
    }
    const int ta = 2 * t, tb = 2 * t + 1;
    if (is_router) {
      if (ta < M) {
        p.logits_ws[ta * p.E + R0] = c[0];
        p.logits_ws[ta * p.E + R1] = c[2];
        if (p.logits_out) {
          p.logits_out[ta * p.E + R0] = c[0];
          p.logits_out[ta * p.E + R1] = c[2];
        }
      }
      if (tb < M) {
        p.logits_ws[tb * p.E + R0] = c[1];
        p.logits_ws[tb * p.E + R1] = c[3];
        if (p.logits_out) {
          p.logits_out[tb * p.E + R0] = c[1];
          p.logits_out[tb * p.E + R1] = c[3];
        }
      }
    } else {
      if (ta < M) p.a_shared[ta * p.Is + 8 * st + g] = silu_f32(c[0]) * c[2];
      if (tb < M) p.a_shared[tb * p.Is + 8 * st + g] = silu_f32(c[1]) * c[3];
    }
  }
  if (!is_router) return;

  // 3. The last router block selects the top-k per token (one warp per token).
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.counter, 1u) == (unsigned)(p.n_rtiles - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (warp < M) {
    const int E = p.E;
    uint32_t key[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = lane + 32 * i;
      key[i] = e < E ? float_key(__ldcg(p.logits_ws + warp * E + e)) : 0u;
    }
    int sel_id[8];
    uint32_t sel_key[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sel_id[j] = 0;
      sel_key[j] = 0u;
      if (j < p.top_k) {
        uint32_t bk = 0u;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (key[i] > bk) {
            bk = key[i];
            bi = lane + 32 * i;
          }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        const int mi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(bk == mk ? bi : 0x7fffffff));
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (lane + 32 * i == mi) key[i] = 0u;
        sel_id[j] = mi;
        sel_key[j] = mk;
      }
    }
    if (lane == 0) {
      const float l0 = key_float(sel_key[0]);
      float den = 0.0f, ex[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ex[j] = (j < p.top_k) ? expf(key_float(sel_key[j]) - l0) : 0.0f;
        den += ex[j];
      }
      for (int j = 0; j < p.top_k; ++j) {
        const int o = warp * p.top_k + j;
        const float wj = ex[j] / den;
        p.ids[o] = sel_id[j];
        p.w[o] = wj;
        if (p.ids_trace) p.ids_trace[o] = sel_id[j];
        if (p.w_trace) p.w_trace[o] = wj;
      }
    }
  }
  if (tid == 0) *p.counter = 0u;
}

// ---------------------------------------------------------------------------
// Shared pieces of the streamed expert kernels
// ---------------------------------------------------------------------------
// f16 copy of x scaled per token by a power of two (exact), for the f16 tensor-core
// operand; inv[t] undoes the scaling.  Run by the NC consumer warps.
__device__ __forceinline__ void stage_x_f16(const __nv_bfloat16* x, int M, int H, uint8_t* xs, uint32_t xss,
                                            float* inv) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ int s_shift[MAX_M];
  for (int tok = warp; tok < MAX_M; tok += N_CONSUMERS) {
    float amax = 0.0f;
    if (tok < M)
      for (int i = lane; i < H; i += 32) amax = fmaxf(amax, fabsf(__bfloat162float(x[(size_t)tok * H + i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) {
      const int sh = f16_range_shift(amax);
      s_shift[tok] = sh;
      inv[tok] = exp2i(-sh);
    }
  }
  named_barrier(1, 32 * N_CONSUMERS);
  for (int i = tid; i < MAX_M * (H / 2); i += 32 * N_CONSUMERS) {
    const int tok = i / (H / 2), c = i % (H / 2);
    __half2 v = __floats2half2_rn(0.0f, 0.0f);
    if (tok < M) {
      const float sc = exp2i(s_shift[tok]);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(x + (size_t)tok * H + 2 * c);
      v = __floats2half2_rn(__low2float(b) * sc, __high2float(b) * sc);
    }
    *reinterpret_cast<__half2*>(xs + tok * xss + 4 * c) = v;
  }
  named_barrier(1, 32 * N_CONSUMERS);
}

// The warp's 16 x K MXFP4 tile against NP passes of (2 tokens x 4 scale blocks):
// thread (g, t) owns scale block 4q+t of rows g and g+8 (16 codes bytes each);
// column n of pass p is (block n%4, token n/4 + 2p) -- the B operand is zero
// outside its block, so every MMA column sums exactly one scale block and the
// E8M0 factor is applied in fp32 afterwards.
//   codes_g/codes_g8: row g / row g+8 codes in shared memory; sc_g/sc_g8: their scale bytes
//   xb: f16 activation rows (stride xss bytes) holding the B operand (block-aligned)
//   acc[p][0/1]: row g / g+8 partial sums for token t/2 + 2p (blocks 2(t&1), 2(t&1)+1)
template <int NP>
__device__ __forceinline__ void mxfp4_tile_dot(const uint8_t* codes_g, const uint8_t* codes_g8,
                                               const uint8_t* sc_g, const uint8_t* sc_g8, int nb,
                                               const uint8_t* xb, uint32_t xss, int M, float (&acc)[NP][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int nq = (nb + 3) / 4;
  for (int q = 0; q < nq; ++q) {
    const int beta = 4 * q + t;
    const bool valid = beta < nb;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const uint4 A0 = valid ? lds128(codes_g + 16 * beta) : zero;
    const uint4 A1 = valid ? lds128(codes_g8 + 16 * beta) : zero;
    const int sb = 4 * q + 2 * (t & 1);
    const float s00 = sb < nb ? e8m0_to_f32(sc_g[sb]) : 0.0f;
    const float s01 = sb + 1 < nb ? e8m0_to_f32(sc_g[sb + 1]) : 0.0f;
    const float s10 = sb < nb ? e8m0_to_f32(sc_g8[sb]) : 0.0f;
    const float s11 = sb + 1 < nb ? e8m0_to_f32(sc_g8[sb + 1]) : 0.0f;
    uint32_t X[NP][16];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int tok = g / 4 + 2 * p;
      const bool active = ((g & 3) == t) && tok < M && valid;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const uint4 v = active ? lds128(xb + tok * xss + 64 * beta + 16 * ii) : zero;
        X[p][4 * ii + 0] = v.x;
        X[p][4 * ii + 1] = v.y;
        X[p][4 * ii + 2] = v.z;
        X[p][4 * ii + 3] = v.w;
      }
    }
    float c[NP][4];
#pragma unroll
    for (int p = 0; p < NP; ++p) c[p][0] = c[p][1] = c[p][2] = c[p][3] = 0.0f;
    const uint32_t a0w[4] = {A0.x, A0.y, A0.z, A0.w};
    const uint32_t a1w[4] = {A1.x, A1.y, A1.z, A1.w};
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t h0, h1, h2, h3, k0, k1, k2, k3;
      e2m1x8_to_f16x2(a0w[wd], h0, h1, h2, h3);
      e2m1x8_to_f16x2(a1w[wd], k0, k1, k2, k3);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        mma_f16(c[p], h0, k0, h1, k1, X[p][4 * wd + 0], X[p][4 * wd + 1]);
        mma_f16(c[p], h2, k2, h3, k3, X[p][4 * wd + 2], X[p][4 * wd + 3]);
      }
    }
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      acc[p][0] = fmaf(c[p][0], s00, fmaf(c[p][1], s01, acc[p][0]));
      acc[p][1] = fmaf(c[p][2], s10, fmaf(c[p][3], s11, acc[p][1]));
    }
  }
}

// ---------------------------------------------------------------------------
// k_experts13: routed MXFP4 W13 + SwiGLU, one item = (distinct expert, 8 rows of I)
// ---------------------------------------------------------------------------
struct E13Params {
  const __nv_bfloat16* x;
  int M, H, I, E, top_k;
  const int32_t* ids;
  const float* w;
  const uint8_t* w13c;
  const uint8_t* w13s;
  float* a_routed;  // [n_unique][M][I]
  int* status;
  int stages;
};

constexpr int EXPERT_THREADS = 32 * (N_CONSUMERS + 1);

__host__ __device__ inline size_t e13_stage_bytes(int H) {
  size_t b = 16 * (size_t)padded_stride(H / 2) + 16 * (size_t)(H / 32);
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline size_t e13_fixed_bytes(int H) { return 128 + 8 * (size_t)padded_stride(2u * H); }

template <int NP>
__global__ void __launch_bounds__(EXPERT_THREADS, 1) k_experts13(E13Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ float s_inv[MAX_M];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, H = p.H, I = p.I, S = p.stages;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t cs = padded_stride(H / 2);
  const int nb = H / 32;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + MAX_STAGES;
  uint8_t* xs = smem + 128;
  uint8_t* stages = smem + e13_fixed_bytes(H);
  const size_t sbytes = e13_stage_bytes(H);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) build_plan(P, p.ids, p.w, M, p.top_k, p.E);
  __syncthreads();

  const int ntile = I / 8;
  const long long T = (long long)P.n_unique * ntile;
  const long long start = T * blockIdx.x / gridDim.x;
  const long long end = T * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(end - start);

  if (warp == N_CONSUMERS) {  // producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t rowb = H / 2, scb = 8 * (H / 32);
      for (int i = 0; i < nloc; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, p.status)) break;
        const long long item = start + i;
        const int u = (int)(item / ntile), r0 = 8 * (int)(item % ntile);
        const size_t e2I = (size_t)P.ids[u] * 2 * I;
        uint8_t* st = stages + s * sbytes;
        mbar_arrive_expect_tx(&full[s], 16 * rowb + 2 * scb);
        for (int rr = 0; rr < 8; ++rr) {
          bulk_g2s(st + rr * cs, p.w13c + (e2I + r0 + rr) * rowb, rowb, &full[s], pol);
          bulk_g2s(st + (8 + rr) * cs, p.w13c + (e2I + I + r0 + rr) * rowb, rowb, &full[s], pol);
        }
        bulk_g2s(st + 16 * cs, p.w13s + (e2I + r0) * (H / 32), scb, &full[s], pol);
        bulk_g2s(st + 16 * cs + scb, p.w13s + (e2I + I + r0) * (H / 32), scb, &full[s], pol);
      }
      // Drain: the last uses of each stage must have landed before the block exits.
      for (int i = (nloc > S ? nloc - S : 0); i < nloc; ++i) mbar_wait(&full[i % S], (i / S) & 1, p.status);
    }
    return;
  }

  stage_x_f16(p.x, M, H, xs, xss, s_inv);
  for (int i = warp; i < nloc; i += N_CONSUMERS) {
    const int s = i % S;
    if (!mbar_wait(&full[s], (i / S) & 1, p.status)) return;
    const long long item = start + i;
    const int u = (int)(item / ntile), r0 = 8 * (int)(item % ntile);
    const uint8_t* st = stages + s * sbytes;
    float acc[NP][2];
#pragma unroll
    for (int q = 0; q < NP; ++q) acc[q][0] = acc[q][1] = 0.0f;
    mxfp4_tile_dot<NP>(st + g * cs, st + (8 + g) * cs, st + 16 * cs + g * (H / 32),
                       st + 16 * cs + (8 + g) * (H / 32), nb, xs, xss, M, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      acc[q][0] += __shfl_xor_sync(0xffffffffu, acc[q][0], 1);
      acc[q][1] += __shfl_xor_sync(0xffffffffu, acc[q][1], 1);
      const int tok = t / 2 + 2 * q;
      if ((t & 1) == 0 && tok < M) {
        const float gate = acc[q][0] * s_inv[tok], up = acc[q][1] * s_inv[tok];
        p.a_routed[((size_t)u * M + tok) * I + r0 + g] = silu_f32(gate) * up;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// k_experts2: routed MXFP4 W2 (weighted) + shared BF16 W2, accumulated into out
// ---------------------------------------------------------------------------
struct E2Params {
  int M, H, I, E, top_k, Is;
  const int32_t* ids;
  const float* w;
  const uint8_t* w2c;
  const uint8_t* w2s;
  const __nv_bfloat16* sw2;  // [H][Is] or null
  const float* a_routed;     // [n_unique][M][I]
  const float* a_shared;     // [M][Is]
  float* out;                // [M][H], accumulated into
  int* status;
  int stages;
};

constexpr int E2_MAX_LOCAL_SLOTS = 3;
constexpr int SHARED_CHUNK = 256;

__host__ __device__ inline size_t e2_stage_bytes(int I, int Is) {
  size_t r = 16 * (size_t)padded_stride(I / 2) + 16 * (size_t)(I / 32);
  size_t s = Is > 0 ? 16 * (size_t)padded_stride(2 * SHARED_CHUNK) : 0;
  size_t b = r > s ? r : s;
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline size_t e2_fixed_bytes(int M, int I, int Is) {
  size_t b = 128;
  b += (size_t)E2_MAX_LOCAL_SLOTS * MAX_M * padded_stride(2u * I);  // f16 a of routed slots
  b += Is > 0 ? 2 * (size_t)MAX_M * padded_stride(2u * Is) : 0;    // bf16 hi/lo of shared a
  (void)M;
  return (b + 127) / 128 * 128;
}

template <int NP>
__global__ void __launch_bounds__(EXPERT_THREADS, 1) k_experts2(E2Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ float s_pscale[E2_MAX_LOCAL_SLOTS][MAX_M];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, H = p.H, I = p.I, Is = p.Is, S = p.stages;
  const uint32_t ass = padded_stride(2u * I);
  const uint32_t sss = Is > 0 ? padded_stride(2u * Is) : 0u;
  const uint32_t cs = padded_stride(I / 2);
  const uint32_t css = padded_stride(2 * SHARED_CHUNK);
  const int nb = I / 32;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + MAX_STAGES;
  uint8_t* af = smem + 128;                                           // f16 [3][8][ass]
  uint8_t* shi = af + (size_t)E2_MAX_LOCAL_SLOTS * MAX_M * ass;       // bf16 [8][sss]
  uint8_t* slo = shi + (size_t)MAX_M * sss;                           // bf16 [8][sss]
  uint8_t* stages = smem + e2_fixed_bytes(M, I, Is);
  const size_t sbytes = e2_stage_bytes(I, Is);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) build_plan(P, p.ids, p.w, M, p.top_k, p.E);
  __syncthreads();

  const int htiles = H / 16;
  const int nch = Is > 0 ? (Is + SHARED_CHUNK - 1) / SHARED_CHUNK : 0;
  const long long Tr = (long long)P.n_unique * htiles;
  const long long T = Tr + (long long)htiles * nch;
  const long long start = T * blockIdx.x / gridDim.x;
  const long long end = T * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(end - start);
  const int u_lo = start < Tr ? (int)(start / htiles) : 0;

  if (warp == N_CONSUMERS) {  // producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int i = 0; i < nloc; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, p.status)) break;
        const long long item = start + i;
        uint8_t* st = stages + s * sbytes;
        if (item < Tr) {
          const int u = (int)(item / htiles), h0 = 16 * (int)(item % htiles);
          const size_t eH = (size_t)P.ids[u] * H;
          const uint32_t rowb = I / 2, scb = 16 * (I / 32);
          mbar_arrive_expect_tx(&full[s], 16 * rowb + scb);
          for (int rr = 0; rr < 16; ++rr)
            bulk_g2s(st + rr * cs, p.w2c + (eH + h0 + rr) * rowb, rowb, &full[s], pol);
          bulk_g2s(st + 16 * cs, p.w2s + (eH + h0) * (I / 32), scb, &full[s], pol);
        } else {
          const long long si = item - Tr;
          const int h0 = 16 * (int)(si / nch), ch = (int)(si % nch);
          const int k0 = ch * SHARED_CHUNK, len = min(SHARED_CHUNK, Is - k0);
          mbar_arrive_expect_tx(&full[s], 16 * 2 * len);
          for (int rr = 0; rr < 16; ++rr)
            bulk_g2s(st + rr * css, p.sw2 + (size_t)(h0 + rr) * Is + k0, 2 * len, &full[s], pol);
        }
      }
      for (int i = (nloc > S ? nloc - S : 0); i < nloc; ++i) mbar_wait(&full[i % S], (i / S) & 1, p.status);
    }
    return;
  }

  // Consumers: stage the routed activations of the slots this block touches as
  // f16 (power-of-two scaled per slot and token) and the shared activations as a
  // bf16 hi + lo pair (two MMA columns per token, error ~2^-17 relative).
  {
    const int u_hi = (end > start && start < Tr) ? (int)((min(end, Tr) - 1) / htiles) : u_lo - 1;
    const int nsl = u_hi - u_lo + 1;
    for (int pr = warp; pr < E2_MAX_LOCAL_SLOTS * MAX_M; pr += N_CONSUMERS) {
      const int uu = pr / MAX_M, tok = pr % MAX_M;
      const int u = u_lo + uu;
      uint8_t* dst = af + (size_t)pr * ass;
      const bool live = uu < nsl && tok < M && P.w[u][tok] != 0.0f;
      float amax = 0.0f;
      const float* src = live ? p.a_routed + ((size_t)u * M + tok) * I : nullptr;
      if (live)
        for (int i = lane; i < I; i += 32) amax = fmaxf(amax, fabsf(src[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const int sh = f16_range_shift(amax);
      const float sc = exp2i(sh);
      for (int i = lane; i < I / 2; i += 32) {
        __half2 v = __floats2half2_rn(0.0f, 0.0f);
        if (live) v = __floats2half2_rn(src[2 * i] * sc, src[2 * i + 1] * sc);
        *reinterpret_cast<__half2*>(dst + 4 * i) = v;
      }
      if (lane == 0) s_pscale[uu][tok] = live ? exp2i(-sh) : 0.0f;
    }
    if (Is > 0 && end > Tr) {
      for (int i = tid; i < MAX_M * Is; i += 32 * N_CONSUMERS) {
        const int tok = i / Is, c = i % Is;
        float a = tok < M ? p.a_shared[(size_t)tok * Is + c] : 0.0f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(a);
        const __nv_bfloat16 lo = __float2bfloat16_rn(a - __bfloat162float(hi));
        *reinterpret_cast<__nv_bfloat16*>(shi + tok * sss + 2 * c) = hi;
        *reinterpret_cast<__nv_bfloat16*>(slo + tok * sss + 2 * c) = lo;
      }
    }
    named_barrier(1, 32 * N_CONSUMERS);
  }

  for (int i = warp; i < nloc; i += N_CONSUMERS) {
    const int s = i % S;
    if (!mbar_wait(&full[s], (i / S) & 1, p.status)) return;
    const long long item = start + i;
    const uint8_t* st = stages + s * sbytes;
    if (item < Tr) {
      const int u = (int)(item / htiles), h0 = 16 * (int)(item % htiles);
      const int uu = u - u_lo;
      float acc[NP][2];
#pragma unroll
      for (int q = 0; q < NP; ++q) acc[q][0] = acc[q][1] = 0.0f;
      mxfp4_tile_dot<NP>(st + g * cs, st + (8 + g) * cs, st + 16 * cs + g * (I / 32),
                         st + 16 * cs + (8 + g) * (I / 32), nb, af + (size_t)uu * MAX_M * ass, ass, M, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        acc[q][0] += __shfl_xor_sync(0xffffffffu, acc[q][0], 1);
        acc[q][1] += __shfl_xor_sync(0xffffffffu, acc[q][1], 1);
        const int tok = t / 2 + 2 * q;
        if ((t & 1) == 0 && tok < M) {
          const float wt = P.w[u][tok];
          if (wt != 0.0f) {
            const float f = wt * s_pscale[uu][tok];
            atomicAdd(p.out + (size_t)tok * H + h0 + g, acc[q][0] * f);
            atomicAdd(p.out + (size_t)tok * H + h0 + g + 8, acc[q][1] * f);
          }
        }
      }
    } else {
      const long long si = item - Tr;
      const int h0 = 16 * (int)(si / nch), ch = (int)(si % nch);
      const int k0 = ch * SHARED_CHUNK, len = min(SHARED_CHUNK, Is - k0);
      const int npass = (M + 3) / 4;
      float c[2][4];
#pragma unroll
      for (int q = 0; q < 2; ++q) c[q][0] = c[q][1] = c[q][2] = c[q][3] = 0.0f;
      for (int j = 0; j < len / 32; ++j) {
        const uint4 A0 = lds128(st + g * css + 64 * j + 16 * t);
        const uint4 A1 = lds128(st + (8 + g) * css + 64 * j + 16 * t);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q < npass) {
            const int tok = g / 2 + 4 * q;
            const uint8_t* src = (g & 1) ? slo : shi;
            const uint4 X = tok < M ? lds128(src + tok * sss + 2 * (k0 + 32 * j + 8 * t)) : make_uint4(0, 0, 0, 0);
            mma_bf16(c[q], A0.x, A1.x, A0.y, A1.y, X.x, X.y);
            mma_bf16(c[q], A0.z, A1.z, A0.w, A1.w, X.z, X.w);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int tok = t + 4 * q;
        if (q < npass && tok < M) {
          atomicAdd(p.out + (size_t)tok * H + h0 + g, c[q][0] + c[q][1]);
          atomicAdd(p.out + (size_t)tok * H + h0 + g + 8, c[q][2] + c[q][3]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// k_final_norm: x_L = bf16(RMSNorm(h_L)) for the LM head (one block)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_final_norm(const float* h, int M, int H, float eps,
                                                    __nv_bfloat16* x_out, __nv_bfloat16* x_trace,
                                                    float* h_trace) {
  __shared__ float s_r[MAX_M];
  rms_rows(h, M, H, eps, s_r);
  __syncthreads();
  for (int i = threadIdx.x; i < M * H; i += blockDim.x) {
    const int tok = i / H;
    const __nv_bfloat16 v = __float2bfloat16_rn(h[i] * s_r[tok]);
    x_out[i] = v;
    if (x_trace) x_trace[i] = v;
    if (h_trace) h_trace[i] = h[i];
  }
}

}  // namespace moe
