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
    for (int c = lane; c < H / 4; c += 32) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(h + (size_t)t * H) + c);
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
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
// f16 copy of x scaled per token by a power of two (exact), for the f16 products;
// shift[t] receives token t's exponent sh (x_t * 2^sh has its largest magnitude in
// [2^14, 2^15)).  Run by the N_CONSUMERS consumer warps.
template <int NC = N_CONSUMERS>  // the consumer warps that run it (warps 0 .. NC-1)
__device__ __forceinline__ void stage_x_f16(const __nv_bfloat16* x, int M, int H, uint8_t* xs, uint32_t xss,
                                            int* shift) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int tok = warp; tok < MAX_M; tok += NC) {
    float amax = 0.0f;
    if (tok < M)
      for (int c = lane; c < H / 8; c += 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)tok * H + 8 * c);
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(__low2float(b[j])), fabsf(__high2float(b[j]))));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) shift[tok] = f16_range_shift(amax);
  }
  named_barrier(1, 32 * NC);
  for (int i = tid; i < MAX_M * (H / 8); i += 32 * NC) {
    const int tok = i / (H / 8), c = i % (H / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (tok < M) {
      v = *reinterpret_cast<const uint4*>(x + (size_t)tok * H + 8 * c);
      const int sh = shift[tok];
      uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
        const __half2 hh = __floats2half2_rn(mul_pow2(__low2float(b), sh), mul_pow2(__high2float(b), sh));
        w[j] = *reinterpret_cast<const uint32_t*>(&hh);
      }
    }
    *reinterpret_cast<uint4*>(xs + tok * xss + 16 * c) = v;
  }
  named_barrier(1, 32 * NC);
}

// Largest and smallest E8M0 scale byte of rows g and g+8 (the 4 lanes of a lane group
// split the row's bytes, 32-bit words when the row allows, and combine with two
// shuffles).  Every lane of group g returns its rows' values.
__device__ __forceinline__ void row_scale_range(const uint8_t* sc_g, const uint8_t* sc_g8, int nb, uint32_t& mx_g,
                                                uint32_t& mx_g8, uint32_t& mn_g, uint32_t& mn_g8) {
  const int t = threadIdx.x & 3;
  uint32_t a = 0u, b = 0u, c = 0xFFFFFFFFu, d = 0xFFFFFFFFu;
  if ((nb & 3) == 0 && ((reinterpret_cast<uintptr_t>(sc_g) | reinterpret_cast<uintptr_t>(sc_g8)) & 3u) == 0) {
    const uint32_t* ga = reinterpret_cast<const uint32_t*>(sc_g);
    const uint32_t* gb = reinterpret_cast<const uint32_t*>(sc_g8);
    for (int i = t; i < nb / 4; i += 4) {
      const uint32_t wa = ga[i], wb = gb[i];
      a = __vmaxu4(a, wa);
      b = __vmaxu4(b, wb);
      c = __vminu4(c, wa);
      d = __vminu4(d, wb);
    }
  } else {
    for (int i = t; i < nb; i += 4) {
      const uint32_t wa = sc_g[i] * 0x01010101u, wb = sc_g8[i] * 0x01010101u;
      a = __vmaxu4(a, wa);
      b = __vmaxu4(b, wb);
      c = __vminu4(c, wa);
      d = __vminu4(d, wb);
    }
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    a = __vmaxu4(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = __vmaxu4(b, __shfl_xor_sync(0xffffffffu, b, o));
    c = __vminu4(c, __shfl_xor_sync(0xffffffffu, c, o));
    d = __vminu4(d, __shfl_xor_sync(0xffffffffu, d, o));
  }
  mx_g = max(max(a & 0xFFu, (a >> 8) & 0xFFu), max((a >> 16) & 0xFFu, a >> 24));
  mx_g8 = max(max(b & 0xFFu, (b >> 8) & 0xFFu), max((b >> 16) & 0xFFu, b >> 24));
  mn_g = min(min(c & 0xFFu, (c >> 8) & 0xFFu), min((c >> 16) & 0xFFu, c >> 24));
  mn_g8 = min(min(d & 0xFFu, (d >> 8) & 0xFFu), min((d >> 16) & 0xFFu, d >> 24));
}

// f16x2 of 2^d in both halves, d = e - ref in [-23, 0]: normal for d >= -14,
// subnormal below.  Every E2M1 value times 2^d is then an exact f16 number (its
// lowest set bit is 2^(d-1) >= 2^-24, the f16 subnormal step).
__device__ __forceinline__ uint32_t pow2_f16x2(int d) {
  uint32_t b = d >= -14 ? (uint32_t)(d + 15) << 10 : (d >= -24 ? 1u << (d + 24) : 0u);
  return b | (b << 16);
}
// Largest scale span (row maximum minus row minimum exponent) over which folding the
// block scales into the f16 codes, relative to the row maximum, stays exact.
constexpr int FOLD_SPAN = 23;

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Activations of the MXFP4 products are f16 rows scaled per token by 2^sh (sh from
// f16_range_shift of the row's largest magnitude): the tile products below return
// results in the true units, the shift undone together with the weight scales.

// The warp's 16 x K MXFP4 tile (rows g and g+8 of each lane group) against up to 8
// token columns on the warp tensor core.  Thread (g, t) owns scale block 4q+t of both
// rows: its 32 codes per row widen to f16 with the hardware e2m1x2 conversion and are
// multiplied by 2^(e - e_ref) with e_ref the row's largest scale -- exact because the
// caller only takes this path when every row's scale span is at most FOLD_SPAN.  Every
// MMA column is one token and the fp32 accumulators run over the whole row; the factor
// 2^(e_ref - 127 - sh_token) is applied once at the end (ldexpf: exact, any range).
// c[]: c0 (row g, token 2t), c1 (row g, token 2t+1), c2 (row g+8, token 2t),
// c3 (row g+8, token 2t+1).  Tokens >= M read zeros.
//   codes_g/codes_g8: row g / row g+8 codes in shared memory; sc_g/sc_g8: their scales
//   xb: f16 activation rows (stride xss bytes), token n at xb + n*xss, shift xsh[n]
// Rows with a multiple of 8 scale blocks (every Ling-shaped tile): two groups per
// iteration into eight accumulators.
__device__ __forceinline__ void mxfp4_tile_dot_x2(const uint8_t* codes_g, const uint8_t* codes_g8,
                                                  const uint8_t* sc_g, const uint8_t* sc_g8, int nb,
                                                  const uint8_t* xb, uint32_t xss, int M, uint32_t ref_g,
                                                  uint32_t ref_g8, float (&acc_out)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  const bool xact = g < M;
  const uint8_t* xrow = xb + g * xss;
  float acc[8][4];
#pragma unroll
  for (int u = 0; u < 8; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.0f;
  for (int q = 0; q < nb / 4; q += 2) {
    uint4 A0[2], A1[2], X[2][4];
    uint32_t e0[2], e1[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int beta = 4 * (q + h) + t;
      A0[h] = lds128(codes_g + 16 * beta);
      A1[h] = lds128(codes_g8 + 16 * beta);
      e0[h] = sc_g[beta];
      e1[h] = sc_g8[beta];
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) X[h][wd] = xact ? lds128(xrow + 64 * beta + 16 * wd) : zero;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t f0 = pow2_f16x2((int)e0[h] - (int)ref_g), f1 = pow2_f16x2((int)e1[h] - (int)ref_g8);
      uint32_t hh[16], kk[16];
      const uint32_t a0w[4] = {A0[h].x, A0[h].y, A0[h].z, A0[h].w};
      const uint32_t a1w[4] = {A1[h].x, A1[h].y, A1[h].z, A1[h].w};
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        e2m1x8_to_f16x2(a0w[wd], hh[4 * wd], hh[4 * wd + 1], hh[4 * wd + 2], hh[4 * wd + 3]);
        e2m1x8_to_f16x2(a1w[wd], kk[4 * wd], kk[4 * wd + 1], kk[4 * wd + 2], kk[4 * wd + 3]);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        hh[j] = hmul2_u32(hh[j], f0);
        kk[j] = hmul2_u32(kk[j], f1);
      }
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        mma_f16(acc[4 * h + wd], hh[4 * wd], kk[4 * wd], hh[4 * wd + 1], kk[4 * wd + 1], X[h][wd].x, X[h][wd].y);
        mma_f16(acc[4 * h + wd], hh[4 * wd + 2], kk[4 * wd + 2], hh[4 * wd + 3], kk[4 * wd + 3], X[h][wd].z,
                X[h][wd].w);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    acc_out[e] = ((acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e])) + ((acc[4][e] + acc[5][e]) + (acc[6][e] + acc[7][e]));
}

// Any row shape: one group per iteration, the next group's codes and scales loaded
// while this one computes.  Same contract as mxfp4_tile_dot_x2.
__device__ __forceinline__ void mxfp4_tile_dot_x1(const uint8_t* codes_g, const uint8_t* codes_g8,
                                                  const uint8_t* sc_g, const uint8_t* sc_g8, int nb,
                                                  const uint8_t* xb, uint32_t xss, int M, uint32_t ref_g,
                                                  uint32_t ref_g8, float (&acc_out)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int nq = (nb + 3) / 4;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  const bool xact = g < M;
  const uint8_t* xrow = xb + g * xss;
  float acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.0f;
  uint4 nA0, nA1;
  uint32_t ns0, ns1;
  {
    const bool v = t < nb;
    nA0 = v ? lds128(codes_g + 16 * t) : zero;
    nA1 = v ? lds128(codes_g8 + 16 * t) : zero;
    ns0 = v ? sc_g[t] : ref_g;
    ns1 = v ? sc_g8[t] : ref_g8;
  }
  for (int q = 0; q < nq; ++q) {
    const uint4 A0 = nA0, A1 = nA1;
    const uint32_t e0 = ns0, e1 = ns1;
    const int beta = 4 * q + t;
    if (q + 1 < nq) {
      const int b2 = beta + 4;
      const bool v = b2 < nb;
      nA0 = v ? lds128(codes_g + 16 * b2) : zero;
      nA1 = v ? lds128(codes_g8 + 16 * b2) : zero;
      ns0 = v ? sc_g[b2] : ref_g;
      ns1 = v ? sc_g8[b2] : ref_g8;
    }
    const bool valid = beta < nb;
    uint4 X[4];
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) X[wd] = (xact && valid) ? lds128(xrow + 64 * beta + 16 * wd) : zero;
    const uint32_t f0 = pow2_f16x2((int)e0 - (int)ref_g), f1 = pow2_f16x2((int)e1 - (int)ref_g8);
    uint32_t h[16], k[16];
    const uint32_t a0w[4] = {A0.x, A0.y, A0.z, A0.w};
    const uint32_t a1w[4] = {A1.x, A1.y, A1.z, A1.w};
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      e2m1x8_to_f16x2(a0w[wd], h[4 * wd], h[4 * wd + 1], h[4 * wd + 2], h[4 * wd + 3]);
      e2m1x8_to_f16x2(a1w[wd], k[4 * wd], k[4 * wd + 1], k[4 * wd + 2], k[4 * wd + 3]);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      h[j] = hmul2_u32(h[j], f0);
      k[j] = hmul2_u32(k[j], f1);
    }
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      mma_f16(acc[wd], h[4 * wd], k[4 * wd], h[4 * wd + 1], k[4 * wd + 1], X[wd].x, X[wd].y);
      mma_f16(acc[wd], h[4 * wd + 2], k[4 * wd + 2], h[4 * wd + 3], k[4 * wd + 3], X[wd].z, X[wd].w);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) acc_out[e] = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
}

// One token on the CUDA cores: a single activation column leaves 7/8 of each m16n8k16
// product idle, so thread (g, t) instead multiplies its blocks t, t+4, ... of rows g
// and g+8 against the token directly -- codes widened to f16 pairs as above, exact
// f16 x f16 products summed in fp32 per block, then the block's factor
// 2^(e - 127 - sh) applied in fp32.  FAST: the caller has checked that every block's
// e - sh lies in [1, 254], so the factor is the normal number with exponent byte e - sh;
// otherwise each factor is built clamped (exact down to 2^-149, the only losses being
// block contributions outside the fp32 range).  The four t lanes then sum their
// partials, so every lane of group g returns a0 = row g, a1 = row g+8.
template <bool FAST>
__device__ __forceinline__ void mxfp4_rows_m1(const uint8_t* codes_g, const uint8_t* codes_g8, const uint8_t* sc_g,
                                              const uint8_t* sc_g8, int nb, const uint8_t* xb, int sh, float& r0,
                                              float& r1) {
  const int t = threadIdx.x & 3;
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll 2
  for (int b = t; b < nb; b += 4) {
    const uint4 X0 = lds128(xb + 64 * b), X1 = lds128(xb + 64 * b + 16);
    const uint4 X2 = lds128(xb + 64 * b + 32), X3 = lds128(xb + 64 * b + 48);
    const uint32_t xw[16] = {X0.x, X0.y, X0.z, X0.w, X1.x, X1.y, X1.z, X1.w,
                             X2.x, X2.y, X2.z, X2.w, X3.x, X3.y, X3.z, X3.w};
    const uint4 C0 = lds128(codes_g + 16 * b), C1 = lds128(codes_g8 + 16 * b);
    float f0, f1;
    if (FAST) {
      f0 = __uint_as_float((uint32_t)((int)sc_g[b] - sh) << 23);
      f1 = __uint_as_float((uint32_t)((int)sc_g8[b] - sh) << 23);
    } else {
      f0 = pow2_clamped((int)sc_g[b] - 127 - sh);
      f1 = pow2_clamped((int)sc_g8[b] - 127 - sh);
    }
    const uint32_t w0[4] = {C0.x, C0.y, C0.z, C0.w}, w1[4] = {C1.x, C1.y, C1.z, C1.w};
    uint32_t h0[16], h1[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      e2m1x8_to_f16x2(w0[k], h0[4 * k], h0[4 * k + 1], h0[4 * k + 2], h0[4 * k + 3]);
      e2m1x8_to_f16x2(w1[k], h1[4 * k], h1[4 * k + 1], h1[4 * k + 2], h1[4 * k + 3]);
    }
    float p0 = 0.0f, p1 = 0.0f, p2 = 0.0f, p3 = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      p0 = fma_f16_lo(h0[j], xw[j], p0);
      p1 = fma_f16_hi(h0[j], xw[j], p1);
      p2 = fma_f16_lo(h1[j], xw[j], p2);
      p3 = fma_f16_hi(h1[j], xw[j], p3);
    }
    a0 = fmaf(p0 + p1, f0, a0);
    a1 = fmaf(p2 + p3, f1, a1);
  }
  a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
  a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
  a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
  a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
  r0 = a0;
  r1 = a1;
}

// The clamped-factor rows (rare: block exponents outside the fast range), out of line.
__device__ __forceinline__ void mxfp4_rows_m1_safe(const uint8_t* codes_g, const uint8_t* codes_g8, const uint8_t* sc_g,
                                                const uint8_t* sc_g8, int nb, const uint8_t* xb, int sh, float& r0,
                                                float& r1) {
  mxfp4_rows_m1<false>(codes_g, codes_g8, sc_g, sc_g8, nb, xb, sh, r0, r1);
}
// A window tile whose rows span more than FOLD_SPAN scale exponents: exact per-block
// fp32 scaling, one token at a time (rare; out of line).
__device__ __forceinline__ void mxfp4_tile_dot_wide(const uint8_t* codes_g, const uint8_t* codes_g8, const uint8_t* sc_g,
                                                 const uint8_t* sc_g8, int nb, const uint8_t* xb, uint32_t xss, int M,
                                                 const int* xsh, float* c) {
  const int t = threadIdx.x & 3;
  c[0] = c[1] = c[2] = c[3] = 0.0f;
  for (int m = 0; m < M; ++m) {
    float r0, r1;
    mxfp4_rows_m1<false>(codes_g, codes_g8, sc_g, sc_g8, nb, xb + m * xss, xsh[m], r0, r1);
    if (m == 2 * t) {
      c[0] = r0;
      c[2] = r1;
    } else if (m == 2 * t + 1) {
      c[1] = r0;
      c[3] = r1;
    }
  }
}

// A window (M >= 2) tile on the warp tensor core; see mxfp4_tile_dot.
__device__ __forceinline__ void mxfp4_tile_dot_win(const uint8_t* codes_g, const uint8_t* codes_g8,
                                                   const uint8_t* sc_g, const uint8_t* sc_g8, int nb,
                                                   const uint8_t* xb, uint32_t xss, int M, const int* xsh,
                                                   float (&c)[4]) {
  const int t = threadIdx.x & 3;
  uint32_t mx_g, mx_g8, mn_g, mn_g8;
  row_scale_range(sc_g, sc_g8, nb, mx_g, mx_g8, mn_g, mn_g8);
  const bool fold = __all_sync(0xffffffffu, (int)(mx_g - mn_g) <= FOLD_SPAN && (int)(mx_g8 - mn_g8) <= FOLD_SPAN);
  if (!fold) {
    mxfp4_tile_dot_wide(codes_g, codes_g8, sc_g, sc_g8, nb, xb, xss, M, xsh, c);
    return;
  }
  float acc[4];
  if ((nb & 7) == 0 && ((reinterpret_cast<uintptr_t>(sc_g) | reinterpret_cast<uintptr_t>(sc_g8)) & 3u) == 0)
    mxfp4_tile_dot_x2(codes_g, codes_g8, sc_g, sc_g8, nb, xb, xss, M, mx_g, mx_g8, acc);
  else
    mxfp4_tile_dot_x1(codes_g, codes_g8, sc_g, sc_g8, nb, xb, xss, M, mx_g, mx_g8, acc);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int tok = 2 * t + (e & 1);
    const int ref = (int)(e < 2 ? mx_g : mx_g8);
    // 2^(ref - 127 - sh) as two exact power-of-two factors (|exponent| <= 290; a result
    // below 2^-252 of the fp32 sum is zero in fp32 anyway)
    const int d = tok < M ? max(ref - 127 - xsh[tok], -252) : 0;
    c[e] = tok < M ? mul_pow2(acc[e], d) : 0.0f;
  }
}

// The warp's 16-row MXFP4 tile (rows g and g+8 of each lane group, nb scale blocks of
// 32) against M <= 8 f16 activation rows xb (stride xss, token n scaled by 2^xsh[n]).
// Returns the products in true units, c as the m16n8 C layout: c0 (row g, token 2t),
// c1 (row g, token 2t+1), c2 (row g+8, token 2t), c3 (row g+8, token 2t+1); for M = 1
// every lane of group g returns c0 = row g, c2 = row g+8 (c1 = c3 = 0).
// Paths (warp-uniform): M = 1 on the CUDA cores; M > 1 on the warp tensor core with
// the scales folded into the codes when every row's scale span is at most FOLD_SPAN,
// otherwise token by token on the CUDA cores (exact for any E8M0 scales).
__device__ __forceinline__ void mxfp4_tile_dot(const uint8_t* codes_g, const uint8_t* codes_g8,
                                               const uint8_t* sc_g, const uint8_t* sc_g8, int nb,
                                               const uint8_t* xb, uint32_t xss, int M, const int* xsh,
                                               float (&c)[4]) {
  if (M > 1) {
    mxfp4_tile_dot_win(codes_g, codes_g8, sc_g, sc_g8, nb, xb, xss, M, xsh, c);
    return;
  }
  uint32_t mx_g, mx_g8, mn_g, mn_g8;
  row_scale_range(sc_g, sc_g8, nb, mx_g, mx_g8, mn_g, mn_g8);
  const int sh = xsh[0];
  // the fast factor needs 1 <= e - sh <= 254 for every block of both rows
  const bool fast = __all_sync(0xffffffffu, (int)min(mn_g, mn_g8) - sh >= 1 && (int)max(mx_g, mx_g8) - sh <= 254);
  float r0, r1;
  if (fast)
    mxfp4_rows_m1<true>(codes_g, codes_g8, sc_g, sc_g8, nb, xb, sh, r0, r1);
  else
    mxfp4_rows_m1_safe(codes_g, codes_g8, sc_g, sc_g8, nb, xb, sh, r0, r1);
  c[0] = r0;
  c[1] = 0.0f;
  c[2] = r1;
  c[3] = 0.0f;
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
  size_t b = 16 * (size_t)(H / 2) + 16 * (size_t)(H / 32);  // contiguous rows: 4 bulk copies per item
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline size_t e13_fixed_bytes(int H) { return 128 + 8 * (size_t)padded_stride(2u * H); }

__global__ void __launch_bounds__(EXPERT_THREADS, 1) k_experts13(E13Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ int s_sh[MAX_M];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, H = p.H, I = p.I, S = p.stages;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t cs = H / 2;
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
        bulk_g2s(st, p.w13c + (e2I + r0) * rowb, 8 * rowb, &full[s], pol);
        bulk_g2s(st + 8 * cs, p.w13c + (e2I + I + r0) * rowb, 8 * rowb, &full[s], pol);
        bulk_g2s(st + 16 * cs, p.w13s + (e2I + r0) * (H / 32), scb, &full[s], pol);
        bulk_g2s(st + 16 * cs + scb, p.w13s + (e2I + I + r0) * (H / 32), scb, &full[s], pol);
      }
      // Drain: the last uses of each stage must have landed before the block exits.
      for (int i = (nloc > S ? nloc - S : 0); i < nloc; ++i) mbar_wait(&full[i % S], (i / S) & 1, p.status);
    }
    return;
  }

  stage_x_f16(p.x, M, H, xs, xss, s_sh);
  for (int i = warp; i < nloc; i += N_CONSUMERS) {
    const int s = i % S;
    if (!mbar_wait(&full[s], (i / S) & 1, p.status)) return;
    const long long item = start + i;
    const int u = (int)(item / ntile), r0 = 8 * (int)(item % ntile);
    const uint8_t* st = stages + s * sbytes;
    float c[4];
    mxfp4_tile_dot(st + g * cs, st + (8 + g) * cs, st + 16 * cs + g * (H / 32), st + 16 * cs + (8 + g) * (H / 32),
                   nb, xs, xss, M, s_sh, c);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = 2 * t + e;  // rows g (gate) and g+8 (up) of intermediate index r0 + g
      if (tok < M) p.a_routed[((size_t)u * M + tok) * I + r0 + g] = silu_f32(c[e]) * c[2 + e];
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
  size_t r = 16 * (size_t)(I / 2) + 16 * (size_t)(I / 32);
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

__global__ void __launch_bounds__(EXPERT_THREADS, 1) k_experts2(E2Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ int s_ash[E2_MAX_LOCAL_SLOTS][MAX_M];  // f16 shift of each staged routed activation
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, H = p.H, I = p.I, Is = p.Is, S = p.stages;
  const uint32_t ass = padded_stride(2u * I);
  const uint32_t sss = Is > 0 ? padded_stride(2u * Is) : 0u;
  const uint32_t cs = I / 2;
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
          bulk_g2s(st, p.w2c + (eH + h0) * rowb, 16 * rowb, &full[s], pol);
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
      for (int i = lane; i < I / 2; i += 32) {
        __half2 v = __floats2half2_rn(0.0f, 0.0f);
        if (live) v = __floats2half2_rn(mul_pow2(src[2 * i], sh), mul_pow2(src[2 * i + 1], sh));
        *reinterpret_cast<__half2*>(dst + 4 * i) = v;
      }
      if (lane == 0) s_ash[uu][tok] = sh;
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
      float c[4];
      mxfp4_tile_dot(st + g * cs, st + (8 + g) * cs, st + 16 * cs + g * (I / 32), st + 16 * cs + (8 + g) * (I / 32),
                     nb, af + (size_t)uu * MAX_M * ass, ass, M, s_ash[uu], c);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = 2 * t + e;
        if (tok < M) {
          const float wt = P.w[u][tok];
          if (wt != 0.0f) {
            atomicAdd(p.out + (size_t)tok * H + h0 + g, c[e] * wt);
            atomicAdd(p.out + (size_t)tok * H + h0 + g + 8, c[2 + e] * wt);
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
