// sample_kernels.cuh -- temperature / top-k / top-p sampling of one token per row of
// fp32 logits, the uniform draw given per row.
//
// Source: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
// 三种方法), the serving settings it reports (temperature, top-k 29, top-p 0.95).
// Reading: z = logits / T; S = the top_k largest logits (ties to the lower index);
// p = softmax of z over S; in that order the nucleus N is the shortest prefix with
// sum p >= top_p; the sample is the first token of N whose cumulative p / sum_N p
// exceeds u (the last of N if rounding leaves none).
//
// One block per row.  The top_k-th largest logit comes from a 4-pass radix select
// on order-preserving 32-bit keys (8 bits a pass, 256-bin shared histogram); the
// keys at or above it are gathered (at most SAMPLE_CAND of them), sorted by (key
// desc, index asc) with a block bitonic sort, and warp 0 takes the first top_k
// through the softmax, the nucleus and the draw.
#pragma once

#include "decode_kernels.cuh"

namespace moe {

constexpr int SAMPLE_THREADS = 1024;
constexpr int SAMPLE_CAND = 1024;  // candidates kept: top_k plus ties at the k-th value
constexpr int SAMPLE_MAX_K = 32;

__global__ void __launch_bounds__(SAMPLE_THREADS) k_sample(const float* __restrict__ logits, int V, float temperature,
                                                          int top_k, float top_p, const float* __restrict__ u,
                                                          int32_t* __restrict__ ids) {
  __shared__ unsigned s_hist[256];
  __shared__ unsigned s_prefix, s_need, s_ncand;
  __shared__ unsigned long long s_cand[SAMPLE_CAND];  // key << 32 | ~index: descending = (key desc, index asc)
  const int tid = threadIdx.x, lane = tid & 31;
  const float* lr = logits + (size_t)blockIdx.x * V;

  // ---- radix select of the top_k-th largest key ----
  if (tid == 0) {
    s_prefix = 0u;
    s_need = (unsigned)top_k;  // rank still to find inside the current prefix (from the top)
  }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const unsigned pmask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = tid; i < 256; i += SAMPLE_THREADS) s_hist[i] = 0u;
    __syncthreads();
    const unsigned prefix = s_prefix;
    for (int i = tid; i < V; i += SAMPLE_THREADS) {
      const unsigned k = float_key(lr[i]);
      if ((k & pmask) == prefix) atomicAdd(&s_hist[(k >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned need = s_need, d = 255;
      while (true) {  // largest digit whose cumulative count from the top reaches need
        const unsigned c = s_hist[d];
        if (c >= need || d == 0) break;
        need -= c;
        --d;
      }
      s_prefix = prefix | (d << shift);
      s_need = need;
    }
    __syncthreads();
  }
  const unsigned kth = s_prefix;  // key of the top_k-th largest logit

  // ---- gather keys >= kth, sort by (key desc, index asc) ----
  if (tid == 0) s_ncand = 0u;
  for (int i = tid; i < SAMPLE_CAND; i += SAMPLE_THREADS) s_cand[i] = 0ull;
  __syncthreads();
  for (int i = tid; i < V; i += SAMPLE_THREADS) {
    const unsigned k = float_key(lr[i]);
    if (k >= kth) {
      const unsigned slot = atomicAdd(&s_ncand, 1u);
      if (slot < SAMPLE_CAND) s_cand[slot] = ((unsigned long long)k << 32) | (0xFFFFFFFFu - (unsigned)i);
    }
  }
  __syncthreads();
  for (unsigned size = 2; size <= SAMPLE_CAND; size <<= 1) {  // bitonic sort, descending
    for (unsigned stride = size >> 1; stride > 0; stride >>= 1) {
      for (unsigned i = tid; i < SAMPLE_CAND; i += SAMPLE_THREADS) {
        const unsigned j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = s_cand[i], b = s_cand[j];
          if (desc ? (a < b) : (a > b)) {
            s_cand[i] = b;
            s_cand[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }

  // ---- softmax over the top_k, nucleus, draw (warp 0, one candidate per lane) ----
  if (tid < 32) {
    const bool in = lane < top_k;
    const unsigned long long c = s_cand[lane];
    const float l = in ? key_float((unsigned)(c >> 32)) : 0.0f;
    const int idx = (int)(0xFFFFFFFFu - (unsigned)(c & 0xFFFFFFFFull));
    const float z = l / temperature;
    const float z0 = __shfl_sync(0xffffffffu, z, 0);
    const float e = in ? expf(z - z0) : 0.0f;
    float den = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float pj = e / den;
    float cum = pj;  // inclusive prefix sum in sorted order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, cum, o);
      if (lane >= o) cum += v;
    }
    // nucleus size n: the first lane whose prefix reaches top_p, plus one
    const unsigned reach = __ballot_sync(0xffffffffu, in && cum >= top_p);
    const int n = reach ? (__ffs(reach)) : top_k;
    const float mass = __shfl_sync(0xffffffffu, cum, n - 1);
    const unsigned over = __ballot_sync(0xffffffffu, lane < n && cum / mass > u[blockIdx.x]);
    const int pick = over ? (__ffs(over) - 1) : n - 1;
    const int chosen = __shfl_sync(0xffffffffu, idx, pick);
    if (lane == 0) ids[blockIdx.x] = chosen;
  }
}

}  // namespace moe
