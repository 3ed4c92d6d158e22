// lmhead_kernels.cuh -- FP8 (e4m3) LM head: online quantisation and the GEMV + argmax.
//
// Source: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
// 三种方法), section 方法/产品要点 item 2: the 157,184 x 2,560 vocabulary projection is
// stored BF16 in the checkpoint and quantised to FP8 when the head is constructed,
// which halves the bytes every generated token has to read.
//
// Quantisation (once): one fp32 scale per output row, s = amax/448, codes =
// e4m3 RNE-saturating of w/s (IEEE fp32 divisions, hardware cvt).
// GEMV: rows stream HBM -> shared memory through bulk copies; e4m3 codes widen to
// f16 exactly (hardware cvt), the warp tensor-core product accumulates in fp32,
// the row scale and the activation's power-of-two range shift are applied in
// the epilogue.  The argmax is folded in: per-thread best -> warp -> block ->
// one 64-bit atomicMax per token (value key << 32 | ~index, so equal values keep
// the lowest index) -> the last block converts the keys to indices.
#pragma once

#include "decode_kernels.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// k_lm_quantize: one warp per row
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_lm_quantize(const __nv_bfloat16* __restrict__ w, int V, int H,
                                                     uint8_t* __restrict__ q, float* __restrict__ rs) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= V) return;
  const __nv_bfloat16* wr = w + row * H;
  float amax = 0.0f;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = *reinterpret_cast<const uint4*>(wr + 8 * c);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__low2float(b[j])));
      amax = fmaxf(amax, fabsf(__high2float(b[j])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (lane == 0) rs[row] = s;
  uint8_t* qr = q + row * H;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = *reinterpret_cast<const uint4*>(wr + 8 * c);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t pr = f32x2_to_e4m3x2(__fdiv_rn(__low2float(b[j]), s), __fdiv_rn(__high2float(b[j]), s));
      if (j < 2)
        lo |= pr << (16 * j);
      else
        hi |= pr << (16 * (j - 2));
    }
    *reinterpret_cast<uint2*>(qr + 8 * c) = make_uint2(lo, hi);
  }
}

// ---------------------------------------------------------------------------
// k_lm_gemv: 16-row tiles, producer warp + 4 consumer warps
// ---------------------------------------------------------------------------
struct LMParams {
  const __nv_bfloat16* x;  // [M][H]
  int M, V, H;
  const uint8_t* w;        // [V][H] e4m3
  const float* rs;         // [V]
  float* logits;           // [M][V] or null
  int32_t* argmax;         // [M]
  unsigned long long* keys;  // [MAX_M], zero on entry
  unsigned* counter;         // zero on entry
  int* status;
  int stages;
  const int32_t* drafts;     // optional [M-1]: draft tokens of a verify window (MTP)
  int32_t* accept;           // [1 + M] when drafts: accepted count, then the accepted tokens
};

// Multi-token-prediction verify (the window holds the last accepted token and M - 1
// drafts; the head's argmax at position t predicts the token after it): draft t + 1
// is accepted while it equals the argmax at t, and the head's own token at the first
// mismatch (or after the last draft) is accepted with them.  out[0] = accepted count
// (1..M), out[1..] = the accepted tokens.
__device__ __forceinline__ void mtp_accept(const int32_t* argmax, const int32_t* drafts, int M, int32_t* out) {
  int n = 0;
  while (n < M - 1 && drafts[n] == argmax[n]) {
    out[1 + n] = drafts[n];
    ++n;
  }
  out[1 + n] = argmax[n];
  out[0] = n + 1;
}

// 8-row tiles (one contiguous bulk copy each) through a ring of LM_STAGES stages, one
// producer warp and LM_CONSUMERS consumer warps taking tiles round-robin.  A tile fills
// rows 0-7 of the m16n8k16 product (rows 8-15 are zero: the head is bound by its
// weight bytes; eight warps keep the e4m3 widening off the critical path).
constexpr int LM_CONSUMERS = 8;
constexpr int LM_THREADS = 32 * (LM_CONSUMERS + 1);
constexpr int LM_STAGES = 8;
static_assert(LM_STAGES == MAX_STAGES && LM_STAGES >= LM_CONSUMERS, "stage barriers: one stage per consumer warp in flight");
__host__ __device__ inline size_t lm_stage_bytes(int H) {
  size_t b = 8 * (size_t)H;  // 8 contiguous rows: one bulk copy per tile
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline size_t lm_fixed_bytes(int H) { return 128 + 8 * (size_t)padded_stride(2u * H); }

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  return ((unsigned long long)float_key(v) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}

__global__ void __launch_bounds__(LM_THREADS, 1) k_lm_gemv(LMParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_sh[MAX_M];
  __shared__ float s_inv[2][MAX_M];  // 2^-sh as two exact factors
  __shared__ unsigned long long s_best[LM_CONSUMERS][MAX_M];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, V = p.V, H = p.H, S = p.stages;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t ls = H;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + LM_STAGES;
  uint8_t* xs = smem + 128;
  uint8_t* stages = smem + lm_fixed_bytes(H);
  const size_t sbytes = lm_stage_bytes(H);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const long long T = (V + 7) / 8;
  const long long start = T * blockIdx.x / gridDim.x;
  const long long end = T * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(end - start);

  if (warp == LM_CONSUMERS) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int i = 0; i < nloc; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, p.status)) break;
        const long long v0 = (start + i) * 8;
        const int nrows = (int)min(8LL, (long long)V - v0);
        uint8_t* st = stages + s * sbytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)nrows * H);
        bulk_g2s(st, p.w + (size_t)v0 * H, (uint32_t)nrows * H, &full[s], pol);
      }
      for (int i = (nloc > S ? nloc - S : 0); i < nloc; ++i) mbar_wait(&full[i % S], (i / S) & 1, p.status);
    }
    return;
  }

  stage_x_f16<LM_CONSUMERS>(p.x, M, H, xs, xss, s_sh);
  if (tid < MAX_M) {
    const int k = -s_sh[tid], k1 = k / 2;
    s_inv[0][tid] = exp2i(k1);
    s_inv[1][tid] = exp2i(k - k1);
  }
  named_barrier(1, 32 * LM_CONSUMERS);
  unsigned long long bestA = 0ull, bestB = 0ull;  // tokens 2t and 2t+1
  const int ta = 2 * t, tb = 2 * t + 1;
  const bool xact = g < M;
  for (int i = warp; i < nloc; i += LM_CONSUMERS) {
    const int s = i % S;
    if (!mbar_wait(&full[s], (i / S) & 1, p.status)) return;
    const long long v0 = (start + i) * 8;
    const uint8_t* row = stages + s * sbytes + g * ls;
    float c4[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) c4[u][0] = c4[u][1] = c4[u][2] = c4[u][3] = 0.0f;
#pragma unroll 2
    for (int j = 0; j < H / 64; ++j) {
      const uint4 A0 = lds128(row + 64 * j + 16 * t);
      const uint4 zero = make_uint4(0, 0, 0, 0);
      const uint4 X0 = xact ? lds128(xs + g * xss + 2 * (64 * j + 16 * t)) : zero;
      const uint4 X1 = xact ? lds128(xs + g * xss + 2 * (64 * j + 16 * t) + 16) : zero;
      uint32_t P[8];
      e4m3x4_to_f16x2(A0.x, P[0], P[1]);
      e4m3x4_to_f16x2(A0.y, P[2], P[3]);
      e4m3x4_to_f16x2(A0.z, P[4], P[5]);
      e4m3x4_to_f16x2(A0.w, P[6], P[7]);
      const uint32_t X[8] = {X0.x, X0.y, X0.z, X0.w, X1.x, X1.y, X1.z, X1.w};
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) mma_f16(c4[s4], P[2 * s4], 0u, P[2 * s4 + 1], 0u, X[2 * s4], X[2 * s4 + 1]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    const long long va = v0 + g;
    const float rsa = va < V ? __ldg(p.rs + va) : 0.0f;
    if (va < V) {
      if (ta < M) {
        const float c = (c4[0][0] + c4[1][0]) + (c4[2][0] + c4[3][0]);
        const float la = ((c * s_inv[0][ta]) * s_inv[1][ta]) * rsa;
        if (p.logits) p.logits[(size_t)ta * V + va] = la;
        bestA = max(bestA, argmax_key(la, (int)va));
      }
      if (tb < M) {
        const float c = (c4[0][1] + c4[1][1]) + (c4[2][1] + c4[3][1]);
        const float lb = ((c * s_inv[0][tb]) * s_inv[1][tb]) * rsa;
        if (p.logits) p.logits[(size_t)tb * V + va] = lb;
        bestB = max(bestB, argmax_key(lb, (int)va));
      }
    }
  }
  // lanes with the same t hold the same tokens: reduce over g
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    bestA = max(bestA, __shfl_xor_sync(0xffffffffu, bestA, o));
    bestB = max(bestB, __shfl_xor_sync(0xffffffffu, bestB, o));
  }
  if (g == 0) {
    s_best[warp][ta] = bestA;
    s_best[warp][tb] = bestB;
  }
  named_barrier(1, 32 * LM_CONSUMERS);
  if (warp == 0 && lane < M) {
    unsigned long long b = 0ull;
    for (int w = 0; w < LM_CONSUMERS; ++w) b = max(b, s_best[w][lane]);
    if (b) atomicMax(p.keys + lane, b);
  }
  __threadfence();
  named_barrier(1, 32 * LM_CONSUMERS);
  if (tid == 0) s_last = (atomicAdd(p.counter, 1u) == gridDim.x - 1);
  named_barrier(1, 32 * LM_CONSUMERS);
  if (s_last) {
    __threadfence();
    if (tid < M) {
      const unsigned long long k = atomicExch(p.keys + tid, 0ull);
      p.argmax[tid] = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
    }
    if (tid == 0) *p.counter = 0u;
    if (p.drafts) {
      named_barrier(1, 32 * LM_CONSUMERS);
      if (tid == 0) mtp_accept(p.argmax, p.drafts, M, p.accept);
    }
  }
}

// ---------------------------------------------------------------------------
// k_lm_gemv_bf16: the same head with the BF16 weights it is quantised from -- the
// comparison the FP8 head is measured against (twice the bytes per logit).  The FP8
// head's pipeline: a producer warp bulk-copies 8-row tiles (contiguous, 16 H bytes)
// into a ring of stages, four consumer warps take tiles round-robin.  A tile fills
// rows 0-7 of the m16n8k16 product (rows 8-15 are zero: the head is bound by its
// weight bytes, not by the tensor core); x stays bf16, so the products are exact.
// ---------------------------------------------------------------------------
__host__ __device__ inline size_t lmb_stage_bytes(int H) {
  size_t b = 8 * 2 * (size_t)H;  // 8 contiguous bf16 rows: one bulk copy per tile
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline size_t lmb_fixed_bytes(int H) { return 128 + MAX_M * (size_t)padded_stride(2u * H); }

__global__ void __launch_bounds__(EXPERT_THREADS, 1) k_lm_gemv_bf16(LMParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ unsigned long long s_best[N_CONSUMERS][MAX_M];
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, V = p.V, H = p.H, S = p.stages;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t ls = 2u * H;
  const __nv_bfloat16* w = reinterpret_cast<const __nv_bfloat16*>(p.w);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + MAX_STAGES;
  uint8_t* xs = smem + 128;
  uint8_t* stages = smem + lmb_fixed_bytes(H);
  const size_t sbytes = lmb_stage_bytes(H);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const long long T = (V + 7) / 8;
  const long long start = T * blockIdx.x / gridDim.x;
  const long long end = T * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(end - start);

  if (warp == N_CONSUMERS) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int i = 0; i < nloc; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, p.status)) break;
        const long long v0 = (start + i) * 8;
        const int nrows = (int)min(8LL, (long long)V - v0);
        mbar_arrive_expect_tx(&full[s], (uint32_t)nrows * ls);
        bulk_g2s(stages + s * sbytes, w + (size_t)v0 * H, (uint32_t)nrows * ls, &full[s], pol);
      }
      for (int i = (nloc > S ? nloc - S : 0); i < nloc; ++i) mbar_wait(&full[i % S], (i / S) & 1, p.status);
    }
    return;
  }

  // activation rows as bf16 (the MMA's B operand), zero rows beyond M
  for (int i = tid; i < MAX_M * (H / 8); i += 32 * N_CONSUMERS) {
    const int tok = i / (H / 8), c = i % (H / 8);
    const uint4 v = tok < M ? *reinterpret_cast<const uint4*>(p.x + (size_t)tok * H + 8 * c) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(xs + tok * xss + 16 * c) = v;
  }
  named_barrier(1, 32 * N_CONSUMERS);
  unsigned long long bestA = 0ull, bestB = 0ull;  // tokens 2t and 2t+1
  const int ta = 2 * t, tb = 2 * t + 1;
  for (int i = warp; i < nloc; i += N_CONSUMERS) {
    const int s = i % S;
    if (!mbar_wait(&full[s], (i / S) & 1, p.status)) return;
    const long long v0 = (start + i) * 8;
    const uint8_t* row = stages + s * sbytes + g * ls;
    float c4[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) c4[u][0] = c4[u][1] = c4[u][2] = c4[u][3] = 0.0f;
#pragma unroll 2
    for (int j = 0; j < H / 64; ++j) {
      // this thread's 16 columns of the chunk: 64j + 16t .. +15 (two 16-byte pieces)
      const uint4 A0 = lds128(row + 128 * j + 32 * t), A0b = lds128(row + 128 * j + 32 * t + 16);
      const uint4 X0 = lds128(xs + g * xss + 2 * (64 * j + 16 * t));
      const uint4 X1 = lds128(xs + g * xss + 2 * (64 * j + 16 * t) + 16);
      const uint32_t P[8] = {A0.x, A0.y, A0.z, A0.w, A0b.x, A0b.y, A0b.z, A0b.w};
      const uint32_t X[8] = {X0.x, X0.y, X0.z, X0.w, X1.x, X1.y, X1.z, X1.w};
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) mma_bf16(c4[s4], P[2 * s4], 0u, P[2 * s4 + 1], 0u, X[2 * s4], X[2 * s4 + 1]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    const float ca = (c4[0][0] + c4[1][0]) + (c4[2][0] + c4[3][0]);
    const float cb = (c4[0][1] + c4[1][1]) + (c4[2][1] + c4[3][1]);
    const long long va = v0 + g;
    if (va < V) {
      if (ta < M) {
        if (p.logits) p.logits[(size_t)ta * V + va] = ca;
        bestA = max(bestA, argmax_key(ca, (int)va));
      }
      if (tb < M) {
        if (p.logits) p.logits[(size_t)tb * V + va] = cb;
        bestB = max(bestB, argmax_key(cb, (int)va));
      }
    }
  }
  // lanes with the same t hold the same tokens: reduce over g
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    bestA = max(bestA, __shfl_xor_sync(0xffffffffu, bestA, o));
    bestB = max(bestB, __shfl_xor_sync(0xffffffffu, bestB, o));
  }
  if (g == 0) {
    s_best[warp][ta] = bestA;
    s_best[warp][tb] = bestB;
  }
  named_barrier(1, 32 * N_CONSUMERS);
  if (warp == 0 && lane < M) {
    unsigned long long b = 0ull;
    for (int w2 = 0; w2 < N_CONSUMERS; ++w2) b = max(b, s_best[w2][lane]);
    if (b) atomicMax(p.keys + lane, b);
  }
  __threadfence();
  named_barrier(1, 32 * N_CONSUMERS);
  if (tid == 0) s_last = (atomicAdd(p.counter, 1u) == gridDim.x - 1);
  named_barrier(1, 32 * N_CONSUMERS);
  if (s_last) {
    __threadfence();
    if (tid < M) {
      const unsigned long long k = atomicExch(p.keys + tid, 0ull);
      p.argmax[tid] = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
    }
    if (tid == 0) *p.counter = 0u;
  }
}

}  // namespace moe
