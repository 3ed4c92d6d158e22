// step_kernel.cuh -- the whole decode step (all MoE layers) as one persistent kernel.
//
// One block per SM for the whole step (cooperative launch: all blocks co-resident).
// Warp 4 of each block is the producer: one thread walks this block's sequence of
// weight tiles for every layer and moves them HBM -> shared memory with bulk copies
// (TMA engine) into a ring of stages; it also issues L2 prefetches for tiles whose
// identity is already known -- the next layer's router/shared-expert tiles and this
// layer's shared-W2 tiles while the layer waits on its router, and a sliding window
// of routed tiles once the routing is known -- so HBM keeps streaming across the
// layer's dependency points.  Warps 0-3 consume the ring in order (item i -> warp
// i % 4) and synchronise only where the data forces it:
//   router tiles complete  -> every block takes the top-k itself (same code, same bits)
//   expert u's W13 complete -> its W2 tiles may start (per-expert counter)
//   shared W13 complete    -> the shared W2 tiles may start
//   residual h complete    -> the next layer's RMSNorm may start (grid-wide counter)
// Every wait is a bounded spin (abort flag + status word after WAIT_LIMIT_NS), so a
// fault in one block ends the step with MOE_ERR_TIMEOUT instead of a hang.
//
// Per layer, in ring order, block c processes (every item one or a few contiguous
// bulk copies -- the copy count, not the byte count, is what a bulk-copy engine
// pays for):
//   A: router items (4 experts' rows) and shared-W13 items (2 gate + 2 up rows),
//      fixed assignment j = c, c+G, ...; weight rows are the MMA's N operand and
//      the tokens its M operand, so one warp covers the full K of its 4 rows.
//   B: routed W13 items (distinct expert, 8 gate + 8 up rows), a contiguous range.
//   C: routed W2 items (distinct expert, 16 output rows), a contiguous range, then
//      shared-W2 items (4 output rows), fixed assignment.
// Sources: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
// 三种方法), 事件概述或研究问题 (batch-1 decode bound by weight reads; 8 of 512 experts
// + 1 shared) and 方法/产品要点 items 1 and 3.
#pragma once

#include "decode_kernels.cuh"

namespace moe {

constexpr int STEP_MAX_LAYERS = 64;
constexpr int STEP_THREADS = 32 * (N_CONSUMERS + 1);
constexpr int CTR_ROUTER = 0, CTR_SHARED = 1, CTR_H = 2, CTR_EXP = 4;
constexpr int CTR_PER_LAYER = CTR_EXP + MAX_SLOTS;
constexpr int STEP_PREFETCH_AHEAD = 8;  // routed items prefetched into L2 ahead of the ring

struct LayerPtrs {
  const __nv_bfloat16* wr;
  const uint8_t* w13c;
  const uint8_t* w13s;
  const uint8_t* w2c;
  const uint8_t* w2s;
  const __nv_bfloat16* sw13;
  const __nv_bfloat16* sw2;
};

struct StepParams {
  int L, M, H, I, E, k, Is;
  float eps;
  int stages;
  uint32_t act_bytes;
  const __nv_bfloat16* x_in;  // [M][H]
  float* h;                   // [M][H] residual stream
  __nv_bfloat16* x_final;     // [M][H] LM-head input
  float* logits;              // [M][E]
  float* a_shared;            // [M][Is]
  float* a_routed;            // [MAX_SLOTS][M][I]
  unsigned* ctr;              // [L][CTR_PER_LAYER], zero on entry
  int* status;
  __nv_bfloat16* x_trace;
  float* h_trace;
  int32_t* ids_trace;
  float* w_trace;
  unsigned long long* timeline;  // optional [2][L][16] %globaltimer stamps (blocks 0 and G-1)
  LayerPtrs layer[STEP_MAX_LAYERS];
};

// Profiling stamp: block 0 and the last block record %globaltimer at phase
// boundaries (slots 0-11 by consumer thread 0, 12-15 by producer lane 0).
__device__ __forceinline__ void stamp(const StepParams& p, int l, int slot) {
  if (!p.timeline) return;
  const bool first = blockIdx.x == 0, last = blockIdx.x == gridDim.x - 1;
  if (!first && !last) return;
  const int tid = threadIdx.x;
  if (tid != 0 && tid != 32 * N_CONSUMERS) return;
  p.timeline[((size_t)(last ? 1 : 0) * p.L + l) * 16 + slot] = globaltimer_ns();
}
// Profiling: block 0's first STEP_ITEM_LOG ring items -- (issued, data ready, done)
// stamps after the [2][L][16] phase stamps.
constexpr int STEP_ITEM_LOG = 4096;
__device__ __forceinline__ void item_stamp(const StepParams& p, long long i, int which) {
  if (!p.timeline || blockIdx.x != 0 || i >= STEP_ITEM_LOG || (threadIdx.x & 31) != 0) return;
  p.timeline[(size_t)2 * p.L * 16 + (size_t)i * 4 + which] = globaltimer_ns();
}

// Stage geometry shared by host and device: the largest item -- 4 bf16 rows of H
// (router / shared W13), 16 MXFP4 rows of H + scales (routed W13), 16 MXFP4 rows of
// I + scales (routed W2), 4 bf16 rows of Is (shared W2).
__host__ __device__ inline size_t step_stage_bytes(int H, int I, int Is) {
  size_t b = 8 * (size_t)H;
  const size_t b13 = 8 * (size_t)H + (size_t)H / 2, b2 = 8 * (size_t)I + (size_t)I / 2, bs = 8 * (size_t)Is;
  if (b13 > b) b = b13;
  if (b2 > b) b = b2;
  if (bs > b) b = bs;
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline uint32_t step_act_bytes(int M, int H, int I, int Is) {
  const uint32_t xs = 2u * M * padded_stride(2u * H);  // bf16 rows (A phase) + f16 rows (B phase)
  const uint32_t c = 2u * M * (Is > 0 ? padded_stride(2u * Is) : 0u) + (uint32_t)N_CONSUMERS * M * padded_stride(2u * I);
  const uint32_t b = xs > c ? xs : c;
  return (b + 127) / 128 * 128;
}
constexpr size_t STEP_FIXED = 256;  // mbarriers

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_volatile_i32(const int* p) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void signal_counter(unsigned* c) {
  __threadfence();
  atomicAdd(c, 1u);
}

// Bounded spin until *c >= target.  Gives up (abort flag + status) after the time
// limit or as soon as another block has reported a failure.
__device__ __noinline__ bool wait_counter(const unsigned* c, unsigned target, int* status, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (ld_acquire_u32(c) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    __nanosleep(40);
    if (ld_acquire_u32(c) >= target) return true;
    if (*abort_flag) return false;
    if (ld_volatile_i32(status) != 0 || globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
      atomicCAS(status, 0, DEV_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}
// mbarrier wait that also honours the block's abort flag.
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
      atomicCAS(status, 0, DEV_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// the per-layer work list of one block
// ---------------------------------------------------------------------------
enum : int { IT_A = 0, IT_B = 1, IT_CR = 2, IT_CS = 3 };

struct Item {
  int type;
  int a, b;  // A: item j;  B: slot, r0;  CR: slot, h0;  CS: first row
};

struct Work {
  int nA;             // A items of this block
  long long b0, nB;   // routed W13 range
  long long c0, nC;   // routed W2 range
  int nS;             // shared-W2 items of this block
  __device__ void init_A(const StepParams& p) {
    const int c = blockIdx.x, G = gridDim.x;
    const int TA = p.E / 4 + p.Is / 2;
    nA = c < TA ? (TA - 1 - c) / G + 1 : 0;
    const int TS = p.Is > 0 ? p.H / 4 : 0;
    nS = c < TS ? (TS - 1 - c) / G + 1 : 0;
    nB = nC = 0;
    b0 = c0 = 0;
  }
  __device__ void init_routed(const StepParams& p, int n_unique) {
    const long long c = blockIdx.x, G = gridDim.x;
    const long long TB = (long long)n_unique * (p.I / 8);
    b0 = TB * c / G;
    nB = TB * (c + 1) / G - b0;
    const long long TC = (long long)n_unique * (p.H / 16);
    c0 = TC * c / G;
    nC = TC * (c + 1) / G - c0;
  }
  __device__ Item at(const StepParams& p, int r) const {
    Item it;
    if (r < nA) {
      it.type = IT_A;
      it.a = blockIdx.x + r * gridDim.x;
      it.b = 0;
      return it;
    }
    r -= nA;
    if (r < nB) {
      const long long x = b0 + r;
      it.type = IT_B;
      it.a = (int)(x / (p.I / 8));
      it.b = 8 * (int)(x % (p.I / 8));
      return it;
    }
    r -= (int)nB;
    if (r < nC) {
      const long long x = c0 + r;
      it.type = IT_CR;
      it.a = (int)(x / (p.H / 16));
      it.b = 16 * (int)(x % (p.H / 16));
      return it;
    }
    r -= (int)nC;
    it.type = IT_CS;
    it.a = 4 * (blockIdx.x + r * gridDim.x);
    it.b = 0;
    return it;
  }
};

// ---------------------------------------------------------------------------
// producer side
// ---------------------------------------------------------------------------
struct Producer {
  const StepParams& p;
  uint8_t* stages;
  size_t sbytes;
  uint64_t* full;
  uint64_t* empty;
  uint64_t pol;
  int S;
  long long i;  // ring index
  volatile int* abort_flag;
  int lane;

  // Run by all 32 lanes of the producer warp: lane 0 takes the stage and arms its
  // barrier, then one lane per contiguous run issues its bulk copy.
  __device__ bool issue(const LayerPtrs& Lp, const Plan& P, const Item& it) {
    const int s = (int)(i % S);
    int ok = 1;
    if (lane == 0 && i >= S) ok = ring_wait(&empty[s], (uint32_t)(((i / S) - 1) & 1), p.status, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) return false;
    uint8_t* st = stages + (size_t)s * sbytes;
    const int H = p.H, I = p.I, Is = p.Is;
    item_stamp(p, i, 0);
    if (it.type == IT_A) {
      const int nr = p.E / 4;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], 4u * 2u * H);
      __syncwarp();
      if (it.a < nr) {
        if (lane == 0) bulk_g2s(st, Lp.wr + (size_t)4 * it.a * H, 4u * 2u * H, &full[s], pol);
      } else {
        const int sh = it.a - nr;  // gate rows 2sh, 2sh+1 -> rows 0,1; up rows -> rows 2,3
        if (lane == 0) bulk_g2s(st, Lp.sw13 + (size_t)2 * sh * H, 2u * 2u * H, &full[s], pol);
        if (lane == 1) bulk_g2s(st + 4 * H, Lp.sw13 + (size_t)(Is + 2 * sh) * H, 2u * 2u * H, &full[s], pol);
      }
    } else if (it.type == IT_B) {
      const size_t e2I = (size_t)P.ids[it.a] * 2 * I;
      const uint32_t runb = 8u * (H / 2), scb = 8u * (H / 32);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], 2 * runb + 2 * scb);
      __syncwarp();
      if (lane == 0) bulk_g2s(st, Lp.w13c + (e2I + it.b) * (H / 2), runb, &full[s], pol);
      if (lane == 1) bulk_g2s(st + runb, Lp.w13c + (e2I + I + it.b) * (H / 2), runb, &full[s], pol);
      if (lane == 2) bulk_g2s(st + 2 * runb, Lp.w13s + (e2I + it.b) * (H / 32), scb, &full[s], pol);
      if (lane == 3) bulk_g2s(st + 2 * runb + scb, Lp.w13s + (e2I + I + it.b) * (H / 32), scb, &full[s], pol);
    } else if (it.type == IT_CR) {
      const size_t eH = (size_t)P.ids[it.a] * H;
      const uint32_t runb = 16u * (I / 2), scb = 16u * (I / 32);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], runb + scb);
      __syncwarp();
      if (lane == 0) bulk_g2s(st, Lp.w2c + (eH + it.b) * (I / 2), runb, &full[s], pol);
      if (lane == 1) bulk_g2s(st + runb, Lp.w2s + (eH + it.b) * (I / 32), scb, &full[s], pol);
    } else {
      if (lane == 0) mbar_arrive_expect_tx(&full[s], 4u * 2u * Is);
      __syncwarp();
      if (lane == 0) bulk_g2s(st, Lp.sw2 + (size_t)it.a * Is, 4u * 2u * Is, &full[s], pol);
    }
    ++i;
    return true;
  }

  // L2 prefetch of an item's bytes (same runs as issue()).
  __device__ void prefetch(const LayerPtrs& Lp, const Plan* P, const Item& it) {
    const int H = p.H, I = p.I, Is = p.Is;
    if (it.type == IT_A) {
      const int nr = p.E / 4;
      if (it.a < nr) {
        if (lane == 0) prefetch_l2(Lp.wr + (size_t)4 * it.a * H, 4u * 2u * H);
      } else {
        const int sh = it.a - nr;
        if (lane == 0) prefetch_l2(Lp.sw13 + (size_t)2 * sh * H, 2u * 2u * H);
        if (lane == 1) prefetch_l2(Lp.sw13 + (size_t)(Is + 2 * sh) * H, 2u * 2u * H);
      }
    } else if (it.type == IT_B) {
      const size_t e2I = (size_t)P->ids[it.a] * 2 * I;
      if (lane == 0) prefetch_l2(Lp.w13c + (e2I + it.b) * (H / 2), 8u * (H / 2));
      if (lane == 1) prefetch_l2(Lp.w13c + (e2I + I + it.b) * (H / 2), 8u * (H / 2));
      if (lane == 2) prefetch_l2(Lp.w13s + (e2I + it.b) * (H / 32), 8u * (H / 32));
      if (lane == 3) prefetch_l2(Lp.w13s + (e2I + I + it.b) * (H / 32), 8u * (H / 32));
    } else if (it.type == IT_CR) {
      const size_t eH = (size_t)P->ids[it.a] * H;
      if (lane == 0) prefetch_l2(Lp.w2c + (eH + it.b) * (I / 2), 16u * (I / 2));
      if (lane == 1) prefetch_l2(Lp.w2s + (eH + it.b) * (I / 32), 16u * (I / 32));
    } else {
      if (lane == 0) prefetch_l2(Lp.sw2 + (size_t)it.a * Is, 4u * 2u * Is);
    }
  }
};

// ---------------------------------------------------------------------------
// consumer-side pieces
// ---------------------------------------------------------------------------
// Consumer-only barrier (the 4 consumer warps; the producer never joins).
__device__ __forceinline__ void csync() { named_barrier(1, 32 * N_CONSUMERS); }

// The layer input in two forms: bf16 x_l (router / shared-expert operand) at
// xb16 and f16 x_l scaled by a per-token power of two (MXFP4 operand) at xf16.
// Layer 0 takes the input; later layers x = bf16(RMSNorm(h)).  One pass collects
// the sum of squares and max |h| per token (deterministic reduction order, the same
// in every block), the second writes both copies.  max_i bf16(|h_i| r) equals
// bf16(max_i |h_i| r) because rounding is monotonic, so the shift is exact.
__device__ void stage_layer_input(const StepParams& p, int l, uint8_t* xb16, uint8_t* xf16, uint32_t xss,
                                  float* s_part, float* s_amx, float* s_r, int* s_sh, float* s_inv) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = p.M, H = p.H, nt = 32 * N_CONSUMERS;
  for (int tok = 0; tok < M; ++tok) {
    float ss = 0.0f, am = 0.0f;
    if (l == 0) {
      for (int c = tid; c < H / 8; c += nt) {
        const uint4 v = *reinterpret_cast<const uint4*>(p.x_in + (size_t)tok * H + 8 * c);
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) am = fmaxf(am, fmaxf(fabsf(__low2float(b[j])), fabsf(__high2float(b[j]))));
      }
    } else {
      for (int c = tid; c < H / 4; c += nt) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p.h + (size_t)tok * H) + c);
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
        am = fmaxf(am, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    }
    if (lane == 0) {
      s_part[tok * N_CONSUMERS + warp] = ss;
      s_amx[tok * N_CONSUMERS + warp] = am;
    }
  }
  csync();
  if (tid < M) {
    float ss = 0.0f, am = 0.0f;
    for (int w = 0; w < N_CONSUMERS; ++w) {
      ss += s_part[tid * N_CONSUMERS + w];
      am = fmaxf(am, s_amx[tid * N_CONSUMERS + w]);
    }
    const float r = l == 0 ? 1.0f : 1.0f / sqrtf(ss / (float)H + p.eps);
    s_r[tid] = r;
    const float amx = l == 0 ? am : __bfloat162float(__float2bfloat16_rn(am * r));
    const int sh = f16_range_shift(amx);
    s_sh[tid] = sh;
    s_inv[tid] = exp2i(-sh);
  }
  csync();
  if (l == 0) {
    for (int i = tid; i < M * (H / 8); i += nt) {
      const int tok = i / (H / 8), c = i % (H / 8);
      uint4 v = *reinterpret_cast<const uint4*>(p.x_in + (size_t)tok * H + 8 * c);
      *reinterpret_cast<uint4*>(xb16 + tok * xss + 16 * c) = v;
      const float sc = exp2i(s_sh[tok]);
      uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
        const __half2 hh = __floats2half2_rn(__low2float(b) * sc, __high2float(b) * sc);
        w[j] = *reinterpret_cast<const uint32_t*>(&hh);
      }
      *reinterpret_cast<uint4*>(xf16 + tok * xss + 16 * c) = v;
    }
  } else {
    for (int i = tid; i < M * (H / 4); i += nt) {
      const int tok = i / (H / 4), c = i % (H / 4);
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p.h + (size_t)tok * H) + c);
      const float r = s_r[tok], sc = exp2i(s_sh[tok]);
      const __nv_bfloat162 a = __floats2bfloat162_rn(v.x * r, v.y * r);
      const __nv_bfloat162 b = __floats2bfloat162_rn(v.z * r, v.w * r);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&a);
      u.y = *reinterpret_cast<const uint32_t*>(&b);
      *reinterpret_cast<uint2*>(xb16 + tok * xss + 8 * c) = u;
      const __half2 ha = __floats2half2_rn(__low2float(a) * sc, __high2float(a) * sc);
      const __half2 hb = __floats2half2_rn(__low2float(b) * sc, __high2float(b) * sc);
      u.x = *reinterpret_cast<const uint32_t*>(&ha);
      u.y = *reinterpret_cast<const uint32_t*>(&hb);
      *reinterpret_cast<uint2*>(xf16 + tok * xss + 8 * c) = u;
    }
  }
  csync();
}

// Top-k of every token from the complete router logits (same rule as k_dense:
// largest logit, lowest index on ties), then the union plan.  The 4 consumer warps
// each take a quarter of the experts and keep their own top-k (a global top-k
// element is always in its quarter's top-k, ties included), then one warp per
// token merges the 4k candidates.
__device__ void step_topk(const StepParams& p, int l, Plan& P, int32_t* s_ids, float* s_wts, uint32_t* s_ck,
                          int32_t* s_ci) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E, k = p.k, M = p.M;
  const int per = (E + N_CONSUMERS - 1) / N_CONSUMERS;  // experts per warp (<= 256)
  const int e0 = warp * per;
  for (int tok = 0; tok < M; ++tok) {
    uint32_t key[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int off = lane + 32 * i, e = e0 + off;
      key[i] = (off < per && e < E) ? float_key(__ldcg(p.logits + tok * E + e)) : 0u;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        uint32_t bk = 0u;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (key[i] > bk) {
            bk = key[i];
            bi = e0 + lane + 32 * i;
          }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        const int mi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(bk == mk ? bi : 0x7fffffff));
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (e0 + lane + 32 * i == mi) key[i] = 0u;
        if (lane == 0) {
          s_ck[(tok * N_CONSUMERS + warp) * 8 + j] = mk;
          s_ci[(tok * N_CONSUMERS + warp) * 8 + j] = mk ? mi : 0x7fffffff;
        }
      }
    }
  }
  csync();
  for (int tok = warp; tok < M; tok += N_CONSUMERS) {
    const int nc = N_CONSUMERS * k;  // <= 32 candidates, one per lane
    uint32_t ck = 0u;
    int ci = 0x7fffffff;
    if (lane < nc) {
      ck = s_ck[(tok * N_CONSUMERS + lane / k) * 8 + lane % k];
      ci = s_ci[(tok * N_CONSUMERS + lane / k) * 8 + lane % k];
    }
    int sel_id = 0;
    uint32_t sel_key = 0u;
    for (int j = 0; j < k; ++j) {
      const uint32_t mk = __reduce_max_sync(0xffffffffu, ck);
      const int mi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(ck == mk ? ci : 0x7fffffff));
      if (ck == mk && ci == mi) {
        ck = 0u;
        ci = 0x7fffffff;
      }
      if (lane == j) {
        sel_id = mi;
        sel_key = mk;
      }
    }
    // lane j holds the j-th selection; softmax over the selected logits
    const float lj = key_float(sel_key);
    const float l0 = __shfl_sync(0xffffffffu, lj, 0);
    const float ex = lane < k ? expf(lj - l0) : 0.0f;
    float den = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane < k) {
      const float wj = ex / den;
      s_ids[tok * k + lane] = sel_id;
      s_wts[tok * k + lane] = wj;
      if (blockIdx.x == 0) {
        const size_t o = ((size_t)l * M + tok) * k + lane;
        if (p.ids_trace) p.ids_trace[o] = sel_id;
        if (p.w_trace) p.w_trace[o] = wj;
      }
    }
  }
  csync();
  if (warp == 0) build_plan(P, s_ids, s_wts, M, k, E);
  csync();
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// 4 weight rows (N operand, rows 0-3 of the MMA's 8 columns) against up to 16
// activation rows (M operand) over K; the B fragment of column n is read from
// shared-memory row rowmap[n] so that pairs of rows can be placed where an
// epilogue wants them.  Activation row m of the M operand is read by lane group g
// (m = g) and g + 8 from act0 / act1 (nullptr: zero).  c[] as the m16n8 C layout.
__device__ __forceinline__ void rows4_dot(const uint8_t* wrows, uint32_t wstride, int wrow_of_g, const uint8_t* act0,
                                          const uint8_t* act1, int K, float (&c)[4]) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  float c4[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u) c4[u][0] = c4[u][1] = c4[u][2] = c4[u][3] = 0.0f;
  const uint8_t* wr = wrow_of_g >= 0 ? wrows + (size_t)wrow_of_g * wstride : nullptr;
  const int nsp = K / 32;
  // four 32-column spans per step: all 12 shared-memory loads first, then 8 MMAs
  for (int j = 0; j < nsp; j += 4) {
    uint4 Bw[4], X0[4], X1[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int js = j + jj;
      const bool v = js < nsp;
      Bw[jj] = (v && wr) ? lds128(wr + 64 * js + 16 * t) : zero;
      X0[jj] = (v && act0) ? lds128(act0 + 64 * js + 16 * t) : zero;
      X1[jj] = (v && act1) ? lds128(act1 + 64 * js + 16 * t) : zero;
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      mma_bf16(c4[jj], X0[jj].x, X1[jj].x, X0[jj].y, X1[jj].y, Bw[jj].x, Bw[jj].y);
      mma_bf16(c4[jj], X0[jj].z, X1[jj].z, X0[jj].w, X1[jj].w, Bw[jj].z, Bw[jj].w);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) c[e] = (c4[0][e] + c4[1][e]) + (c4[2][e] + c4[3][e]);
}

__global__ void __launch_bounds__(STEP_THREADS, 1) k_step(const __grid_constant__ StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ float s_part[MAX_M * N_CONSUMERS];
  __shared__ float s_r[MAX_M];
  __shared__ float s_inv[MAX_M];
  __shared__ float s_pscale[N_CONSUMERS][MAX_M];
  __shared__ int32_t s_ids[MAX_SLOTS];
  __shared__ float s_wts[MAX_SLOTS];
  __shared__ float s_amx[MAX_M * N_CONSUMERS];
  __shared__ int s_sh[MAX_M];
  __shared__ uint32_t s_ck[MAX_M * N_CONSUMERS * 8];
  __shared__ int32_t s_ci[MAX_M * N_CONSUMERS * 8];
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = p.M, H = p.H, I = p.I, Is = p.Is, L = p.L, S = p.stages;
  const unsigned G = gridDim.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + MAX_STAGES;
  uint64_t* plan_bar = empty + MAX_STAGES;
  uint8_t* stages = smem + STEP_FIXED;
  const size_t sbytes = step_stage_bytes(H, I, Is);
  uint8_t* act = stages + (size_t)S * sbytes;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t sss = Is > 0 ? padded_stride(2u * Is) : 0u;
  const uint32_t ass = padded_stride(2u * I);
  uint8_t* xb16 = act;                                 // A/B phases: bf16 x rows [M][xss]
  uint8_t* xf16 = act + (size_t)M * xss;               //             f16 x rows  [M][xss]
  uint8_t* shi = act;                                  // C phase: shared a, bf16 hi  [M][sss]
  uint8_t* slo = act + (size_t)M * sss;                //                    bf16 lo  [M][sss]
  uint8_t* afw = act + 2 * (size_t)M * sss;            //          routed a per warp [4][M][ass]

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(plan_bar, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  // ---------------- producer ----------------
  if (warp == N_CONSUMERS) {
    Producer pr{p, stages, sbytes, full, empty, policy_evict_first(), S, 0, &s_abort, lane};
    bool ok = true;
    for (int l = 0; l < L && ok; ++l) {
      const LayerPtrs& Lp = p.layer[l];
      Work W;
      W.init_A(p);
      for (int r = 0; r < W.nA && ok; ++r) ok = pr.issue(Lp, P, W.at(p, r));
      if (!ok) break;
      stamp(p, l, 12);
      // routing-independent items: this layer's shared W2, the next layer's router/shared W13
      for (int r = 0; r < W.nS; ++r) pr.prefetch(Lp, nullptr, W.at(p, W.nA + r));
      if (l + 1 < L)
        for (int r = 0; r < W.nA; ++r) pr.prefetch(p.layer[l + 1], nullptr, W.at(p, r));
      int got = 1;
      if (lane == 0) got = ring_wait(plan_bar, (uint32_t)(l & 1), p.status, &s_abort);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      stamp(p, l, 13);
      W.init_routed(p, P.n_unique);
      const int nR = (int)(W.nB + W.nC);
      for (int r = 0; r < nR && r < STEP_PREFETCH_AHEAD; ++r) pr.prefetch(Lp, &P, W.at(p, W.nA + r));
      for (int r = 0; r < nR && ok; ++r) {
        if (r + STEP_PREFETCH_AHEAD < nR) pr.prefetch(Lp, &P, W.at(p, W.nA + r + STEP_PREFETCH_AHEAD));
        ok = pr.issue(Lp, P, W.at(p, W.nA + r));
      }
      stamp(p, l, 14);
      for (int r = 0; r < W.nS && ok; ++r) ok = pr.issue(Lp, P, W.at(p, W.nA + nR + r));
      stamp(p, l, 15);
    }
    // drain: the last use of every stage has landed before the block may exit
    if (lane == 0 && !s_abort)
      for (long long j = (pr.i > S ? pr.i - S : 0); j < pr.i; ++j)
        ring_wait(&full[j % S], (uint32_t)((j / S) & 1), p.status, &s_abort);
    return;
  }

  // ---------------- consumers ----------------
  unsigned* ctr = p.ctr;
  long long i = 0;  // ring index
  for (int l = 0; l < L; ++l) {
    unsigned* lc = ctr + (size_t)l * CTR_PER_LAYER;
    stamp(p, l, 0);
    if (l > 0) {
      if (tid == 0) wait_counter(ctr + (size_t)(l - 1) * CTR_PER_LAYER + CTR_H, G, p.status, &s_abort);
      csync();
    }
    stamp(p, l, 1);
    stage_layer_input(p, l, xb16, xf16, xss, s_part, s_amx, s_r, s_sh, s_inv);
    stamp(p, l, 2);
    if (blockIdx.x == 0) {
      for (int e = tid; e < M * H; e += 32 * N_CONSUMERS) {
        const int tok = e / H, c = e % H;
        const __nv_bfloat16 xv = *reinterpret_cast<const __nv_bfloat16*>(xb16 + tok * xss + 2 * c);
        float hv;
        if (l == 0) {
          hv = __bfloat162float(xv);
          p.h[e] = hv;
        } else {
          hv = __ldcg(p.h + e);
        }
        if (p.x_trace) p.x_trace[(size_t)l * M * H + e] = xv;
        if (p.h_trace) p.h_trace[(size_t)l * M * H + e] = hv;
      }
      if (l == 0) {
        csync();
        if (tid == 0) signal_counter(ctr + 3);  // h initialised
      }
    }

    // ---- A: router items (4 experts) and shared-W13 items (2 gate + 2 up rows) ----
    Work W;
    W.init_A(p);
    const int nr = p.E / 4;
    for (int r = 0; r < W.nA; ++r) {
      const long long ii = i + r;
      if ((int)(ii % N_CONSUMERS) != warp) continue;
      const int s = (int)(ii % S);
      const Item it = W.at(p, r);
      const bool router = it.a < nr;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      item_stamp(p, ii, 3);
      if (ring_wait(&full[s], (uint32_t)((ii / S) & 1), p.status, &s_abort)) {
        item_stamp(p, ii, 1);
        // shared items: columns (0,1,2,3) = (gate 2s, up 2s, gate 2s+1, up 2s+1) from
        // smem rows (0, 2, 1, 3), so a thread's two columns are a (gate, up) pair
        const int wrow = g < 4 ? (router ? g : ((g & 1) ? 2 : 0) + (g >> 1)) : -1;
        rows4_dot(stages + (size_t)s * sbytes, 2u * H, wrow, g < M ? xb16 + g * xss : nullptr, nullptr, H, c);
      }
      __syncwarp();
      item_stamp(p, ii, 2);
      if (lane == 0) mbar_arrive(&empty[s]);
      if (t < 2 && g < M) {
        if (router) {
          p.logits[g * p.E + 4 * it.a + 2 * t] = c[0];
          p.logits[g * p.E + 4 * it.a + 2 * t + 1] = c[1];
        } else {
          p.a_shared[g * Is + 2 * (it.a - nr) + t] = silu_f32(c[0]) * c[1];
        }
      }
      __syncwarp();
      if (lane == 0) signal_counter(lc + (router ? CTR_ROUTER : CTR_SHARED));
    }
    i += W.nA;
    stamp(p, l, 3);

    // ---- top-k and plan (every block, identical) ----
    if (tid == 0) wait_counter(lc + CTR_ROUTER, (unsigned)(p.E / 4), p.status, &s_abort);
    csync();
    stamp(p, l, 4);
    step_topk(p, l, P, s_ids, s_wts, s_ck, s_ci);
    if (tid == 0) mbar_arrive(plan_bar);
    stamp(p, l, 5);
    W.init_routed(p, P.n_unique);
    stamp(p, l, 6);

    // ---- B: routed W13 + SwiGLU ----
    for (int r = 0; r < W.nB; ++r) {
      const long long ii = i + r;
      if ((int)(ii % N_CONSUMERS) != warp) continue;
      const int s = (int)(ii % S);
      const Item it = W.at(p, W.nA + r);
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      item_stamp(p, ii, 3);
      if (ring_wait(&full[s], (uint32_t)((ii / S) & 1), p.status, &s_abort)) {
        item_stamp(p, ii, 1);
        const uint8_t* st = stages + (size_t)s * sbytes;
        const uint8_t* sc = st + 8 * H;  // 16 scale rows of H/32 after the 16 code rows of H/2
        mxfp4_tile_dot(st + g * (H / 2), st + (8 + g) * (H / 2), sc + g * (H / 32), sc + (8 + g) * (H / 32), H / 32,
                       xf16, xss, M, c);
      }
      __syncwarp();
      item_stamp(p, ii, 2);
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = 2 * t + e;  // rows g (gate) and g+8 (up) of intermediate index it.b + g
        if (tok < M)
          p.a_routed[((size_t)it.a * M + tok) * I + it.b + g] = silu_f32(c[e] * s_inv[tok]) * (c[2 + e] * s_inv[tok]);
      }
      __syncwarp();
      if (lane == 0) signal_counter(lc + CTR_EXP + it.a);
    }
    i += W.nB;
    stamp(p, l, 7);
    csync();  // the activation region is free for the C phase
    stamp(p, l, 8);

    // ---- C: routed W2 (weighted) + shared W2, accumulated into h ----
    if (W.nS > 0) {
      if (tid == 0) wait_counter(lc + CTR_SHARED, (unsigned)(Is / 2), p.status, &s_abort);
      csync();
      for (int e = tid; e < M * (Is / 4); e += 32 * N_CONSUMERS) {
        const int tok = e / (Is / 4), c4 = e % (Is / 4);
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p.a_shared + (size_t)tok * Is) + c4);
        const float a4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat16 hi = __float2bfloat16_rn(a4[j]);
          const __nv_bfloat16 lo = __float2bfloat16_rn(a4[j] - __bfloat162float(hi));
          *reinterpret_cast<__nv_bfloat16*>(shi + tok * sss + 2 * (4 * c4 + j)) = hi;
          *reinterpret_cast<__nv_bfloat16*>(slo + tok * sss + 2 * (4 * c4 + j)) = lo;
        }
      }
      csync();
    }
    if (l == 0) {
      if (tid == 0) wait_counter(ctr + 3, 1u, p.status, &s_abort);  // h initialised by block 0
      csync();
    }
    stamp(p, l, 9);
    int cached_slot = -1;
    uint8_t* my_af = afw + (size_t)warp * M * ass;
    const int nC = (int)W.nC;
    for (int r = 0; r < nC + W.nS; ++r) {
      const long long ii = i + r;
      if ((int)(ii % N_CONSUMERS) != warp) continue;
      const int s = (int)(ii % S);
      const Item it = W.at(p, W.nA + (int)W.nB + r);
      const uint8_t* st = stages + (size_t)s * sbytes;
      if (it.type == IT_CR) {
        const int u = it.a;
        if (u != cached_slot) {
          if (lane == 0) wait_counter(lc + CTR_EXP + u, (unsigned)(I / 8), p.status, &s_abort);
          __syncwarp();
          for (int tok = 0; tok < M; ++tok) {
            const bool live = P.w[u][tok] != 0.0f;
            const float4* src = reinterpret_cast<const float4*>(p.a_routed + ((size_t)u * M + tok) * I);
            float4 v[8];  // I <= 1024: at most 8 float4 per lane
            float amax = 0.0f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int c4 = lane + 32 * jj;
              v[jj] = (live && c4 < I / 4) ? __ldcg(src + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
              amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[jj].x), fabsf(v[jj].y)), fmaxf(fabsf(v[jj].z), fabsf(v[jj].w))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const int sh = f16_range_shift(amax);
            const float scl = exp2i(sh);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int c4 = lane + 32 * jj;
              if (c4 < I / 4) {
                const __half2 h0 = __floats2half2_rn(v[jj].x * scl, v[jj].y * scl);
                const __half2 h1 = __floats2half2_rn(v[jj].z * scl, v[jj].w * scl);
                uint2 u2;
                u2.x = *reinterpret_cast<const uint32_t*>(&h0);
                u2.y = *reinterpret_cast<const uint32_t*>(&h1);
                *reinterpret_cast<uint2*>(my_af + tok * ass + 8 * c4) = u2;
              }
            }
            if (lane == 0) s_pscale[warp][tok] = live ? exp2i(-sh) : 0.0f;
          }
          __syncwarp();
          cached_slot = u;
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        item_stamp(p, ii, 3);
      if (ring_wait(&full[s], (uint32_t)((ii / S) & 1), p.status, &s_abort)) {
          item_stamp(p, ii, 1);
          const uint8_t* sc = st + 8 * I;  // 16 scale rows of I/32 after the 16 code rows of I/2
          mxfp4_tile_dot(st + g * (I / 2), st + (8 + g) * (I / 2), sc + g * (I / 32), sc + (8 + g) * (I / 32), I / 32,
                         my_af, ass, M, c);
        }
        __syncwarp();
        item_stamp(p, ii, 2);
        if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = 2 * t + e;
          if (tok < M) {
            const float wt = P.w[u][tok];
            if (wt != 0.0f) {
              const float f = wt * s_pscale[warp][tok];
              atomicAdd(p.h + (size_t)tok * H + it.b + g, c[e] * f);
              atomicAdd(p.h + (size_t)tok * H + it.b + g + 8, c[2 + e] * f);
            }
          }
        }
      } else {
        // shared W2: 4 output rows (N) against the activation rows m = 2*token + {hi, lo} (M)
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        item_stamp(p, ii, 3);
      if (ring_wait(&full[s], (uint32_t)((ii / S) & 1), p.status, &s_abort)) {
          item_stamp(p, ii, 1);
          const uint8_t* src = (g & 1) ? slo : shi;
          const int t0 = g >> 1, t1 = 4 + (g >> 1);
          rows4_dot(st, 2u * Is, g < 4 ? g : -1, t0 < M ? src + t0 * sss : nullptr,
                    t1 < M ? src + t1 * sss : nullptr, Is, c);
        }
        __syncwarp();
        item_stamp(p, ii, 2);
        if (lane == 0) mbar_arrive(&empty[s]);
        // hi + lo: rows m = 2tok (lane group g even) and 2tok + 1 (g odd)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] += __shfl_xor_sync(0xffffffffu, c[e], 4);
        if ((g & 1) == 0 && t < 2) {
          const int t0 = g >> 1, t1 = 4 + (g >> 1);
          if (t0 < M) {
            atomicAdd(p.h + (size_t)t0 * H + it.a + 2 * t, c[0]);
            atomicAdd(p.h + (size_t)t0 * H + it.a + 2 * t + 1, c[1]);
          }
          if (t1 < M) {
            atomicAdd(p.h + (size_t)t1 * H + it.a + 2 * t, c[2]);
            atomicAdd(p.h + (size_t)t1 * H + it.a + 2 * t + 1, c[3]);
          }
        }
      }
    }
    i += nC + W.nS;
    stamp(p, l, 10);
    csync();
    if (tid == 0) signal_counter(lc + CTR_H);
    stamp(p, l, 11);
  }

  // ---- LM-head input: bf16(RMSNorm(h_L)) by block 0 ----
  if (blockIdx.x != 0) return;
  if (tid == 0) wait_counter(ctr + (size_t)(L - 1) * CTR_PER_LAYER + CTR_H, G, p.status, &s_abort);
  csync();
  for (int tok = 0; tok < M; ++tok) {
    float ss = 0.0f;
    for (int c = tid; c < H / 4; c += 32 * N_CONSUMERS) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p.h + (size_t)tok * H) + c);
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_part[tok * N_CONSUMERS + warp] = ss;
  }
  csync();
  if (tid < M) {
    float ss = 0.0f;
    for (int w = 0; w < N_CONSUMERS; ++w) ss += s_part[tid * N_CONSUMERS + w];
    s_r[tid] = 1.0f / sqrtf(ss / (float)H + p.eps);
  }
  csync();
  for (int e = tid; e < M * H; e += 32 * N_CONSUMERS) {
    const int tok = e / H;
    const float hv = __ldcg(p.h + e);
    const __nv_bfloat16 v = __float2bfloat16_rn(hv * s_r[tok]);
    p.x_final[e] = v;
    if (p.x_trace) p.x_trace[(size_t)L * M * H + e] = v;
    if (p.h_trace) p.h_trace[(size_t)L * M * H + e] = hv;
  }
}

}  // namespace moe
