// step_kernel.cuh -- the whole decode step (all MoE layers) as one persistent kernel.
//
// One block per SM for the whole step (cooperative launch: all blocks co-resident).
// The last warp of each block is the producer: it walks this block's sequence of weight
// tiles for every layer and moves them HBM -> shared memory with bulk copies (TMA
// engine) into a byte-addressed ring, each tile taking exactly its own bytes, so the
// bytes in flight per SM stay high whatever the tile mix.  The tiles whose identity
// does not depend on the routing (router rows, shared-expert rows) come first in
// every layer, so the producer runs ahead across the layer boundary and the
// routing-dependent tiles are the only ones that wait for the top-k.  Warps 0-7
// consume the ring in order (item i -> warp i % 8) and synchronise only where the
// data forces it:
//   router tiles complete  -> every block takes the top-k itself (same code, same bits)
//   shared W13 complete    -> the shared W2 tiles may start
// (router logits and shared activations carry the layer number in the same 64-bit
// word, so readers poll the data itself: no writer fence, no separate counter)
//   expert u's W13 complete -> its W2 tiles may start (per-expert counter)
//   residual h complete    -> the next layer's RMSNorm may start (grid-wide counter)
// The residual is double-buffered by layer parity: layer l adds into h[l & 1], which
// every block first initialises (its slice) from h[(l - 1) & 1] while it reads that
// buffer for its RMSNorm, so no block's accumulation can reach a buffer another
// block is still normalising.
// Every wait is a bounded spin (abort flag + status word after WAIT_LIMIT_NS), so a
// fault in one block ends the step with MOE_ERR_TIMEOUT instead of a hang.
//
// Per layer, in ring order, block c processes (every item one or a few contiguous
// bulk copies):
//   A:  router items (4 experts' rows) and shared-W13 items (2 gate + 2 up rows),
//       fixed assignment j = c, c+G, ...; weight rows are the MMA's N operand and
//       the tokens its M operand, so one warp covers the full K of its 4 rows.
//   CS: shared-W2 items (4 output rows), fixed assignment.
//   B:  routed W13 items (distinct expert, 8 gate + 8 up rows), a contiguous range.
//   CR: routed W2 items (distinct expert, 16 output rows), a contiguous range.
// Sources: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
// 三种方法), 事件概述或研究问题 (batch-1 decode bound by weight reads; 8 of 512 experts
// + 1 shared) and 方法/产品要点 items 1 and 3.
#pragma once

#include "decode_kernels.cuh"

namespace moe {

constexpr int STEP_MAX_LAYERS = 64;
constexpr int STEP_CONSUMERS = 8;  // consumer warps: two per SM sub-partition, to hide latency
constexpr int STEP_THREADS = 32 * (STEP_CONSUMERS + 1);  // consumer warps 0-7, producer warp 8
constexpr int CR_CACHE = 4;         // routed experts whose W2 activation a block keeps staged
constexpr int STEP_SLOTS = 32;  // ring items in flight at most (one full/empty mbarrier pair each)
constexpr int CTR_H = 2, CTR_HINIT = 3, CTR_EXP = 4;  // slots 0-1 unused
constexpr int CTR_PER_LAYER = CTR_EXP + MAX_SLOTS;
constexpr size_t STEP_FIXED = 1024;  // full[32], empty[32], plan and h-init barriers
constexpr int STAGE_REG_F4 = 4;  // residual float4s a consumer thread keeps in registers (M = 1 at H = 2560)
constexpr int STAGE_BATCH = 5;   // larger inputs: residual loads a thread keeps in flight

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
  uint32_t ring_bytes;
  uint32_t act_bytes;
  const __nv_bfloat16* x_in;  // [M][H]
  float* h;                   // [2][M][H] residual stream, buffer l & 1 is layer l's output
  __nv_bfloat16* x_final;     // [M][H] LM-head input
  unsigned long long* logits;    // [M][E] tagged: (l + 1) << 32 | fp32 bits, zero on entry
  unsigned long long* a_shared;  // [M][Is] tagged like logits
  float* a_routed;            // [MAX_SLOTS][M][I]
  unsigned* ctr;              // [L][CTR_PER_LAYER], zero on entry
  int* status;
  __nv_bfloat16* x_trace;
  float* h_trace;
  int32_t* ids_trace;
  float* w_trace;
  unsigned long long* timeline;  // optional [2][L][16] %globaltimer stamps (blocks 0 and G-1)
  int hold_layer;                // testing the timeout path: this layer's residual is never published (-1: none)
  LayerPtrs layer[STEP_MAX_LAYERS];
};

// Profiling stamp: block 0 and the last block record %globaltimer at phase
// boundaries (slots 0-11 by consumer thread 0, 12-15 by producer lane 0).
__device__ __noinline__ void stamp_write(const StepParams& p, int l, int slot);
// DBG: the instantiation taken when a timeline or a trace buffer is passed; the other
// one carries none of the profiling or trace code.
template <bool DBG>
__device__ __forceinline__ void stamp(const StepParams& p, int l, int slot) {
  if constexpr (DBG) {
    if (p.timeline) stamp_write(p, l, slot);
  }
}
__device__ __noinline__ void stamp_write(const StepParams& p, int l, int slot) {
  const bool first = blockIdx.x == 0, last = blockIdx.x == gridDim.x - 1;
  if (!first && !last) return;
  const int tid = threadIdx.x;
  if (tid != 0 && tid != 32 * STEP_CONSUMERS) return;
  p.timeline[((size_t)(last ? 1 : 0) * p.L + l) * 16 + slot] = globaltimer_ns();
}
// Profiling: block 0's first STEP_ITEM_LOG ring items, 8 stamps each after the
// [2][L][16] phase stamps: 0 copies issued, 1 data seen by the consumer, 2 consumer
// done, 3 consumer started waiting, 4 producer entered issue().
constexpr int STEP_ITEM_LOG = 2048;
__device__ __noinline__ void item_stamp_write(const StepParams& p, long long i, int which) {
  if (blockIdx.x != 0 || i >= STEP_ITEM_LOG || (threadIdx.x & 31) != 0) return;
  p.timeline[(size_t)2 * p.L * 16 + (size_t)i * 8 + which] = globaltimer_ns();
}
template <bool DBG>
__device__ __forceinline__ void item_stamp(const StepParams& p, long long i, int which) {
  if constexpr (DBG) {
    if (p.timeline) item_stamp_write(p, i, which);
  }
}
// Profiling: every block's own phase ends, [G][L][16] after the item log (written by
// the calling thread): 0 residual seen, 1 layer input staged, 2 router item published,
// 3 router/shared-W13 items done, 4 routing plan built, 5 shared W2 done, 6 routed W13
// done, 7 routed W2 done; 8-12 finer marks inside the top-k; 13-15 data arrivals.
__device__ __noinline__ void blk_stamp_write(const StepParams& p, int l, int slot) {
  p.timeline[(size_t)2 * p.L * 16 + (size_t)STEP_ITEM_LOG * 8 + ((size_t)blockIdx.x * p.L + l) * 16 + slot] =
      globaltimer_ns();
}
template <bool DBG>
__device__ __forceinline__ void blk_stamp(const StepParams& p, int l, int slot) {
  if constexpr (DBG) {
    if (p.timeline) blk_stamp_write(p, l, slot);
  }
}

// ---------------------------------------------------------------------------
// geometry shared by host and device
// ---------------------------------------------------------------------------
enum : int { IT_A = 0, IT_B = 1, IT_CR = 2, IT_CS = 3 };

// Ring bytes of one item: 4 bf16 rows of H (router / shared W13), 16 MXFP4 rows of
// H + their scales (routed W13), 16 MXFP4 rows of I + scales (routed W2), 4 bf16
// rows of Is (shared W2); 128-byte granules.
__host__ __device__ inline uint32_t step_item_bytes(int type, int H, int I, int Is) {
  size_t b;
  if (type == IT_A)
    b = 8 * (size_t)H;
  else if (type == IT_B)
    b = 8 * (size_t)H + (size_t)H / 2;
  else if (type == IT_CR)
    b = 8 * (size_t)I + (size_t)I / 2;
  else
    b = 8 * (size_t)Is;
  return (uint32_t)((b + 127) / 128 * 128);
}
__host__ __device__ inline uint32_t step_max_item_bytes(int H, int I, int Is) {
  uint32_t b = step_item_bytes(IT_A, H, I, Is);
  for (int t = IT_B; t <= IT_CS; ++t) {
    const uint32_t x = step_item_bytes(t, H, I, Is);
    if (x > b) b = x;
  }
  return b;
}
// Activation region: A/B phases hold the bf16 layer input xb16 [M][xss] at 0 and the
// f16 copy xf16 [M][xss] after it; the shared-W2 phase adds the hi/lo bf16 halves of
// the shared activation [2][M][sss], over xb16 when they fit there (xb16 is dead once
// the router and shared-W13 items are done); the routed-W2 phase holds the f16
// activations of the (at most CR_CACHE) experts of the block's range [CR_CACHE][M][ass] at 0.
__host__ __device__ inline bool step_shared_over_xb16(int H, int Is) {
  return 2u * (Is > 0 ? padded_stride(2u * Is) : 0u) <= padded_stride(2u * H);
}
__host__ __device__ inline uint32_t step_act_bytes(int M, int H, int I, int Is) {
  const uint32_t xss = padded_stride(2u * H), sss = Is > 0 ? padded_stride(2u * Is) : 0u;
  uint32_t a = 2u * M * xss + (step_shared_over_xb16(H, Is) ? 0u : 2u * M * sss);
  const uint32_t c = (uint32_t)CR_CACHE * M * padded_stride(2u * I);
  if (c > a) a = c;
  return (a + 127) / 128 * 128;
}
// Deterministic placement in the byte ring on monotonic virtual byte positions (the
// producer and every consumer warp walk the same item sequence and compute the same
// offsets): an item that would cross the end of the ring starts at the next multiple
// of R.  The cursor keeps the ring offset beside the virtual position, so placing an
// item needs no division.  Returns the ring offset; *vstart receives the virtual start.
struct RingCursor {
  unsigned long long v;  // virtual byte position
  uint32_t off;          // v % R
};
__device__ __forceinline__ uint32_t ring_take(RingCursor& c, uint32_t n, uint32_t R,
                                              unsigned long long* vstart = nullptr) {
  if (c.off + n > R) {
    c.v += R - c.off;
    c.off = 0u;
  }
  const uint32_t o = c.off;
  if (vstart) *vstart = c.v;
  c.v += n;
  c.off += n;
  if (c.off == R) c.off = 0u;
  return o;
}

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
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_tagged(unsigned long long* p, float v, uint32_t tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
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
  const unsigned long long t0 = globaltimer_ns(), lim = wait_limit(status);
  while (true) {
    __nanosleep(32);
    if (ld_acquire_u32(c) >= target) return true;
    if (*abort_flag) return false;
    if (ld_volatile_i32(status) != 0 || globaltimer_ns() - t0 > lim) {
      atomicCAS(status, 0, DEV_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}
// mbarrier wait that also honours the block's abort flag: the first try inline, the
// bounded loop out of line.
__device__ __forceinline__ bool ring_wait_slow(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag);
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  return ring_wait_slow(bar, parity, status, abort_flag);
}
__device__ __forceinline__ bool ring_wait_slow(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  const unsigned long long t0 = globaltimer_ns(), lim = wait_limit(status);
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > lim) {
      atomicCAS(status, 0, DEV_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}
// The same wait for a whole warp: lane 0 waits, the others take its answer.
__device__ __forceinline__ bool warp_ring_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = ring_wait(bar, parity, status, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}
// Gives up the whole step: records the timeout once and raises the block's abort flag.
__device__ __noinline__ void step_give_up(int* status, volatile int* abort_flag) {
  atomicCAS(status, 0, DEV_ERR_TIMEOUT);
  *abort_flag = 1;
}
// Tagged reads: n words (n <= 8, pointers in w[]) are loaded together and retried
// until every tag equals `tag` (bounded; false after the limit or an abort).
__device__ __forceinline__ bool await_tagged(const unsigned long long* const* w, int n, uint32_t tag, float* v,
                                             int* status, volatile int* abort_flag) {
  unsigned long long x[8];
  unsigned long long t0 = 0;
  while (true) {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = j < n ? ld_relaxed_u64(w[j]) : ((unsigned long long)tag << 32);
    bool ok = true;
#pragma unroll
    for (int j = 0; j < 8; ++j) ok = ok && (uint32_t)(x[j] >> 32) == tag;
    if (ok) break;
    if (*abort_flag) return false;
    if (t0 == 0) t0 = globaltimer_ns();
    if (globaltimer_ns() - t0 > wait_limit(status)) {
      step_give_up(status, abort_flag);
      return false;
    }
    __nanosleep(20);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < n) v[j] = __uint_as_float((uint32_t)x[j]);
  return true;
}
// Time-bounded wait for a copy to land, used only when the block is about to exit
// (the abort flag is ignored: copies in flight must finish before shared memory goes;
// the full default limit, whatever the test limit, since a copy in flight always lands).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 500u))
    if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) return;
}

// ---------------------------------------------------------------------------
// the per-layer work list of one block: A, CS, then (after the routing) B, CR
// ---------------------------------------------------------------------------
struct Item {
  int type;
  int a, b;  // A: item j;  CS: first row;  B: slot, r0;  CR: slot, h0
};

struct Work {
  int nA;             // A items of this block
  int nS;             // shared-W2 items of this block
  int b0, nB;         // routed W13 range
  int c0, nC;         // routed W2 range
  __device__ void init_fixed(const StepParams& p) {
    const int c = blockIdx.x, G = gridDim.x;
    const int TA = p.E / 4 + p.Is / 2;
    nA = c < TA ? (TA - 1 - c) / G + 1 : 0;
    const int TS = p.Is > 0 ? p.H / 4 : 0;
    nS = c < TS ? (TS - 1 - c) / G + 1 : 0;
    nB = nC = 0;
    b0 = c0 = 0;
  }
  __device__ void init_routed(const StepParams& p, int n_unique) {
    // n_unique <= MAX_SLOTS: tiles per expert * n_unique * blocks stays far below 2^31
    const int c = blockIdx.x, G = gridDim.x;
    const int TB = n_unique * (p.I / 8);
    b0 = TB * c / G;
    nB = TB * (c + 1) / G - b0;
    const int TC = n_unique * (p.H / 16);
    c0 = TC * c / G;
    nC = TC * (c + 1) / G - c0;
  }
  __device__ Item at(const StepParams& p, long long r) const {
    Item it;
    if (r < nA) {
      it.type = IT_A;
      it.a = blockIdx.x + (int)r * gridDim.x;
      it.b = 0;
      return it;
    }
    r -= nA;
    if (r < nS) {
      it.type = IT_CS;
      it.a = 4 * (blockIdx.x + (int)r * gridDim.x);
      it.b = 0;
      return it;
    }
    r -= nS;
    if (r < nB) {
      const long long x = b0 + r;
      it.type = IT_B;
      it.a = (int)(x / (p.I / 8));
      it.b = 8 * (int)(x % (p.I / 8));
      return it;
    }
    r -= nB;
    const long long x = c0 + r;
    it.type = IT_CR;
    it.a = (int)(x / (p.H / 16));
    it.b = 16 * (int)(x % (p.H / 16));
    return it;
  }
};

// Consecutive routed tiles of one expert travel as one ring item (their rows are
// contiguous in HBM: one copy per run instead of one per tile).  Walks tiles
// x .. end-1 of the block's range (T tiles per expert), at most cap per group.
struct GroupWalk {
  int x, end;
  int T, cap;
  __device__ bool next(int& u, int& r0, int& nt) {
    if (x >= end) return false;
    u = x / T;
    r0 = x - u * T;
    const int lim = min(end, (u + 1) * T);
    nt = min(cap, lim - x);
    x += nt;
    return true;
  }
};
// Tiles per group: a third of the ring at most, so two groups and the smaller items
// around them are in flight together.
__host__ __device__ inline int step_group_cap(uint32_t R, uint32_t tile_bytes, int maxcap) {
  const int c = (int)(R / (3u * tile_bytes));
  return c < 1 ? 1 : (c > maxcap ? maxcap : c);
}

// ---------------------------------------------------------------------------
// producer side
// ---------------------------------------------------------------------------
template <bool DBG>
struct Producer {
  const StepParams& p;
  uint8_t* ring;
  uint32_t R;
  uint64_t* full;
  uint64_t* empty;
  unsigned long long* vst;  // [STEP_SLOTS] virtual start of the items in flight (lane 0)
  uint64_t pol;
  long long i;               // next ring item
  long long oldest;          // oldest item whose release lane 0 has not seen yet
  RingCursor vpos;           // virtual placement cursor
  volatile int* abort_flag;
  int lane;

  // Run by all 32 lanes of the producer warp: lane 0 waits, in FIFO order, for the
  // release of the oldest items until the new item and every item still in flight
  // fit in one ring-length window of virtual bytes (then no two overlap in the ring)
  // and the new item's barrier slot is free, and arms the barrier; then one lane per
  // contiguous run issues its bulk copy.
  __device__ bool acquire(uint32_t n, uint32_t& s0, int& slot) {
    item_stamp<DBG>(p, i, 4);
    unsigned long long vs;
    s0 = ring_take(vpos, n, R, &vs);
    slot = (int)(i % STEP_SLOTS);
    int ok = 1;
    if (lane == 0) {
      while (oldest < i) {
        const int os = (int)(oldest % STEP_SLOTS);
        const bool need = (i - oldest >= STEP_SLOTS) || (vs + n - vst[os] > R);
        if (!need) break;
        if (!ring_wait(&empty[os], (uint32_t)((oldest / STEP_SLOTS) & 1), p.status, abort_flag)) {
          ok = 0;
          break;
        }
        ++oldest;
      }
      vst[slot] = vs;
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) item_stamp<DBG>(p, i, 0);
    return ok != 0;
  }

  // routed W13 group: tiles r0 .. r0+nt-1 (8 gate + 8 up rows each) of expert slot u;
  // layout [gate codes][up codes][gate scales][up scales], nt*8 rows each
  __device__ bool issue_b(const LayerPtrs& Lp, const Plan& P, int u, int r0, int nt) {
    const int H = p.H, I = p.I;
    const uint32_t codes = (uint32_t)nt * 8u * (H / 2), scales = (uint32_t)nt * 8u * (H / 32);
    uint32_t s0;
    int slot;
    if (!acquire(2 * codes + 2 * scales, s0, slot)) return false;
    uint8_t* st = ring + s0;
    uint64_t* fb = &full[slot];
    const size_t row = (size_t)P.ids[u] * 2 * I + 8 * (size_t)r0;
    if (lane == 0) mbar_arrive_expect_tx(fb, 2 * codes + 2 * scales);
    __syncwarp();
    if (lane == 0) bulk_g2s(st, Lp.w13c + row * (H / 2), codes, fb, pol);
    if (lane == 1) bulk_g2s(st + codes, Lp.w13c + (row + I) * (H / 2), codes, fb, pol);
    if (lane == 2) bulk_g2s(st + 2 * codes, Lp.w13s + row * (H / 32), scales, fb, pol);
    if (lane == 3) bulk_g2s(st + 2 * codes + scales, Lp.w13s + (row + I) * (H / 32), scales, fb, pol);
    item_stamp<DBG>(p, i, 5);
    ++i;
    return true;
  }
  // routed W2 group: tiles c0 .. c0+nt-1 (16 output rows each) of expert slot u;
  // layout [codes][scales], nt*16 rows each
  __device__ bool issue_c(const LayerPtrs& Lp, const Plan& P, int u, int c0, int nt) {
    const int H = p.H, I = p.I;
    const uint32_t codes = (uint32_t)nt * 16u * (I / 2), scales = (uint32_t)nt * 16u * (I / 32);
    uint32_t s0;
    int slot;
    if (!acquire(codes + scales, s0, slot)) return false;
    uint8_t* st = ring + s0;
    uint64_t* fb = &full[slot];
    const size_t row = (size_t)P.ids[u] * H + 16 * (size_t)c0;
    if (lane == 0) mbar_arrive_expect_tx(fb, codes + scales);
    __syncwarp();
    if (lane == 0) bulk_g2s(st, Lp.w2c + row * (I / 2), codes, fb, pol);
    if (lane == 1) bulk_g2s(st + codes, Lp.w2s + row * (I / 32), scales, fb, pol);
    item_stamp<DBG>(p, i, 5);
    ++i;
    return true;
  }

  // router / shared items (one tile each) through the ring
  __device__ bool issue(const LayerPtrs& Lp, const Plan& P, const Item& it) {
    uint32_t s0;
    int slot;
    if (!acquire(step_item_bytes(it.type, p.H, p.I, p.Is), s0, slot)) return false;
    copy_item(Lp, it, ring + s0, &full[slot]);
    item_stamp<DBG>(p, i, 5);
    ++i;
    return true;
  }
  // the copies of one router / shared item into st, completing on fb
  __device__ void copy_item(const LayerPtrs& Lp, const Item& it, uint8_t* st, uint64_t* fb) {
    const int H = p.H, Is = p.Is;
    if (it.type == IT_A) {
      const int nr = p.E / 4;
      if (lane == 0) mbar_arrive_expect_tx(fb, 4u * 2u * H);
      __syncwarp();
      if (it.a < nr) {
        if (lane == 0) bulk_g2s(st, Lp.wr + (size_t)4 * it.a * H, 4u * 2u * H, fb, pol);
      } else {
        const int sh = it.a - nr;  // gate rows 2sh, 2sh+1 -> rows 0,1; up rows -> rows 2,3
        if (lane == 0) bulk_g2s(st, Lp.sw13 + (size_t)2 * sh * H, 2u * 2u * H, fb, pol);
        if (lane == 1) bulk_g2s(st + 4 * H, Lp.sw13 + (size_t)(Is + 2 * sh) * H, 2u * 2u * H, fb, pol);
      }
    } else {
      if (lane == 0) mbar_arrive_expect_tx(fb, 4u * 2u * Is);
      __syncwarp();
      if (lane == 0) bulk_g2s(st, Lp.sw2 + (size_t)it.a * Is, 4u * 2u * Is, fb, pol);
    }
  }
};

// ---------------------------------------------------------------------------
// consumer-side pieces
// ---------------------------------------------------------------------------
// Consumer-only barrier (the 4 consumer warps; the producer never joins).
__device__ __forceinline__ void csync() { named_barrier(1, 32 * STEP_CONSUMERS); }
// Consumer barrier that also returns, to every consumer thread, whether any of them
// passed a true predicate (one decision for the whole block: leaving a loop on it
// never splits the consumers across a later barrier).
__device__ __forceinline__ bool csync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(32 * STEP_CONSUMERS)
      : "memory");
  return r != 0;
}

// The layer input in two forms: bf16 x_l (router / shared-expert operand) at
// xb16 and f16 x_l scaled by a per-token power of two (MXFP4 operand) at xf16.
// Layer 0 takes the input; later layers x = bf16(RMSNorm(h)), h the previous
// layer's residual buffer.  The same pass copies this block's slice of that
// residual (or of fp32(input) at layer 0) into this layer's accumulation buffer.
// The residual is read once when a thread's share fits in registers (STAGE_REG_F4
// float4s), else twice.  Every block reduces in the same order (per thread over its
// float4s, then the warp butterfly, then warps 0..3), so all blocks get the same
// bits -- they take the top-k independently and must agree.  max_i bf16(|h_i| r)
// equals bf16(max_i |h_i| r) because rounding is monotonic, so the shift is exact.
__device__ __forceinline__ float4 load_residual4(const StepParams& p, int l, const float* hin, int q) {
  if (l == 0) {
    const uint2 u = *reinterpret_cast<const uint2*>(p.x_in + 4 * (size_t)q);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
  }
  return __ldcg(reinterpret_cast<const float4*>(hin) + q);
}
// Byte offset of element e of a one-token f16 activation row held chunk-major:
// chunk w (elements 8w..8w+7) of scale block b at (w * nb + b) * 16.  Lanes that walk
// consecutive blocks then read consecutive 16-byte chunks (no bank conflicts).
__device__ __forceinline__ uint32_t chunk_major_off(int e, int nb) {
  return (uint32_t)((((e >> 3) & 3) * nb + (e >> 5)) * 16 + (e & 7) * 2);
}

__device__ __forceinline__ void write_layer_input4(uint8_t* xb16, uint8_t* xf16, uint32_t off, uint32_t off16, float4 v,
                                                   float r, int sh) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x * r, v.y * r);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v.z * r, v.w * r);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(xb16 + off) = u;
  const __half2 ha = __floats2half2_rn(mul_pow2(__low2float(a), sh), mul_pow2(__high2float(a), sh));
  const __half2 hb = __floats2half2_rn(mul_pow2(__low2float(b), sh), mul_pow2(__high2float(b), sh));
  u.x = *reinterpret_cast<const uint32_t*>(&ha);
  u.y = *reinterpret_cast<const uint32_t*>(&hb);
  *reinterpret_cast<uint2*>(xf16 + off16) = u;
}
__device__ __forceinline__ void accumulate4(float4 v, float& ss, float& am) {
  ss = fmaf(v.x, v.x, ss);
  ss = fmaf(v.y, v.y, ss);
  ss = fmaf(v.z, v.z, ss);
  ss = fmaf(v.w, v.w, ss);
  am = fmaxf(am, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
}

// The window's layer input (one token: stage1): x = bf16(RMSNorm(h)) (layer 0: the
// given x) as bf16 rows at xb16 and as f16 rows scaled by 2^sh at xf16 (stride xss,
// row-major for the tensor-core tiles); [q0, q1) is this block's slice of the
// residual's float4s, copied into hout in the same pass.
__device__ void stage_window_input(const StepParams& p, int l, const float* hin, float* hout, uint8_t* xb16,
                                   uint8_t* xf16, uint32_t xss, float* s_part, float* s_amx, float* s_r, int* s_sh,
                                   int q0, int q1) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = p.M, H = p.H, nt = 32 * STEP_CONSUMERS;
  const int per = H / 4, Q = M * per;  // float4s per token / in total

  float4* hout4 = reinterpret_cast<float4*>(hout);
  const bool inreg = Q <= STAGE_REG_F4 * nt;
  float4 v[STAGE_REG_F4];
  int tq[STAGE_REG_F4], cq[STAGE_REG_F4];  // token and float4 column of q = tid + nt*j
  if (inreg) {
    {
      int tok = tid / per, c = tid - tok * per;
#pragma unroll
      for (int j = 0; j < STAGE_REG_F4; ++j) {
        tq[j] = tok;
        cq[j] = c;
        c += nt;
        while (c >= per) {
          c -= per;
          ++tok;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < STAGE_REG_F4; ++j) {
      const int q = tid + nt * j;
      v[j] = q < Q ? load_residual4(p, l, hin, q) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < STAGE_REG_F4; ++j) {
      const int q = tid + nt * j;
      if (q >= q0 && q < q1) hout4[q] = v[j];
    }
    for (int tok = 0; tok < M; ++tok) {
      float ss = 0.0f, am = 0.0f;
#pragma unroll
      for (int j = 0; j < STAGE_REG_F4; ++j)
        if (tq[j] == tok) accumulate4(v[j], ss, am);  // q >= Q: token M, never matched
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      }
      if (lane == 0) {
        s_part[tok * STEP_CONSUMERS + warp] = ss;
        s_amx[tok * STEP_CONSUMERS + warp] = am;
      }
    }
  } else {
    // Streamed in batches of STAGE_BATCH independent loads.  H/4 is a multiple of 32,
    // so the 32 consecutive q of a warp share one token, and a thread's q only grow:
    // each warp meets each of its tokens in one run and reduces it when the run ends.
    for (int e = tid; e < M * STEP_CONSUMERS; e += nt) {
      s_part[e] = 0.0f;
      s_amx[e] = 0.0f;
    }
    csync();
    int cur = -1;
    float ss = 0.0f, am = 0.0f;
    auto flush = [&]() {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      }
      if (lane == 0) {
        s_part[cur * STEP_CONSUMERS + warp] = ss;
        s_amx[cur * STEP_CONSUMERS + warp] = am;
      }
    };
    for (int qb = tid; qb < Q; qb += STAGE_BATCH * nt) {
      float4 w[STAGE_BATCH];
#pragma unroll
      for (int j = 0; j < STAGE_BATCH; ++j) {
        const int q = qb + j * nt;
        w[j] = q < Q ? load_residual4(p, l, hin, q) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < STAGE_BATCH; ++j) {
        const int q = qb + j * nt;
        if (q < Q) {  // uniform across the warp (Q is a multiple of 32)
          const int tok = q / per;
          if (tok != cur) {
            if (cur >= 0) flush();
            cur = tok;
            ss = 0.0f;
            am = 0.0f;
          }
          if (q >= q0 && q < q1) hout4[q] = w[j];
          accumulate4(w[j], ss, am);
        }
      }
    }
    if (cur >= 0) flush();
  }
  csync();
  if (tid < M) {
    float ss = 0.0f, am = 0.0f;
    for (int w = 0; w < STEP_CONSUMERS; ++w) {
      ss += s_part[tid * STEP_CONSUMERS + w];
      am = fmaxf(am, s_amx[tid * STEP_CONSUMERS + w]);
    }
    const float r = l == 0 ? 1.0f : 1.0f / sqrtf(ss / (float)H + p.eps);
    s_r[tid] = r;
    s_sh[tid] = f16_range_shift(__bfloat162float(__float2bfloat16_rn(am * r)));
  }
  csync();
  if (inreg) {
#pragma unroll
    for (int j = 0; j < STAGE_REG_F4; ++j)
      if (tq[j] < M)
        write_layer_input4(xb16, xf16, tq[j] * xss + 8 * cq[j], tq[j] * xss + 8 * cq[j], v[j], s_r[tq[j]],
                           s_sh[tq[j]]);
  } else {
    for (int qb = tid; qb < Q; qb += STAGE_BATCH * nt) {
      float4 w[STAGE_BATCH];
#pragma unroll
      for (int j = 0; j < STAGE_BATCH; ++j) {
        const int q = qb + j * nt;
        w[j] = q < Q ? load_residual4(p, l, hin, q) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < STAGE_BATCH; ++j) {
        const int q = qb + j * nt;
        if (q < Q) {
          const int tok = q / per, c = q - tok * per;
          write_layer_input4(xb16, xf16, tok * xss + 8 * c, tok * xss + 8 * c, w[j], s_r[tok], s_sh[tok]);
        }
      }
    }
  }
  csync();  // also orders this block's slice stores before the h-init hand-off
}

// Top-k of every token from the complete router logits (same rule as k_dense:
// largest logit, lowest index on ties), then the union plan.  Candidates are ranked
// by one 64-bit order key, (logit key << 32) | ~expert, so a larger order key is the
// better candidate and no two are equal.
__device__ __forceinline__ unsigned long long order_key(uint32_t key, int e) {
  return ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)e);
}
constexpr int TOPK_CAND = 32;  // survivors ranked directly (one per lane)

// Exact k-round selection over all E logits of token tok by one warp (the path for
// tokens whose logits cluster above the survivor bound): each round takes the
// largest remaining order key.  Writes the k order keys, best first, to sel[].
__device__ __noinline__ void topk_token_full(const StepParams& p, int l, int tok, unsigned long long* sel,
                                             volatile int* abort_flag) {
  const int lane = threadIdx.x & 31, E = p.E;
  uint32_t key[32];  // expert lane + 32 i (E <= 1024)
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const unsigned long long* w[8];
    int n = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * (i + j);
      w[j] = p.logits + (size_t)tok * E + (e < E ? e : 0);
      if (e < E) n = j + 1;
    }
    float lv[8];
    if (!await_tagged(w, n, (uint32_t)l + 1u, lv, p.status, abort_flag)) n = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) key[i + j] = j < n ? float_key(lv[j]) : 0u;
  }
  for (int j = 0; j < p.k; ++j) {
    uint32_t bk = 0u;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (key[i] > bk) {  // strict: the first (lowest) index wins a tie within the lane
        bk = key[i];
        bi = lane + 32 * i;
      }
    const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
    const int mi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(bk == mk ? bi : 0x7fffffff));
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (lane + 32 * i == mi) key[i] = 0u;
    if (lane == 0) sel[j] = order_key(mk, mi);
  }
}

// Top-k of a window of tokens from the complete router logits (same rule as k_dense:
// largest logit, lowest index on ties), then the union plan.  The 8 consumer warps
// form TG token groups x EP expert parts (TG the largest power of two <= min(M, 8)
// whose parts hold at most 256 experts): each keeps its part's top-k of its tokens
// (a global top-k element is always in its part's top-k, ties included), then one
// warp per token merges the EP*k candidates.
template <bool DBG>
__device__ void step_topk_win(const StepParams& p, int l, Plan& P, int32_t* s_ids, float* s_wts, uint32_t* s_ck,
                          int32_t* s_ci, volatile int* s_abort_ptr) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E, k = p.k, M = p.M;
  int TG = 1;
  while (2 * TG <= M && 2 * TG <= STEP_CONSUMERS && E <= 256 * (STEP_CONSUMERS / (2 * TG))) TG *= 2;
  const int EP = STEP_CONSUMERS / TG;
  const int per = (E + EP - 1) / EP;  // experts per part (<= 256)
  const int part = warp % EP;
  const int e0 = part * per;
  for (int tok = warp / EP; tok < M; tok += TG) {
    uint32_t key[8];
    {
      const unsigned long long* w[8];
      int n = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int off = lane + 32 * i, e = e0 + off;
        w[i] = p.logits + tok * E + e;
        if (off < per && e < E) n = i + 1;  // valid columns are a prefix
      }
      float lv[8];
      if (!await_tagged(w, n, (uint32_t)l + 1u, lv, p.status, s_abort_ptr))
        n = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) key[i] = i < n ? float_key(lv[i]) : 0u;
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
          s_ck[(tok * STEP_CONSUMERS + part) * 8 + j] = mk;
          s_ci[(tok * STEP_CONSUMERS + part) * 8 + j] = mk ? mi : 0x7fffffff;
        }
      }
    }
  }
  csync();
  for (int tok = warp; tok < M; tok += STEP_CONSUMERS) {
    const int nc = EP * k;  // <= 64 candidates, two per lane
    uint32_t ck[2] = {0u, 0u};
    int ci[2] = {0x7fffffff, 0x7fffffff};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int c = lane + 32 * r;
      if (c < nc) {
        ck[r] = s_ck[(tok * STEP_CONSUMERS + c / k) * 8 + c % k];
        ci[r] = s_ci[(tok * STEP_CONSUMERS + c / k) * 8 + c % k];
      }
    }
    int sel_id = 0;
    uint32_t sel_key = 0u;
    for (int j = 0; j < k; ++j) {
      const int b = (ck[1] > ck[0] || (ck[1] == ck[0] && ci[1] < ci[0])) ? 1 : 0;
      const uint32_t bk = b ? ck[1] : ck[0];
      const int bi = b ? ci[1] : ci[0];
      const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
      const int mi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(bk == mk ? bi : 0x7fffffff));
#pragma unroll
      for (int r = 0; r < 2; ++r)
        if (ck[r] == mk && ci[r] == mi) {
          ck[r] = 0u;
          ci[r] = 0x7fffffff;
        }
      if (lane == j) {
        sel_id = mi;
        sel_key = mk;
      }
    }
    // an id outside [0, E) (only after a failed wait) is replaced by 0: nothing reads
    // out of bounds while the step winds down
    sel_id = (unsigned)sel_id < (unsigned)E ? sel_id : 0;
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
      if constexpr (DBG) {
        if (blockIdx.x == 0) {
          const size_t o = ((size_t)l * M + tok) * k + lane;
          if (p.ids_trace) p.ids_trace[o] = sel_id;
          if (p.w_trace) p.w_trace[o] = wj;
        }
      }
    }
  }
  csync();
  if (warp == 0) build_plan(P, s_ids, s_wts, M, k, E);
  csync();
}

// ---------------------------------------------------------------------------
// one-token MXFP4 row products (the routed experts at M = 1)
// ---------------------------------------------------------------------------
// R MXFP4 rows (codes rows[q], E8M0 scales scs[q], nb blocks of 32) against one f16
// activation row xc (chunk-major, scaled by 2^sh), lanes along K: each group of LPR
// lanes takes blocks l, l+LPR, ... (l = lane % LPR) of all R rows, so the activation
// chunks load once for R rows.  Products exact in fp32, summed per block; the block
// factor 2^(e - 127 - sh) applied in fp32.  Fast factors (SAFE false) are the normal
// number with exponent byte e - sh; a block with e - sh outside [1, 254] sets `bad`
// and the caller repeats the rows with SAFE (clamped factors, exact down to 2^-149).
// Every lane of the group returns the R row sums.  All 32 lanes must call it.
template <int LPR, int R, bool SAFE>
__device__ __forceinline__ void rows_dot_m1(const uint8_t* const (&rows)[R], const uint8_t* const (&scs)[R], int nb,
                                            const uint8_t* xc, int sh, bool& bad, float (&out)[R]) {
  const int l = threadIdx.x & (LPR - 1);
  float a[R];
#pragma unroll
  for (int q = 0; q < R; ++q) a[q] = 0.0f;
  // one block per iteration, not unrolled: the loop is entered once per row set, and a
  // compact body stays in the instruction cache
#pragma unroll 1
  for (int b = l; b < nb; b += LPR) {
    uint32_t xw[16];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint4 X = lds128(xc + (w * nb + b) * 16);
      xw[4 * w] = X.x;
      xw[4 * w + 1] = X.y;
      xw[4 * w + 2] = X.z;
      xw[4 * w + 3] = X.w;
    }
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const uint4 C = lds128(rows[q] + 16 * b);
      const int e = scs[q][b];
      float f;
      if (SAFE) {
        f = pow2_clamped(e - 127 - sh);
      } else {
        const int d = e - sh;
        bad |= (unsigned)(d - 1) > 253u;
        f = __uint_as_float((uint32_t)d << 23);
      }
      const uint32_t cw[4] = {C.x, C.y, C.z, C.w};
      uint32_t hv[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) e2m1x8_to_f16x2(cw[k], hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
      float p0 = 0.0f, p1 = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        p0 = fma_f16_lo(hv[j], xw[j], p0);
        p1 = fma_f16_hi(hv[j], xw[j], p1);
      }
      a[q] = fmaf(p0 + p1, f, a[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < R; ++q) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) a[q] += __shfl_xor_sync(0xffffffffu, a[q], o);
    out[q] = a[q];
  }
}
template <int LPR, int R>
__device__ __forceinline__ void rows_dot_m1_safe(const uint8_t* const (&rows)[R], const uint8_t* const (&scs)[R], int nb,
                                              const uint8_t* xc, int sh, float (&out)[R]) {
  bool bad = false;
  rows_dot_m1<LPR, R, true>(rows, scs, nb, xc, sh, bad, out);
}
// rows_dot_m1 with the fast factors, repeated out of line with exact clamped ones when
// any lane of the warp met a block outside the fast range.
template <int LPR, int R>
__device__ __forceinline__ void rows_dot_m1_exact(const uint8_t* const (&rows)[R], const uint8_t* const (&scs)[R], int nb,
                                                  const uint8_t* xc, int sh, float (&out)[R]) {
  bool bad = false;
  rows_dot_m1<LPR, R, false>(rows, scs, nb, xc, sh, bad, out);
  if (__any_sync(0xffffffffu, bad)) rows_dot_m1_safe<LPR, R>(rows, scs, nb, xc, sh, out);
}

// The one-token layer input: x = bf16(RMSNorm(h)) (layer 0: the given x) as bf16 at xb16
// and as f16 scaled by 2^sh (largest magnitude in [2^14, 2^15)) chunk-major at xf16; the
// same pass copies this block's slice [q0, q1) of h into hout.  Every thread forms the
// norm and the shift from the 8 warp partials in the same order, so every block gets
// the same bits (each block takes the top-k itself).  One barrier.
__device__ void stage1(const StepParams& p, int l, const float* hin, float* hout, uint8_t* xb16, uint8_t* xf16,
                       float* s_part, float* s_amx, int* s_sh, int q0, int q1) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nt = 32 * STEP_CONSUMERS;
  const int H = p.H, Q = H / 4, nb = H / 32;
  float4 v[STAGE_REG_F4];
  float ss = 0.0f, am = 0.0f;
#pragma unroll
  for (int j = 0; j < STAGE_REG_F4; ++j) {
    const int q = tid + nt * j;
    v[j] = q < Q ? load_residual4(p, l, hin, q) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int j = 0; j < STAGE_REG_F4; ++j) {
    const int q = tid + nt * j;
    if (q >= q0 && q < q1) reinterpret_cast<float4*>(hout)[q] = v[j];
    accumulate4(v[j], ss, am);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  if (lane == 0) {
    s_part[warp] = ss;
    s_amx[warp] = am;
  }
  csync();
  float t = 0.0f, a = 0.0f;
#pragma unroll
  for (int w = 0; w < STEP_CONSUMERS; ++w) {
    t += s_part[w];
    a = fmaxf(a, s_amx[w]);
  }
  const float r = l == 0 ? 1.0f : 1.0f / sqrtf(t / (float)H + p.eps);
  const int sh = f16_range_shift(__bfloat162float(__float2bfloat16_rn(a * r)));
  if (tid == 0) s_sh[0] = sh;
  const float f1 = exp2i(sh / 2), f2 = exp2i(sh - sh / 2);
#pragma unroll
  for (int j = 0; j < STAGE_REG_F4; ++j) {
    const int q = tid + nt * j;
    if (q < Q) {
      const __nv_bfloat162 b0 = __floats2bfloat162_rn(v[j].x * r, v[j].y * r);
      const __nv_bfloat162 b1 = __floats2bfloat162_rn(v[j].z * r, v[j].w * r);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&b0);
      u.y = *reinterpret_cast<const uint32_t*>(&b1);
      *reinterpret_cast<uint2*>(xb16 + 8 * q) = u;
      const __half2 h0 = __floats2half2_rn((__low2float(b0) * f1) * f2, (__high2float(b0) * f1) * f2);
      const __half2 h1 = __floats2half2_rn((__low2float(b1) * f1) * f2, (__high2float(b1) * f1) * f2);
      u.x = *reinterpret_cast<const uint32_t*>(&h0);
      u.y = *reinterpret_cast<const uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(xf16 + chunk_major_off(4 * q, nb)) = u;
    }
  }
  csync();  // also orders this block's slice stores before the h-init hand-off
}

// One token's top-k and routing plan.  Warp w holds experts [w*per, (w+1)*per),
// per = E/8 (at most 4 per lane); the smallest of the 8 warp maxima bounds the k-th
// largest logit, the survivors (at most TOPK_CAND, else the exact k-round selection)
// are ranked by their order keys, and warp 0 writes the plan directly: the k selected
// experts are distinct, so slot i holds the i-th smallest id with its weight.
template <bool DBG>
__device__ void topk1(const StepParams& p, int l, Plan& P, uint32_t* s_wmax, int* s_ncand,
                      unsigned long long* s_cand, unsigned long long* s_sel, volatile int* s_abort_ptr) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int E = p.E, k = p.k;
  const int per = E / STEP_CONSUMERS;
  const int e0 = warp * per;
  if (tid == 0) s_ncand[0] = 0;
  uint32_t key[4];
  {
    const unsigned long long* w[8];
    int n = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int off = lane + 32 * i;
      w[i] = p.logits + e0 + (i < 4 && off < per ? off : 0);
      if (i < 4 && off < per) n = i + 1;
    }
    float lv[8];
    if (!await_tagged(w, n, (uint32_t)l + 1u, lv, p.status, s_abort_ptr)) n = 0;
    uint32_t mx = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      key[i] = i < n ? float_key(lv[i]) : 0u;
      mx = max(mx, key[i]);
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) s_wmax[warp] = mx;
  }
  if (tid == 0) blk_stamp<DBG>(p, l, 8);
  csync();
  uint32_t bound = 0xFFFFFFFFu;
#pragma unroll
  for (int w = 0; w < STEP_CONSUMERS; ++w) bound = min(bound, s_wmax[w]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int off = lane + 32 * i;
    if (off < per && key[i] >= bound) {
      const int pos = atomicAdd(&s_ncand[0], 1);
      if (pos < TOPK_CAND) s_cand[pos] = order_key(key[i], e0 + off);
    }
  }
  if (tid == 0) blk_stamp<DBG>(p, l, 9);
  csync();
  if (warp == 0) {
    const int n = s_ncand[0];
    if (n <= TOPK_CAND) {
      const unsigned long long mine = lane < n ? s_cand[lane] : 0ull;
      int rank = 0;
      for (int j = 0; j < n; ++j) rank += s_cand[j] > mine ? 1 : 0;
      if (lane < n && rank < k) s_sel[rank] = mine;
    } else {
      topk_token_full(p, l, 0, s_sel, s_abort_ptr);
    }
    __syncwarp();
    // lane j holds the j-th selection; softmax over the selected logits
    // an id outside [0, E) (only after a failed wait) is replaced by 0: nothing reads out of bounds
    const unsigned long long sj = lane < k ? s_sel[lane] : 0ull;
    int id = (int)(~(uint32_t)sj);
    id = (unsigned)id < (unsigned)E ? id : 0;
    const float lj = key_float((uint32_t)(sj >> 32));
    const float l0 = __shfl_sync(0xffffffffu, lj, 0);
    const float ex = lane < k ? expf(lj - l0) : 0.0f;
    float den = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float wj = ex / den;
    // plan: slot = number of selected ids below this one
    int slot = 0;
    for (int i = 0; i < k; ++i) slot += __shfl_sync(0xffffffffu, id, i) < id ? 1 : 0;
    if (lane < k) {
      P.ids[slot] = id;
      P.w[slot][0] = wj;
      if constexpr (DBG) {
        if (blockIdx.x == 0) {
          const size_t o = (size_t)l * k + lane;
          if (p.ids_trace) p.ids_trace[o] = id;
          if (p.w_trace) p.w_trace[o] = wj;
        }
      }
    }
    if (lane == 0) P.n_unique = k;
  }
  if (tid == 0) blk_stamp<DBG>(p, l, 12);
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

// One token (M = 1) on the CUDA cores: column n of the four reads shared-memory row
// (rmap >> 4n) & 3; lane L covers K columns 8L + 256j.  Exact bf16 products summed in
// fp32 against act0 (plus act1 when given: a hi/lo split of one fp32 row); every lane
// returns all four column sums.
__device__ __forceinline__ void rows4_dot_m1(const uint8_t* wrows, uint32_t wstride, uint32_t rmap,
                                             const uint8_t* act0, const uint8_t* act1, int K, float (&o)[4]) {
  const int lane = threadIdx.x & 31;
  float a[4][2];
#pragma unroll
  for (int n = 0; n < 4; ++n) a[n][0] = a[n][1] = 0.0f;
  const uint8_t* wr[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) wr[n] = wrows + (size_t)((rmap >> (4 * n)) & 3u) * wstride;
#pragma unroll 2
  for (int k = 8 * lane; k < K; k += 256) {
    const uint4 X = lds128(act0 + 2 * k);
    const uint32_t xw[4] = {X.x, X.y, X.z, X.w};
    uint32_t yw[4] = {0u, 0u, 0u, 0u};
    if (act1) {
      const uint4 Y = lds128(act1 + 2 * k);
      yw[0] = Y.x; yw[1] = Y.y; yw[2] = Y.z; yw[3] = Y.w;
    }
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const uint4 W = lds128(wr[n] + 2 * k);
      const uint32_t ww[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a[n][0] = fma_bf16_lo(ww[j], xw[j], a[n][0]);
        a[n][1] = fma_bf16_hi(ww[j], xw[j], a[n][1]);
      }
      if (act1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          a[n][0] = fma_bf16_lo(ww[j], yw[j], a[n][0]);
          a[n][1] = fma_bf16_hi(ww[j], yw[j], a[n][1]);
        }
      }
    }
  }
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    float v = a[n][0] + a[n][1];
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
    o[n] = v;
  }
}

// ONE: the one-token instantiation (lanes-along-K products, chunk-major activations);
// otherwise a verify window of M >= 2 tokens (tensor-core tiles).  Separate
// instantiations keep each one's code small enough for the instruction caches.
template <bool ONE, bool DBG>
__global__ void __launch_bounds__(STEP_THREADS, 1) k_step(const __grid_constant__ StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ float s_part[MAX_M * STEP_CONSUMERS];
  __shared__ float s_r[MAX_M];
  __shared__ int s_ash[CR_CACHE][MAX_M];  // f16 shift of each staged routed activation
  __shared__ int32_t s_ids[MAX_SLOTS];
  __shared__ float s_wts[MAX_SLOTS];
  __shared__ float s_amx[MAX_M * STEP_CONSUMERS];
  __shared__ int s_sh[MAX_M];
  __shared__ uint32_t s_wmax[MAX_M * STEP_CONSUMERS];
  __shared__ uint32_t s_ck[ONE ? 1 : MAX_M * STEP_CONSUMERS * 8];
  __shared__ int32_t s_ci[ONE ? 1 : MAX_M * STEP_CONSUMERS * 8];
  __shared__ int s_ncand[MAX_M];
  __shared__ unsigned long long s_cand[MAX_M * TOPK_CAND];
  __shared__ unsigned long long s_sel[MAX_M * 8];
  __shared__ unsigned long long s_vst[STEP_SLOTS];
  __shared__ int s_gdone[STEP_SLOTS];  // tiles of a grouped ring item finished so far
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = ONE ? 1 : p.M, H = p.H, I = p.I, Is = p.Is, L = p.L;
  const uint32_t R = p.ring_bytes;
  const unsigned G = gridDim.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + STEP_SLOTS;
  uint64_t* plan_bar = empty + STEP_SLOTS;  // consumers -> producer: this layer's plan is built
  uint64_t* hinit_bar = plan_bar + 1;       // consumers -> producer: this block's h slice is copied
  uint8_t* ring = smem + STEP_FIXED;
  uint8_t* act = ring + R;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t sss = Is > 0 ? padded_stride(2u * Is) : 0u;
  const uint32_t ass = padded_stride(2u * I);
  uint8_t* xb16 = act;                    // A phase: bf16 x rows [M][xss]
  uint8_t* xf16 = act + (size_t)M * xss;  // B phase: f16 x rows  [M][xss] (one token: chunk-major)
  uint8_t* shi = step_shared_over_xb16(H, Is) ? act : act + 2 * (size_t)M * xss;  // CS: shared a, bf16 hi
  uint8_t* slo = shi + (size_t)M * sss;                                            //     bf16 lo
  uint8_t* afc = act;                     // CR phase: routed a of the block's experts [CR_CACHE][M][ass]
  const uint32_t bytesA = step_item_bytes(IT_A, H, I, Is), bytesS = step_item_bytes(IT_CS, H, I, Is);
  const uint32_t bytesB = step_item_bytes(IT_B, H, I, Is), bytesC = step_item_bytes(IT_CR, H, I, Is);
  const int capB = step_group_cap(R, bytesB, 8), capC = step_group_cap(R, bytesC, 16);
  static_assert(STEP_CONSUMERS == 8, "window groups: at most one W13 and two W2 tiles per consumer warp");

  if (tid == 0) {
    for (int s = 0; s < STEP_SLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(plan_bar, 1);
    mbar_init(hinit_bar, 1);
    for (int s = 0; s < STEP_SLOTS; ++s) s_gdone[s] = 0;
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  // ---------------- producer ----------------
  if (warp == STEP_CONSUMERS) {
    Producer<DBG> pr{p, ring, R, full, empty, s_vst, policy_evict_first(), 0, 0, RingCursor{0ull, 0u}, &s_abort, lane};
    bool ok = true;
    for (int l = 0; l < L && ok; ++l) {
      const LayerPtrs& Lp = p.layer[l];
      Work W;
      W.init_fixed(p);
      for (int r = 0; r < W.nA + W.nS && ok; ++r) ok = pr.issue(Lp, P, W.at(p, r));
      if (!ok) break;
      stamp<DBG>(p, l, 12);
      int got = 1;
      // the consumers' slice copy of h (ordered before their arrive by a block
      // barrier) is published here, off their critical path: fence, then count
      if (lane == 0) {
        got = ring_wait(hinit_bar, (uint32_t)(l & 1), p.status, &s_abort);
        if (got) signal_counter(p.ctr + (size_t)l * CTR_PER_LAYER + CTR_HINIT);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      if (lane == 0) got = ring_wait(plan_bar, (uint32_t)(l & 1), p.status, &s_abort);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      stamp<DBG>(p, l, 13);
      W.init_routed(p, P.n_unique);
      stamp<DBG>(p, l, 15);
      {
        int u, r0, nt;
        GroupWalk gb{W.b0, W.b0 + W.nB, p.I / 8, capB};
        while (ok && gb.next(u, r0, nt)) ok = pr.issue_b(Lp, P, u, r0, nt);
        GroupWalk gc{W.c0, W.c0 + W.nC, p.H / 16, capC};
        while (ok && gc.next(u, r0, nt)) ok = pr.issue_c(Lp, P, u, r0, nt);
      }
      stamp<DBG>(p, l, 14);
    }
    // every copy issued lands before the block may exit
    if (lane == 0)
      for (long long j = (pr.i > STEP_SLOTS ? pr.i - STEP_SLOTS : 0); j < pr.i; ++j)
        drain_wait(&full[j % STEP_SLOTS], (uint32_t)((j / STEP_SLOTS) & 1));
    return;
  }

  // ---------------- consumers ----------------
  unsigned* ctr = p.ctr;
  const int QH = M * (H / 4);  // float4s of the residual
  const int slice_q0 = (int)((long long)QH * blockIdx.x / G), slice_q1 = (int)((long long)QH * (blockIdx.x + 1) / G);
  long long i = 0;   // ring item
  RingCursor pos{0ull, 0u};  // virtual ring cursor (same walk as the producer's)
  for (int l = 0; l < L; ++l) {
    unsigned* lc = ctr + (size_t)l * CTR_PER_LAYER;
    float* hout = p.h + (size_t)(l & 1) * M * H;
    const float* hin = p.h + (size_t)((l + 1) & 1) * M * H;  // layer l-1's buffer
    stamp<DBG>(p, l, 0);
    if (l > 0) {
      if (tid == 0) wait_counter(ctr + (size_t)(l - 1) * CTR_PER_LAYER + CTR_H, G, p.status, &s_abort);
      csync();
    }
    stamp<DBG>(p, l, 1);
    if (tid == 0) blk_stamp<DBG>(p, l, 0);
    if constexpr (ONE)
      stage1(p, l, hin, hout, xb16, xf16, s_part, s_amx, s_sh, slice_q0, slice_q1);
    else
      stage_window_input(p, l, hin, hout, xb16, xf16, xss, s_part, s_amx, s_r, s_sh, slice_q0, slice_q1);
    if (tid == 0) mbar_arrive(hinit_bar);
    stamp<DBG>(p, l, 2);
    if (tid == 0) blk_stamp<DBG>(p, l, 1);
    if (DBG && blockIdx.x == 0 && (p.x_trace || p.h_trace)) {
      for (int e = tid; e < M * H; e += 32 * STEP_CONSUMERS) {
        const int tok = e / H, c = e % H;
        const __nv_bfloat16 xv = *reinterpret_cast<const __nv_bfloat16*>(xb16 + tok * xss + 2 * c);
        const float hv = l == 0 ? __bfloat162float(p.x_in[e]) : __ldcg(hin + e);
        if (p.x_trace) p.x_trace[(size_t)l * M * H + e] = xv;
        if (p.h_trace) p.h_trace[(size_t)l * M * H + e] = hv;
      }
    }

    // ---- A: router items (4 experts) and shared-W13 items (2 gate + 2 up rows) ----
    Work W;
    W.init_fixed(p);
    const int nr = p.E / 4;
    for (int r = 0; r < W.nA; ++r) {
      const uint8_t* src;
      uint64_t* eb;
      bool ready;
      {
        const uint32_t s0 = ring_take(pos, bytesA, R);
        const long long ii = i++;
        if ((int)(ii % STEP_CONSUMERS) != warp) continue;
        const int slot = (int)(ii % STEP_SLOTS);
        src = ring + s0;
        eb = &empty[slot];
        item_stamp<DBG>(p, ii, 3);
        ready = ring_wait(&full[slot], (uint32_t)((ii / STEP_SLOTS) & 1), p.status, &s_abort);
      }
      ready = __all_sync(0xffffffffu, ready);
      const Item it = W.at(p, r);
      const bool router = it.a < nr;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      if (ready) {
        // shared items: columns (0,1,2,3) = (gate 2s, up 2s, gate 2s+1, up 2s+1) from
        // smem rows (0, 2, 1, 3), so a thread's two columns are a (gate, up) pair
        if constexpr (ONE) {
          float o[4];
          rows4_dot_m1(src, 2u * H, router ? 0x3210u : 0x3120u, xb16, nullptr, H, o);
          c[0] = t == 0 ? o[0] : o[2];
          c[1] = t == 0 ? o[1] : o[3];
        } else {
          const int wrow = g < 4 ? (router ? g : ((g & 1) ? 2 : 0) + (g >> 1)) : -1;
          rows4_dot(src, 2u * H, wrow, g < M ? xb16 + g * xss : nullptr, nullptr, H, c);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(eb);
      if (t < 2 && g < M) {
        const uint32_t tag = (uint32_t)l + 1u;
        if (router) {
          st_tagged(p.logits + g * p.E + 4 * it.a + 2 * t, c[0], tag);
          st_tagged(p.logits + g * p.E + 4 * it.a + 2 * t + 1, c[1], tag);
          if (lane == 0) blk_stamp<DBG>(p, l, 2);
        } else {
          st_tagged(p.a_shared + g * Is + 2 * (it.a - nr) + t, silu_f32(c[0]) * c[1], tag);
        }
      }
    }
    stamp<DBG>(p, l, 3);
    if (tid == 0) blk_stamp<DBG>(p, l, 3);

    // ---- top-k and plan (every block, identical; polls the tagged logits) ----
    stamp<DBG>(p, l, 4);
    if constexpr (ONE)
      topk1<DBG>(p, l, P, s_wmax, s_ncand, s_cand, s_sel, &s_abort);
    else
      step_topk_win<DBG>(p, l, P, s_ids, s_wts, s_ck, s_ci, &s_abort);
    if (tid == 0) mbar_arrive(plan_bar);
    stamp<DBG>(p, l, 5);
    if (tid == 0) blk_stamp<DBG>(p, l, 4);

    // ---- CS: shared W2 (activation as bf16 hi + lo), accumulated into h, ahead of the
    //      routed tiles whose copies it waits for ----
    {
      if (W.nS > 0) {
        for (int e = tid; e < M * (Is / 8); e += 32 * STEP_CONSUMERS) {
          const int tok = e / (Is / 8), c8 = e % (Is / 8);
          const unsigned long long* w[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) w[j] = p.a_shared + (size_t)tok * Is + 8 * c8 + j;
          float a8[8];
          if (!await_tagged(w, 8, (uint32_t)l + 1u, a8, p.status, &s_abort)) {
#pragma unroll
            for (int j = 0; j < 8; ++j) a8[j] = 0.0f;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(a8[j]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(a8[j] - __bfloat162float(hi));
            *reinterpret_cast<__nv_bfloat16*>(shi + tok * sss + 2 * (8 * c8 + j)) = hi;
            *reinterpret_cast<__nv_bfloat16*>(slo + tok * sss + 2 * (8 * c8 + j)) = lo;
          }
        }
      }
      if (tid == 0) wait_counter(lc + CTR_HINIT, G, p.status, &s_abort);  // every slice of h initialised
      csync();
      stamp<DBG>(p, l, 6);
      for (int r = 0; r < W.nS; ++r) {
        const uint8_t* src;
        uint64_t* eb;
        bool ready;
        {
          const uint32_t s0 = ring_take(pos, bytesS, R);
          const long long ii = i++;
          if ((int)(ii % STEP_CONSUMERS) != warp) continue;
          const int slot = (int)(ii % STEP_SLOTS);
          src = ring + s0;
          eb = &empty[slot];
          item_stamp<DBG>(p, ii, 3);
          ready = ring_wait(&full[slot], (uint32_t)((ii / STEP_SLOTS) & 1), p.status, &s_abort);
        }
        ready = __all_sync(0xffffffffu, ready);
        const Item it = W.at(p, W.nA + r);
        // 4 output rows (N) against the activation rows m = 2*token + {hi, lo} (M)
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        if (ready) {
          if constexpr (ONE) {
            // the full hi + lo sum lands in lane group 0; group 1 adds zeros below
            float o[4];
            rows4_dot_m1(src, 2u * Is, 0x3210u, shi, slo, Is, o);
            c[0] = g == 0 ? (t == 0 ? o[0] : o[2]) : 0.0f;
            c[1] = g == 0 ? (t == 0 ? o[1] : o[3]) : 0.0f;
          } else {
            const uint8_t* sa = (g & 1) ? slo : shi;
            const int t0 = g >> 1, t1 = 4 + (g >> 1);
            rows4_dot(src, 2u * Is, g < 4 ? g : -1, t0 < M ? sa + t0 * sss : nullptr,
                      t1 < M ? sa + t1 * sss : nullptr, Is, c);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(eb);
        // hi + lo: rows m = 2tok (lane group g even) and 2tok + 1 (g odd)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] += __shfl_xor_sync(0xffffffffu, c[e], 4);
        if ((g & 1) == 0 && t < 2) {
          const int t0 = g >> 1, t1 = 4 + (g >> 1);
          if (t0 < M) {
            atomicAdd(hout + (size_t)t0 * H + it.a + 2 * t, c[0]);
            atomicAdd(hout + (size_t)t0 * H + it.a + 2 * t + 1, c[1]);
          }
          if (t1 < M) {
            atomicAdd(hout + (size_t)t1 * H + it.a + 2 * t, c[2]);
            atomicAdd(hout + (size_t)t1 * H + it.a + 2 * t + 1, c[3]);
          }
        }
      }
      stamp<DBG>(p, l, 7);
      if (tid == 0) blk_stamp<DBG>(p, l, 5);
    }

    // ---- B: routed W13 + SwiGLU ----
    // Groups of consecutive tiles of one expert share a ring item.  One token: the
    // units (gate row, up row of one intermediate index) of the block's range go
    // round-robin to the 16 half-warps, each unit a lanes-along-K product over its two
    // rows.  A window: tile j of a group (global tile tc + j of this phase) is computed
    // by warp (tc + j) % 8 on the tensor core.  The last warp to finish a group's
    // share releases the group; expert u's counter reaches I (one token: units) or
    // I/8 (a window: tiles) when its activations are complete.
    W.init_routed(p, P.n_unique);
    if constexpr (ONE) {
      GroupWalk gb{W.b0, W.b0 + W.nB, p.I / 8, capB};
      int u, r0, nt, q0 = 0;
      const int hw = 2 * warp + (lane >> 4);  // half-warp 0..15
      while (gb.next(u, r0, nt)) {
        const uint32_t codes = (uint32_t)nt * 8u * (H / 2), scales = (uint32_t)nt * 8u * (H / 32);
        const uint32_t s0 = ring_take(pos, 2 * codes + 2 * scales, R);
        const int slot = (int)(i % STEP_SLOTS);
        const int U = 8 * nt;
        const int f = ((hw - q0) % 16 + 16) % 16;  // my first unit of the group
        const int nmine = f < U ? (U - 1 - f) / 16 + 1 : 0;
        const int nw = max(__shfl_sync(0xffffffffu, nmine, 0), __shfl_sync(0xffffffffu, nmine, 16));
        if (nw > 0) {
          item_stamp<DBG>(p, i, 3);
          const bool ready =
              __all_sync(0xffffffffu, ring_wait(&full[slot], (uint32_t)((i / STEP_SLOTS) & 1), p.status, &s_abort));
          item_stamp<DBG>(p, i, 1);
          const uint8_t* gate = ring + s0;
          const uint8_t* up = gate + codes;
          const uint8_t* gs = gate + 2 * codes;
          const uint8_t* us = gs + scales;
          for (int m = 0; m < nw; ++m) {
            const int q = f + 16 * m;
            const bool live = q < U;
            const int qq = live ? q : 0;
            const uint8_t* const rows[2] = {gate + qq * (H / 2), up + qq * (H / 2)};
            const uint8_t* const scs[2] = {gs + qq * (H / 32), us + qq * (H / 32)};
            float r[2] = {0.0f, 0.0f};
            if (ready) rows_dot_m1_exact<16, 2>(rows, scs, H / 32, xf16, s_sh[0], r);
            if (live && (lane & 15) == 0) p.a_routed[(size_t)u * I + 8 * r0 + q] = silu_f32(r[0]) * r[1];
          }
          __syncwarp();
          item_stamp<DBG>(p, i, 2);
          const int done = __shfl_sync(0xffffffffu, nmine, 0) + __shfl_sync(0xffffffffu, nmine, 16);
          if (lane == 0) {
            // the ring space goes back first: the publish below (fence, counter) no
            // longer needs the rows
            if (atomicAdd(&s_gdone[slot], done) + done == U) {
              s_gdone[slot] = 0;
              mbar_arrive(&empty[slot]);
            }
            if (done > 0) {
              __threadfence();
              atomicAdd(lc + CTR_EXP + u, (unsigned)done);
            }
          }
        }
        q0 += U;
        ++i;
      }
    } else {
      GroupWalk gb{W.b0, W.b0 + W.nB, p.I / 8, capB};
      int u, r0, nt, tc = 0;
      while (gb.next(u, r0, nt)) {
        const uint32_t codes = (uint32_t)nt * 8u * (H / 2), scales = (uint32_t)nt * 8u * (H / 32);
        const uint32_t s0 = ring_take(pos, 2 * codes + 2 * scales, R);
        const int slot = (int)(i % STEP_SLOTS);
        const int j0 = ((warp - tc) % STEP_CONSUMERS + STEP_CONSUMERS) % STEP_CONSUMERS;
        if (j0 < nt) {
          item_stamp<DBG>(p, i, 3);
          const bool ready = ring_wait(&full[slot], (uint32_t)((i / STEP_SLOTS) & 1), p.status, &s_abort);
          item_stamp<DBG>(p, i, 1);
          const uint8_t* gate = ring + s0;
          const uint8_t* up = gate + codes;
          const uint8_t* gs = gate + 2 * codes;
          const uint8_t* us = gs + scales;
          // groups hold at most capB <= STEP_CONSUMERS tiles: one tile per warp
          const int j = j0;
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          if (ready) {
            const int rg = 8 * j + g;  // tile row: gate row and up row of intermediate 8 (r0 + j) + g
            mxfp4_tile_dot_win(gate + rg * (H / 2), up + rg * (H / 2), gs + rg * (H / 32), us + rg * (H / 32),
                               H / 32, xf16, xss, M, s_sh, c);
          }
          __syncwarp();  // every lane is done reading the tile: its ring space goes back first
          item_stamp<DBG>(p, i, 2);
          if (lane == 0 && atomicAdd(&s_gdone[slot], 1) + 1 == nt) {
            s_gdone[slot] = 0;
            mbar_arrive(&empty[slot]);
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tok = 2 * t + e;
            if (tok < M) p.a_routed[((size_t)u * M + tok) * I + 8 * (r0 + j) + g] = silu_f32(c[e]) * c[2 + e];
          }
          __syncwarp();
          if (lane == 0) signal_counter(lc + CTR_EXP + u);
        }
        tc += nt;
        ++i;
      }
    }
    stamp<DBG>(p, l, 8);
    if (tid == 0) blk_stamp<DBG>(p, l, 6);
    csync();  // xf16 and the shared halves are dead: the routed-W2 activation copies take the region
    stamp<DBG>(p, l, 9);

    // ---- CR: routed W2 (weighted), accumulated into h ----
    // The block's contiguous range touches experts u_first..u_last (at most CR_CACHE,
    // checked by the host).  Warp w stages expert u_first + w's activation once its
    // W13 items are complete everywhere: f16 with its own power-of-two shift.
    const long long baseC = W.nA + W.nS + W.nB;
    const int u_first = W.nC > 0 ? W.at(p, baseC).a : 0;
    if (W.nC > 0) {
      const int u_last = W.at(p, baseC + W.nC - 1).a;
      const int u = u_first + warp;
      if (warp < CR_CACHE && u <= u_last) {
        if (lane == 0) wait_counter(lc + CTR_EXP + u, (unsigned)(ONE ? I : I / 8), p.status, &s_abort);
        __syncwarp();
        uint8_t* dst = afc + (size_t)warp * M * ass;
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
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int c4 = lane + 32 * jj;
            if (c4 < I / 4) {
              const __half2 h0 = __floats2half2_rn(mul_pow2(v[jj].x, sh), mul_pow2(v[jj].y, sh));
              const __half2 h1 = __floats2half2_rn(mul_pow2(v[jj].z, sh), mul_pow2(v[jj].w, sh));
              uint2 u2;
              u2.x = *reinterpret_cast<const uint32_t*>(&h0);
              u2.y = *reinterpret_cast<const uint32_t*>(&h1);
              *reinterpret_cast<uint2*>(dst + (ONE ? chunk_major_off(4 * c4, I / 32) : tok * ass + 8 * c4)) = u2;
            }
          }
          if (lane == 0) s_ash[warp][tok] = sh;
        }
      }
      csync();
    }
    if constexpr (ONE) {
      // one token: the block's W2 rows go round-robin to 32 row slots of 8 lanes (4
      // per warp), each slot taking its rows of a group two at a time (same expert:
      // the activation chunks load once for both), lanes along K
      GroupWalk gc{W.c0, W.c0 + W.nC, p.H / 16, capC};
      int u, c0, nt, q0 = 0;
      const int rs = 4 * warp + (lane >> 3);  // row slot 0..31
      while (gc.next(u, c0, nt)) {
        const uint32_t codes = (uint32_t)nt * 16u * (I / 2), scales = (uint32_t)nt * 16u * (I / 32);
        const uint32_t s0 = ring_take(pos, codes + scales, R);
        const int slot = (int)(i % STEP_SLOTS);
        const int Rg = 16 * nt;
        const int f = ((rs - q0) % 32 + 32) % 32;  // my first row of the group
        const int nmine = f < Rg ? (Rg - 1 - f) / 32 + 1 : 0;
        int nw = max(nmine, __shfl_xor_sync(0xffffffffu, nmine, 8));
        nw = max(nw, __shfl_xor_sync(0xffffffffu, nw, 16));
        if (nw > 0) {
          const int cu = u - u_first;  // cache entry
          const uint8_t* my_af = afc + (size_t)cu * ass;
          item_stamp<DBG>(p, i, 3);
          const bool ready =
              __all_sync(0xffffffffu, ring_wait(&full[slot], (uint32_t)((i / STEP_SLOTS) & 1), p.status, &s_abort));
          item_stamp<DBG>(p, i, 1);
          const uint8_t* cd = ring + s0;
          const uint8_t* sc = cd + codes;
          const float wt = P.w[u][0];
          for (int m = 0; m < nw; m += 2) {
            const int qa = f + 32 * m, qb = qa + 32;
            const bool la = qa < Rg, lb = qb < Rg;
            const int ra = la ? qa : 0, rb = lb ? qb : 0;
            const uint8_t* const rows[2] = {cd + ra * (I / 2), cd + rb * (I / 2)};
            const uint8_t* const scs[2] = {sc + ra * (I / 32), sc + rb * (I / 32)};
            float r[2] = {0.0f, 0.0f};
            if (ready) rows_dot_m1_exact<8, 2>(rows, scs, I / 32, my_af, s_ash[cu][0], r);
            if ((lane & 7) == 0 && wt != 0.0f) {
              if (la) atomicAdd(hout + 16 * c0 + qa, r[0] * wt);
              if (lb) atomicAdd(hout + 16 * c0 + qb, r[1] * wt);
            }
          }
          __syncwarp();
          item_stamp<DBG>(p, i, 2);
          int done = nmine + __shfl_xor_sync(0xffffffffu, nmine, 8);
          done += __shfl_xor_sync(0xffffffffu, done, 16);
          if (lane == 0 && atomicAdd(&s_gdone[slot], done) + done == Rg) {
            s_gdone[slot] = 0;
            mbar_arrive(&empty[slot]);
          }
        }
        q0 += Rg;
        ++i;
      }
    } else {
      GroupWalk gc{W.c0, W.c0 + W.nC, p.H / 16, capC};
      int u, c0, nt, tc = 0;
      while (gc.next(u, c0, nt)) {
        const uint32_t codes = (uint32_t)nt * 16u * (I / 2), scales = (uint32_t)nt * 16u * (I / 32);
        const uint32_t s0 = ring_take(pos, codes + scales, R);
        const int slot = (int)(i % STEP_SLOTS);
        const int j0 = ((warp - tc) % STEP_CONSUMERS + STEP_CONSUMERS) % STEP_CONSUMERS;
        if (j0 < nt) {
          const int cu = u - u_first;  // cache entry
          const uint8_t* my_af = afc + (size_t)cu * M * ass;
          item_stamp<DBG>(p, i, 3);
          const bool ready = ring_wait(&full[slot], (uint32_t)((i / STEP_SLOTS) & 1), p.status, &s_abort);
          item_stamp<DBG>(p, i, 1);
          const uint8_t* cd = ring + s0;
          const uint8_t* sc = cd + codes;
          // groups hold at most capC <= 2 * STEP_CONSUMERS tiles: one or two per warp,
          // both computed before the ring space goes back, then added into h
          const int ja = j0, jb = j0 + STEP_CONSUMERS;
          const int mine = jb < nt ? 2 : 1;
          float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          if (ready) {
#pragma unroll 1
            for (int q = 0; q < mine; ++q) {  // one inlined copy of the product
              const int j = q ? jb : ja;
              const int rg = 16 * j + g;  // tile rows rg and rg + 8: output rows 16 (c0 + j) + g (+8)
              float v[4];
              mxfp4_tile_dot_win(cd + rg * (I / 2), cd + (rg + 8) * (I / 2), sc + rg * (I / 32),
                                 sc + (rg + 8) * (I / 32), I / 32, my_af, ass, M, s_ash[cu], v);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                c[0][e] = q ? c[0][e] : v[e];
                c[1][e] = q ? v[e] : c[1][e];
              }
            }
          }
          __syncwarp();
          item_stamp<DBG>(p, i, 2);
          if (lane == 0 && atomicAdd(&s_gdone[slot], mine) + mine == nt) {
            s_gdone[slot] = 0;
            mbar_arrive(&empty[slot]);
          }
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int h0 = 16 * (c0 + (q ? jb : ja)) + g;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int tok = 2 * t + e;
              if (q < mine && tok < M) {
                const float wt = P.w[u][tok];
                if (wt != 0.0f) {
                  atomicAdd(hout + (size_t)tok * H + h0, c[q][e] * wt);
                  atomicAdd(hout + (size_t)tok * H + h0 + 8, c[q][2 + e] * wt);
                }
              }
            }
          }
        }
        tc += nt;
        ++i;
      }
    }
    stamp<DBG>(p, l, 10);
    csync();
    if (tid == 0) blk_stamp<DBG>(p, l, 7);
    if (tid == 0 && l != p.hold_layer) signal_counter(lc + CTR_H);
    stamp<DBG>(p, l, 11);
  }

  // ---- LM-head input: bf16(RMSNorm(h_L)) by block 0 ----
  if (blockIdx.x != 0) return;
  if (tid == 0) wait_counter(ctr + (size_t)(L - 1) * CTR_PER_LAYER + CTR_H, G, p.status, &s_abort);
  csync();
  const float* hf = p.h + (size_t)((L - 1) & 1) * M * H;
  for (int tok = 0; tok < M; ++tok) {
    float ss = 0.0f;
    for (int c = tid; c < H / 4; c += 32 * STEP_CONSUMERS) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(hf + (size_t)tok * H) + c);
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_part[tok * STEP_CONSUMERS + warp] = ss;
  }
  csync();
  if (tid < M) {
    float ss = 0.0f;
    for (int w = 0; w < STEP_CONSUMERS; ++w) ss += s_part[tid * STEP_CONSUMERS + w];
    s_r[tid] = 1.0f / sqrtf(ss / (float)H + p.eps);
  }
  csync();
  for (int e = tid; e < M * H; e += 32 * STEP_CONSUMERS) {
    const int tok = e / H;
    const float hv = __ldcg(hf + e);
    const __nv_bfloat16 v = __float2bfloat16_rn(hv * s_r[tok]);
    p.x_final[e] = v;
    if constexpr (DBG) {
      if (p.x_trace) p.x_trace[(size_t)L * M * H + e] = v;
      if (p.h_trace) p.h_trace[(size_t)L * M * H + e] = hv;
    }
  }
}

}  // namespace moe
