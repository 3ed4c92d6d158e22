// prefill_kernels.cuh -- one MoE layer over a prefill chunk (M tokens, M a multiple of
// 128) on the 5th-generation tensor cores.
//
// Source: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
// 三种方法), 方法/产品要点 items 1 and 3 (MXFP4 expert weights, 8 of 512 experts plus one
// shared expert); the prefill activations are MXFP8 (a power-of-two scale per 32
// elements along K, e4m3 codes) because the block-scaled MMA takes both operands in
// an MX format.
//
// Every GEMM of the layer is one launch of k_umma, a persistent warp-specialised
// kernel (one CTA per SM):
//   warp 4      TMA producer: per K chunk, one tensor copy for the weight tile (two
//               64-row halves -- gate/up, or consecutive rows -- through a 3-D map)
//               and one for the 64-token tile, into a ring of stages (the TMA engine
//               takes copies at a bounded rate, so every copy moves as much as it can);
//   warp 5      MMA issuer: one elected thread issues tcgen05.mma (M = 128 weight rows,
//               N = tokens, fp32 accumulator in tensor memory) and commits each stage
//               back to the producer and each finished tile to the epilogue;
//   warps 0-3   epilogue: tcgen05.ld of the accumulator (warp w owns TMEM lanes
//               32w..32w+31), the mode's arithmetic and the global stores; for the
//               block-scaled modes they also place the tile's E8M0 scale factors in
//               tensor memory (tcgen05.st) before its MMAs start -- with two column
//               buffers (K <= 3072) during the previous tile's MMAs, the producer having
//               fetched them a tile ahead.
// Modes: router logits (bf16 x bf16), shared W13 + SwiGLU (bf16), shared W2 (bf16,
// stores y), routed W13 + SwiGLU + MXFP8 re-quantisation (E2M1 x E4M3 block-scaled),
// routed W2 with the routing weight, added into y.
//
// Shared-memory operand layout: K-major, 128-byte swizzle (rows of 128 bytes, 8-row
// atoms of 1024 bytes).  E2M1 weights reach shared memory through the tensor map type
// that leaves an 8-byte gap after every 8 bytes (16 codes), the form the block-scaled
// MMA reads for 4-bit operands, so a 128-element K chunk is 128 bytes per row for
// every operand type.  Scale factors in tensor memory: the E8M0 of operand row m,
// K blocks 4c..4c+3 (one per byte, selected by the instruction's scale-factor id), is
// the 32-bit word at lane m % 32 + 32q (every q), column base + 4c + m / 32.
#pragma once

#include <cuda.h>

#include "decode_kernels.cuh"

namespace moe {

enum : int { PF_ROUTER = 0, PF_SH13 = 1, PF_SH2 = 2, PF_R13 = 3, PF_R2 = 4 };
constexpr int PF_THREADS = 192;        // warps 0-3 epilogue, 4 producer, 5 MMA
constexpr int PF_BN = 64;              // token tile (MMA N <= 64)
constexpr int PF_STAGE_BYTES = 24576;  // per K chunk: weight tile 16 KB + token tile 8 KB
constexpr int PF_MAX_STAGES = 9;
constexpr int PF_TMEM_COLS = 512;      // accumulators 0..63 and 64..127, then the scale columns
constexpr int PF_SF_COL = 128;         // first scale column: per buffer SFA (4 per K chunk), then SFB
constexpr int PF_MAX_CHUNKS = 32;      // K / 128 for the block-scaled modes (SF columns)

struct alignas(64) PrefillParams {
  // Both maps put the K chunk (64 bf16 or 128 E2M1 / E4M3 elements: 128 bytes a row in
  // shared memory) in an outer dimension, so one copy brings kc chunks, each landing as
  // the swizzled tile one chunk of MMAs reads.
  CUtensorMap tmA;  // weights: dims {chunk, rows, 2 halves, K / chunk}, box {chunk, 64, 2, kc}
  CUtensorMap tmB;  // activations: dims {chunk, rows, K / chunk}, box {chunk, 64, kc}
  CUtensorMap tmB32;  // routed modes: the same with 32-row boxes, for tiles of at most 32 tokens
  int mode;
  int K;
  int m_tiles;   // weight tiles per problem
  int up_off;    // 13 modes: row offset of the up half within a problem
  int prob_rows; // weight rows per problem (expert) for the routed modes
  int M;         // dense modes: tokens
  int E;
  const int* ntile_prefix;  // routed: [E+1] prefix sums of ceil(n_e / 128)
  const int* goff;          // routed: [E+1] first grouped row of each expert
  const uint16_t* tile_e;   // routed: [ntile_prefix[E]] expert of each 64-token tile
  const int32_t* g_tok;     // routed: [G] token of each grouped row
  const float* g_w;         // routed: [G] routing weight of each grouped row
  const uint8_t* sfa;       // routed: weight scales [rows][K/32]
  const uint8_t* sfb;       // routed: activation scales [G][sf_ld]
  int sf_ld;                // routed: bytes per activation-scale row (K/32 rounded up to 16)
  int out_ld;               // leading dimension of the output
  float* out_f32;           // router logits [M][E], y [M][H]
  __nv_bfloat16* out_bf16;  // shared activation [M][Is]
  uint8_t* out_q;           // routed activation e4m3 [G][I]
  uint8_t* out_qs;          // routed activation E8M0 [G][out_qs_ld]
  int out_qs_ld;
  int stages;
  int sf_bufs;  // block-scaled modes: shared-memory scale buffers (2, or 1 when two do not fit)
  int kc;  // K chunks per pipeline stage (one copy per operand per stage)
  int* status;
};

// ---------------------------------------------------------------------------
// tcgen05 / TMA primitives
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  tc_wait_ld();
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32
__device__ __forceinline__ void umma_bf16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// D[tmem] (+)= (A * 2^sfa)[smem] * (B * 2^sfb)[smem]^T, E2M1 x E4M3 with E8M0 per 32 of K
__device__ __forceinline__ void umma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc,
                                        uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}
// K-major operand, 128-byte swizzle: start >> 4, LBO 1 (unused when swizzled), SBO 1024 B
// between 8-row atoms, descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)64u << 32) | ((uint64_t)1u << 46) |
         ((uint64_t)2u << 61);
}
// Instruction descriptors (M = 128, both operands K-major).
__host__ __device__ inline uint32_t idesc_bf16(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__host__ __device__ inline uint32_t idesc_mx(int N, uint32_t sf_id) {
  return (sf_id << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(128 >> 4) << 24) | (sf_id << 29);
}

// Bounded mbarrier wait; once any thread of the CTA has given up, every later wait
// returns false at once, so all roles reach the final block barrier.  The first
// timeout of a workspace also records where it happened (status[4..7]: wait site,
// mode, block, parity).
enum : int { PFW_EMPTY = 1, PFW_DRAIN = 2, PFW_ACC_EMPTY = 3, PFW_SF = 4, PFW_FULL = 5, PFW_ACC_FULL = 6 };
__device__ __noinline__ bool pf_wait_slow(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag,
                                          int site, int mode) {
  const unsigned long long t0 = globaltimer_ns();
  for (unsigned n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) != 0) continue;  // the clock and the flag are read every 64 polls
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
      if (atomicCAS(status, 0, DEV_ERR_TIMEOUT) == 0) {
        status[4] = site;
        status[5] = mode;
        status[6] = (int)blockIdx.x;
        status[7] = (int)parity;
      }
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}
// Bounded mbarrier wait: the first try inline (a stage or tile that is ready costs no
// call), the polling loop out of line.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag, int site,
                                        int mode) {
  return mbar_try_wait(bar, parity) || pf_wait_slow(bar, parity, status, abort_flag, site, mode);
}

// ---------------------------------------------------------------------------
// work items
// ---------------------------------------------------------------------------
struct PfItem {
  int e;       // expert (routed modes)
  int mt;      // weight tile
  int n0;      // first token of the tile within the problem
  int ncnt;    // tokens in the tile
  int grow0;   // activation row of token n0
  int ya0, ya1;  // weight rows of the two 64-row halves
};

__host__ __device__ constexpr bool pf_routed(int mode) { return mode == PF_R13 || mode == PF_R2; }
__host__ __device__ constexpr bool pf_13(int mode) { return mode == PF_SH13 || mode == PF_R13; }

#ifdef PF_TIMELINE
#ifndef PF_TIMELINE_MODE
#define PF_TIMELINE_MODE PF_R13
#endif
// Profiling builds only (compiled with -DPF_TIMELINE; -DPF_TIMELINE_MODE picks the
// launch, the routed W13 one by default): block 0 of that launch
// stamps its SM clock (clock64, cycles; every role of block 0 runs on one SM) into pf_tl.  [4q + 0..2] for stage q < 128: producer issued
// its copies, MMA issuer saw them land, MMA issuer committed the stage; [512 + 8n + 0..5]
// for item n < 32: MMA issuer saw the item's scales placed, saw its accumulator free,
// epilogue saw the accumulator full, placed the next item's scales, finished the item,
// producer issued the item's scale copies, epilogue loaded its first 16 columns, finished
// its first 16 columns; [768 + 8n + 0..6] for item n < 32, first 16 columns: warp 0
// past the exchange barrier, SwiGLU done, quantised and stored, past the closing
// barrier; warp 2 wrote its exchange values, finished its load, started its load.  In
// the routed W2 launch [768 + 8n + 0..2] are instead: scale placement of item n began,
// ended (warp 0), warp 3 finished item n.
__device__ unsigned long long pf_tl[1024];
#define PF_STAMP(idx)                                                                         \
  do {                                                                                         \
    if (blockIdx.x == 0 && MODE == PF_TIMELINE_MODE && (idx) < 1024) pf_tl[(idx)] = (unsigned long long)clock64(); \
  } while (0)
#else
#define PF_STAMP(idx) \
  do {                \
  } while (0)
#endif

constexpr int PF_MAX_E = 512;
// routed token tiles of a chunk: sum over experts of ceil(n_e / 64) <= M k / 64 + E
constexpr int PF_MAX_TILES = 16384 * 8 / PF_BN + PF_MAX_E;
// Routed modes: tile prefix and grouped offsets are copied to shared memory once per
// CTA (every role decodes every tile; a search over global memory would put a chain
// of dependent loads in front of each tile).
__device__ inline int pf_total_items(const PrefillParams& p, int mode, const int* s_ntp) {
  if (pf_routed(mode)) return p.m_tiles * s_ntp[p.E];
  return p.m_tiles * ((p.M + PF_BN - 1) / PF_BN);
}
__device__ inline PfItem pf_item(const PrefillParams& p, int mode, int idx, const int* s_ntp, const int* s_goff,
                                 const uint16_t* s_te) {
  PfItem it;
  it.mt = idx % p.m_tiles;
  const int j = idx / p.m_tiles;
  int rows0;
  if (pf_routed(mode)) {
    const int lo = s_te[j];  // the expert whose tiles include j
    it.e = lo;
    it.n0 = (j - s_ntp[lo]) * PF_BN;
    const int g0 = s_goff[lo], ne = s_goff[lo + 1] - g0;
    it.ncnt = min(PF_BN, ne - it.n0);
    it.grow0 = g0 + it.n0;
    rows0 = lo * p.prob_rows;
  } else {
    it.e = 0;
    it.n0 = j * PF_BN;
    it.ncnt = min(PF_BN, p.M - it.n0);
    it.grow0 = it.n0;
    rows0 = 0;
  }
  if (pf_13(mode)) {
    it.ya0 = rows0 + 64 * it.mt;              // gate rows
    it.ya1 = rows0 + p.up_off + 64 * it.mt;   // up rows
  } else {
    it.ya0 = rows0 + 128 * it.mt;
    it.ya1 = it.ya0 + 64;
  }
  return it;
}

// *p[0..3] += {a, b, c, d} in one reduction (p 16-byte aligned)
__device__ __forceinline__ void red_add_f32x4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// silu(g) = g / (1 + e^-g): the fast division (2 ulp; g / inf = -0 for g < -88) keeps the
// epilogue short -- the IEEE division's special-case branches serialised it.
__device__ __forceinline__ float pf_silu(float g) { return __fdividef(g, 1.0f + expf(-g)); }

// floor(log2(a)) of a finite a > 0, exact (subnormals from the mantissa's top bit).
__device__ __forceinline__ int floor_log2_f32(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = (int)((b >> 23) & 0xFFu);
  if (e != 0) return e - 127;
  return (31 - __clz(b & 0x7FFFFFu)) - 149;
}
// MXFP8 scale exponent of a 32-block with max |v| = amax: clamp(floor(log2 amax) - 8).
__device__ __forceinline__ int mxfp8_exponent(float amax) {
  if (amax == 0.0f) return -127;
  int s = floor_log2_f32(amax) - 8;
  return s < -127 ? -127 : (s > 127 ? 127 : s);
}
__device__ __forceinline__ uint8_t e4m3_of(float v) {
  return (uint8_t)(f32x2_to_e4m3x2(v, 0.0f) & 0xFFu);
}

// ---------------------------------------------------------------------------
// k_umma
// ---------------------------------------------------------------------------
// Shared memory: the 1024-aligned stage ring (kc chunks a stage: chunk c's weight tile
// at +16384 c, its token tile at +16384 kc + 8192 c), then for the block-scaled modes one
// or two buffers of a tile's E8M0 rows (weight rows at +0, K/32 bytes each; token rows
// after them, sf_ld bytes each), filled by the producer with bulk copies and emptied
// into tensor memory by the epilogue warps.  With two, the producer fetches a tile's
// rows while the previous tile's still wait to be placed.
__host__ __device__ inline uint32_t pf_sf_buf_bytes(int K, int sf_ld) {
  const uint32_t a = (uint32_t)(128 * (K / 32) + 15) / 16 * 16;
  return a + (uint32_t)PF_BN * (uint32_t)sf_ld;  // weight rows, then at most PF_BN token rows
}

// One instantiation per mode (MODE equals p.mode): each launch carries only its own
// epilogue, so the code every role runs stays small enough for the instruction caches.
template <int MODE>
__global__ void __launch_bounds__(PF_THREADS, 1) k_umma(const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t pf_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[PF_MAX_STAGES], empty[PF_MAX_STAGES];
  __shared__ uint64_t acc_full[2], acc_empty[2], sf_full[2], sf_empty[2], sf_ready[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int s_abort;
  // 13 modes: up-half values handed from warps 2,3 to warps 0,1; routed W2: each warp's
  // 8 tokens x 32 rows, read back as four consecutive rows of one token
  __shared__ __align__(16) float xch[2][32][17];
  __shared__ int s_ntp[PF_MAX_E + 1], s_goff[PF_MAX_E + 1];
  __shared__ uint16_t s_te[pf_routed(MODE) ? PF_MAX_TILES : 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.stages;
  constexpr bool mx = pf_routed(MODE);
  const int kbox = mx ? 128 : 64;  // K elements per chunk (128 bytes per row)
  const int nch = p.K / kbox;
  const int KC = p.kc;             // chunks per stage (divides nch)
  const size_t stage_bytes = (size_t)PF_STAGE_BYTES * KC;
  if (mx)
    for (int e = tid; e <= p.E; e += PF_THREADS) {
      s_ntp[e] = __ldg(p.ntile_prefix + e);
      s_goff[e] = __ldg(p.goff + e);
    }
  __syncthreads();
  if (mx) {
    const int nt = s_ntp[p.E];  // <= PF_MAX_TILES (the host bounds M, k and E)
    for (int j = tid; j < nt; j += PF_THREADS) s_te[j] = __ldg(p.tile_e + j);
    __syncthreads();
  }
  const int total = pf_total_items(p, MODE, s_ntp);
  const int G = gridDim.x;
  const int kb = p.K / 32;  // E8M0 bytes per weight row
  const uint32_t sfa_bytes = (uint32_t)(128 * kb + 15) / 16 * 16;
  uint8_t* sfbuf = smem + (size_t)S * stage_bytes;
  const uint32_t sfbuf_bytes = pf_sf_buf_bytes(p.K, p.sf_ld);
  const int NB = p.sf_bufs > 1 ? 2 : 1;  // shared-memory scale buffers
  // Scale columns in tensor memory: two buffers when they fit beside the accumulators
  // (K <= 3072), so a tile's scales are placed while the previous tile's MMAs run;
  // otherwise one, placed once the previous tile's MMAs are done.
  const bool sf2 = PF_SF_COL + 16 * nch <= PF_TMEM_COLS;
  auto sfa_col = [&](int n) { return (uint32_t)(PF_SF_COL + (sf2 ? 8 * nch * (n & 1) : 0)); };
  auto sfb_col = [&](int n) { return sfa_col(n) + 4u * (uint32_t)nch; };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
      mbar_init(&sf_full[b], 1);
      mbar_init(&sf_empty[b], 4);
    }
    mbar_init(&sf_ready[0], 4);
    mbar_init(&sf_ready[1], 4);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 5) {
    tmem_alloc(&tmem_base_s, PF_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      long long q = 0;
      int n_item = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total && ok; idx += G, ++n_item) {
        const PfItem it = pf_item(p, MODE, idx, s_ntp, s_goff, s_te);
        if (mx) {
          // scale rows of a tile -- weight rows (two 64-row runs or one 128-row run) and
          // the token rows -- into shared buffer m % NB.  With two tensor-memory buffers the
          // next tile's rows are fetched here too, a tile ahead of its MMAs.
          auto fetch_scales = [&](int m, const PfItem& t) -> bool {
            // buffer m % NB: tile m's rows wait until tile m - NB's are in tensor memory
            const int b = m % NB;
            if (m >= NB && !pf_wait(&sf_empty[b], (uint32_t)((m / NB - 1) & 1), p.status, &s_abort, PFW_SF, MODE))
              return false;
            uint8_t* dst = sfbuf + (size_t)b * sfbuf_bytes;
            const uint32_t half = 64u * (uint32_t)kb, tok = (uint32_t)t.ncnt * (uint32_t)p.sf_ld;
            mbar_arrive_expect_tx(&sf_full[b], 2 * half + tok);
            const uint64_t pol = policy_evict_first();
            bulk_g2s(dst, p.sfa + (size_t)t.ya0 * kb, half, &sf_full[b], pol);
            bulk_g2s(dst + half, p.sfa + (size_t)t.ya1 * kb, half, &sf_full[b], pol);
            bulk_g2s(dst + sfa_bytes, p.sfb + (size_t)t.grow0 * p.sf_ld, tok, &sf_full[b], pol);
            return true;
          };
          if (!sf2 || n_item == 0) ok = fetch_scales(n_item, it);
          if (ok && sf2 && idx + G < total) ok = fetch_scales(n_item + 1, pf_item(p, MODE, idx + G, s_ntp, s_goff, s_te));
          if (!ok) break;
          if (n_item < 32) PF_STAMP(512 + 8 * n_item + 5);
        }
        for (int ch = 0; ch < nch; ch += KC, ++q) {
          const int s = (int)(q % S);
          if (q >= S && !pf_wait(&empty[s], (uint32_t)(((q / S) - 1) & 1), p.status, &s_abort, PFW_EMPTY, MODE)) {
            ok = false;
            break;
          }
          if (q < 128) PF_STAMP(4 * (int)q);
          uint8_t* st = smem + (size_t)s * stage_bytes;
          // transaction bytes count the global (packed) side: 128 rows of 128 E2M1
          // codes are 8 KB although they fill 16 KB of shared memory; the token box
          // is always whole (rows past the tensor read as zeros and still count)
          // a routed tile of at most 32 tokens takes the 32-row token box (half the bytes
          // through the copy engine); its chunks then sit 4 KB apart instead of 8 KB
          const bool half = mx && it.ncnt <= 32;
          mbar_arrive_expect_tx(&full[s], (uint32_t)KC * ((mx ? 8192u : 16384u) + (half ? 4096u : 8192u)));
          tma_load_4d(st, &p.tmA, 0, it.ya0, 0, ch, &full[s]);
          tma_load_3d(st + 16384 * KC, half ? &p.tmB32 : &p.tmB, 0, it.grow0, ch, &full[s]);
        }
      }
      // every copy issued lands before the CTA may finish
      for (long long j = (q > S ? q - S : 0); j < q; ++j)
        pf_wait(&full[j % S], (uint32_t)((j / S) & 1), p.status, &s_abort, PFW_DRAIN, MODE);
      if (mx)
        for (int j = (n_item > NB ? n_item - NB : 0); j < n_item; ++j)
          pf_wait(&sf_full[j % NB], (uint32_t)((j / NB) & 1), p.status, &s_abort, PFW_DRAIN, MODE);
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      long long q = 0;
      int n_item = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total && ok; idx += G, ++n_item) {
        const PfItem it = pf_item(p, MODE, idx, s_ntp, s_goff, s_te);
        const int N = (it.ncnt + 15) & ~15;
        const int ab = n_item & 1;
        if (n_item >= 2 && !pf_wait(&acc_empty[ab], (uint32_t)(((n_item >> 1) - 1) & 1), p.status, &s_abort,
                                    PFW_ACC_EMPTY, MODE))
          break;
        if (n_item < 32) PF_STAMP(512 + 8 * n_item + 1);
        if (mx && !pf_wait(&sf_ready[sf2 ? ab : 0], (uint32_t)((sf2 ? n_item >> 1 : n_item) & 1), p.status,
                           &s_abort, PFW_SF, MODE))
          break;
        if (n_item < 32) PF_STAMP(512 + 8 * n_item + 0);
        tc_fence_after();
        const uint32_t dacc = tbase + 64u * ab;
        const uint32_t tsfa = tbase + sfa_col(n_item), tsfb = tbase + sfb_col(n_item);
        // the tile's instruction descriptors (one per 32-wide K step of a chunk) and its
        // token-chunk stride in descriptor units, formed once per tile
        uint32_t idk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) idk[k] = mx ? idesc_mx(N, (uint32_t)k) : idesc_bf16(N);
        const uint32_t bstride = (mx && it.ncnt <= 32) ? 4096u : 8192u;  // token chunk stride (box rows x 128 B)
        for (int ch = 0; ch < nch; ch += KC, ++q) {
          const int s = (int)(q % S);
          if (!pf_wait(&full[s], (uint32_t)((q / S) & 1), p.status, &s_abort, PFW_FULL, MODE)) {
            ok = false;
            break;
          }
          if (q < 128) PF_STAMP(4 * (int)q + 1);
          // no thread-side fence here: the copies and the MMAs are both in the async
          // proxy, and the stage's barrier orders them
          // the stage's operands: base descriptors of its first weight and token chunks;
          // chunk c sits 16 KB (1024 descriptor units) and bstride further on, and each
          // 32-wide K step 32 bytes (2 units) into the swizzled rows -- the start-address
          // field (address / 16, 14 bits) never carries, shared memory being < 256 KB
          const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes);
          const uint64_t a0 = sw128_desc(sa), b0 = sw128_desc(sa + 16384u * KC);
          const uint32_t acc0 = ch > 0 ? 1u : 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // KC <= 4 chunks per stage
            if (c < KC) {
              const uint64_t ac = a0 + 1024u * (uint32_t)c, bc = b0 + (bstride >> 4) * (uint32_t)c;
              const uint32_t sfc = 4u * (uint32_t)(ch + c);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t accum = (c > 0 || k > 0) ? 1u : acc0;
                if (mx)
                  umma_mx(dacc, ac + 2u * k, bc + 2u * k, idk[k], accum, tsfa + sfc, tsfb + sfc);
                else
                  umma_bf16(dacc, ac + 2u * k, bc + 2u * k, idk[k], accum);
              }
            }
          }
          tc_commit(&empty[s]);  // the stage returns to the producer once these MMAs are done
          if (q < 128) PF_STAMP(4 * (int)q + 2);
        }
        if (!ok) break;
        tc_commit(&acc_full[ab]);  // accumulator ab is complete (and so are this tile's reads of the scales)
      }
    }
  } else {
    // ---------------- epilogue warps 0-3 ----------------
    const int r = lane;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * warp) << 16);
    // E8M0 words of a tile from its scale buffer into tensor memory (lane r of every
    // quarter, column base + 4ch + c: operand row r + 32c, K blocks 4ch..4ch+3)
    auto put_scales = [&](int n_item, const PfItem& it) -> bool {
      if (MODE == PF_R2 && tid == 0 && n_item < 32) PF_STAMP(768 + 8 * n_item + 0);
      const int b = n_item & 1;      // tensor-memory scale buffer (with two of them)
      const int sb_i = n_item % NB;  // shared-memory scale buffer
      if (!pf_wait(&sf_full[sb_i], (uint32_t)((n_item / NB) & 1), p.status, &s_abort, PFW_SF, MODE)) return false;
      const uint8_t* sa = sfbuf + (size_t)sb_i * sfbuf_bytes;
      const uint8_t* sb = sa + sfa_bytes;
      for (int ch = 0; ch < nch; ++ch) {
        uint32_t wa[4], wb[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int m = r + 32 * c;
          wa[c] = *reinterpret_cast<const uint32_t*>(sa + m * kb + 4 * ch);
          wb[c] = m < it.ncnt ? *reinterpret_cast<const uint32_t*>(sb + m * p.sf_ld + 4 * ch) : 0x7F7F7F7Fu;
        }
        tmem_st4(lane_base + sfa_col(n_item) + 4 * ch, wa[0], wa[1], wa[2], wa[3]);
        tmem_st4(lane_base + sfb_col(n_item) + 4 * ch, wb[0], wb[1], wb[2], wb[3]);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sf_ready[sf2 ? b : 0]);
        mbar_arrive(&sf_empty[sb_i]);
      }
      if (MODE == PF_R2 && tid == 0 && n_item < 32) PF_STAMP(768 + 8 * n_item + 1);
      return true;
    };
    bool live = true;
    if (mx && blockIdx.x < total) live = put_scales(0, pf_item(p, MODE, blockIdx.x, s_ntp, s_goff, s_te));
    if (mx && sf2 && live && blockIdx.x + G < total) live = put_scales(1, pf_item(p, MODE, blockIdx.x + G, s_ntp, s_goff, s_te));
    int n_item = 0;
    for (int idx = blockIdx.x; idx < total; idx += G, ++n_item) {
      const PfItem it = pf_item(p, MODE, idx, s_ntp, s_goff, s_te);
      const int ab = n_item & 1;
      // routed W2: the tile's tokens and routing weights (lane j holds grouped rows j and
      // j + 32), fetched before the accumulator wait so their latency stays off the epilogue
      int tk_lo = 0, tk_hi = 0;
      float tw_lo = 0.0f, tw_hi = 0.0f;
      if (MODE == PF_R2) {
        if (r < it.ncnt) {
          tk_lo = __ldg(p.g_tok + it.grow0 + r);
          tw_lo = __ldg(p.g_w + it.grow0 + r);
        }
        if (r + 32 < it.ncnt) {
          tk_hi = __ldg(p.g_tok + it.grow0 + r + 32);
          tw_hi = __ldg(p.g_w + it.grow0 + r + 32);
        }
      }
      if (live) pf_wait(&acc_full[ab], (uint32_t)((n_item >> 1) & 1), p.status, &s_abort, PFW_ACC_FULL, MODE);
      if (tid == 0 && n_item < 32) PF_STAMP(512 + 8 * n_item + 2);
      named_barrier(2, 128);  // the four epilogue warps take the same decision below
      if (s_abort) break;
      tc_fence_after();
      // one scale buffer: the MMAs of this tile are complete, its columns may take the next tile's
      if (mx && !sf2 && idx + G < total) live = put_scales(n_item + 1, pf_item(p, MODE, idx + G, s_ntp, s_goff, s_te));
      if (tid == 0 && n_item < 32) PF_STAMP(512 + 8 * n_item + 3);
      const uint32_t acc_lane = lane_base + 64u * ab;
      for (int j0 = 0; j0 < it.ncnt; j0 += 16) {
        float v[16];
        if (tid == 64 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 6);
        tmem_ld16(acc_lane + (uint32_t)j0, v);
        if (tid == 0 && n_item < 32 && j0 == 0) PF_STAMP(512 + 8 * n_item + 6);
        if (tid == 64 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 5);
        const int jn = min(16, it.ncnt - j0);
        if (MODE == PF_ROUTER || MODE == PF_SH2) {
          const int row = 128 * it.mt + 32 * warp + r;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < jn) p.out_f32[(size_t)(it.n0 + j0 + j) * p.out_ld + row] = v[j];
        } else if (MODE == PF_R2) {
          // y[token][rows r0..r0+3] += w * four values with one 16-byte reduction: per 8
          // tokens the warp's 32 x 8 block goes through shared memory, and lane r (quad
          // index qd = r % 4) takes tokens 2 qd and 2 qd + 1 of the four rows r0 = r - qd
          float* buf = &xch[0][0][0] + 256 * warp;  // [8 tokens][32 rows]
          const int qd = r & 3;
          const int row0 = 128 * it.mt + 32 * warp + (r & ~3);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) buf[32 * jj + r] = v[8 * h + jj];
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int jj = 8 * h + 2 * qd + u;  // token of the chunk
              const int src = (j0 & 31) + jj;
              const int tok = __shfl_sync(0xffffffffu, j0 < 32 ? tk_lo : tk_hi, src);
              const float wt = __shfl_sync(0xffffffffu, j0 < 32 ? tw_lo : tw_hi, src);
              const float4 a = *reinterpret_cast<const float4*>(buf + 32 * (2 * qd + u) + (r & ~3));
              if (jj < jn) red_add_f32x4(p.out_f32 + (size_t)tok * p.out_ld + row0, wt * a.x, wt * a.y, wt * a.z, wt * a.w);
            }
            __syncwarp();  // buf is rewritten by the next 8 tokens
          }
        } else {
          // 13 modes: warps 0,1 hold gate rows, warps 2,3 the matching up rows.  Each
          // pair (w, w+2) splits the 16 tokens: the gate warp finishes tokens 0-7 and
          // the up warp tokens 8-15, after handing each other the missing half.
          const int pr = warp & 1;
          const bool gate = warp < 2;
#pragma unroll
          for (int j = 0; j < 8; ++j) xch[pr][r][(gate ? 0 : 8) + j] = gate ? v[8 + j] : v[j];
          if (tid == 64 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 4);
          named_barrier(2, 128);
          if (tid == 0 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 0);
          const int i = 64 * it.mt + 32 * pr + r;  // intermediate index
          const int jb = gate ? 0 : 8;             // this warp's first token of the chunk
          float a[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            a[j] = gate ? pf_silu(v[j]) * xch[pr][r][8 + j] : pf_silu(xch[pr][r][j]) * v[8 + j];
          if (tid == 0 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 1);
          if (MODE == PF_SH13) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (jb + j < jn) p.out_bf16[(size_t)(it.n0 + j0 + jb + j) * p.out_ld + i] = __float2bfloat16_rn(a[j]);
          } else {
            // MXFP8 of each token's 32-block (this warp's 32 rows): the block maximum
            // of |a| is one warp max over the bit patterns (monotonic for x >= 0)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float am = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(a[j]))));
              const int s = mxfp8_exponent(am);
              if (jb + j < jn) {
                const size_t g = (size_t)(it.grow0 + j0 + jb + j);
                p.out_q[g * p.out_ld + i] = am == 0.0f ? (uint8_t)0 : e4m3_of(a[j] * exp2i(-s));
                if (r == 0) p.out_qs[g * p.out_qs_ld + (64 * it.mt + 32 * pr) / 32] = (uint8_t)(s + 127);
              }
            }
            if (tid == 0 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 2);
          }
          named_barrier(2, 128);  // xch is rewritten by the next chunk
          if (tid == 0 && n_item < 32 && j0 == 0) PF_STAMP(768 + 8 * n_item + 3);
        }
        if (tid == 0 && n_item < 32 && j0 == 0) PF_STAMP(512 + 8 * n_item + 7);
      }
      if (tid == 0 && n_item < 32) PF_STAMP(512 + 8 * n_item + 4);
      if (MODE == PF_R2 && tid == 96 && n_item < 32) PF_STAMP(768 + 8 * n_item + 2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      // two scale buffers: this tile's MMAs are done, so its buffer takes the tile after
      // next while the next tile's MMAs run
      if (mx && sf2 && live && idx + 2 * G < total)
        live = put_scales(n_item + 2, pf_item(p, MODE, idx + 2 * G, s_ntp, s_goff, s_te));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, PF_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// routing and grouping for the chunk
// ---------------------------------------------------------------------------
// One warp per token: top-k of logits [M][E] (largest, lowest index on ties), softmax
// over the selected, per-expert counts.
__global__ void __launch_bounds__(256) k_pf_topk(const float* __restrict__ logits, int M, int E, int k,
                                                  int32_t* __restrict__ ids, float* __restrict__ w,
                                                  int* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= M) return;
  const float* lr = logits + (size_t)t * E;
  uint32_t key[16];  // E <= 512
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? float_key(lr[e]) : 0u;
  }
  float sel_l = 0.0f;
  int sel_i = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (key[i] > bk) {
        bk = key[i];
        bi = lane + 32 * i;
      }
    const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
    const int mi = (int)__reduce_min_sync(0xffffffffu, (unsigned)(bk == mk ? bi : 0x7fffffff));
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (lane + 32 * i == mi) key[i] = 0u;
    if (lane == j) {
      sel_l = key_float(mk);
      sel_i = mi;
    }
  }
  const float l0 = __shfl_sync(0xffffffffu, sel_l, 0);
  const float ex = lane < k ? expf(sel_l - l0) : 0.0f;
  float den = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    ids[(size_t)t * k + lane] = sel_i;
    w[(size_t)t * k + lane] = ex / den;
    atomicAdd(counts + sel_i, 1);
  }
}

// One block: exclusive prefix of the counts (grouped offsets) and of the 128-token
// tiles per expert; clears the fill cursors.
__global__ void __launch_bounds__(1024) k_pf_scan(const int* __restrict__ counts, int E, int* __restrict__ goff,
                                                   int* __restrict__ ntile_prefix, int* __restrict__ fill,
                                                   uint16_t* __restrict__ tile_e) {
  __shared__ int s_c[1024], s_t[1024];
  const int e = threadIdx.x;
  const int c = e < E ? counts[e] : 0;
  s_c[e] = c;
  s_t[e] = (c + PF_BN - 1) / PF_BN;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int a = e >= o ? s_c[e - o] : 0, b = e >= o ? s_t[e - o] : 0;
    __syncthreads();
    s_c[e] += a;
    s_t[e] += b;
    __syncthreads();
  }
  if (e < E) {
    goff[e + 1] = s_c[e];
    ntile_prefix[e + 1] = s_t[e];
    fill[e] = 0;
    const int nt = (c + PF_BN - 1) / PF_BN;  // this expert's tiles end at s_t[e]
    for (int j = s_t[e] - nt; j < s_t[e]; ++j) tile_e[j] = (uint16_t)e;
  }
  if (e == 0) {
    goff[0] = 0;
    ntile_prefix[0] = 0;
  }
}

// Per-expert counts of a routing given by the caller (ids outside [0, E) count for
// nothing, as in the decode path).
__global__ void k_pf_count(const int32_t* __restrict__ ids, int n, int E, int* __restrict__ counts) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int e = ids[i];
  if (e >= 0 && e < E) atomicAdd(counts + e, 1);
}

// Grouped rows: each (token, selection) gets a slot in its expert's range (pos -1 for an
// id outside [0, E)).
__global__ void k_pf_scatter(const int32_t* __restrict__ ids, const float* __restrict__ w, int M, int k, int E,
                             const int* __restrict__ goff, int* __restrict__ fill, int32_t* __restrict__ g_tok,
                             float* __restrict__ g_w, int32_t* __restrict__ pos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * k) return;
  const int e = ids[i];
  if (e < 0 || e >= E) {
    pos[i] = -1;
    return;
  }
  const int g = goff[e] + atomicAdd(fill + e, 1);
  g_tok[g] = i / k;
  g_w[g] = w[i];
  pos[i] = g;
}

// MXFP8 of the chunk's input, written to every grouped row of its token: one thread per
// (token, 32-block) -- the block's 64 bytes in four 16-byte loads, its maximum formed
// locally, its 32 codes out as two 16-byte stores per grouped row.
__global__ void __launch_bounds__(256) k_pf_quant_x(const __nv_bfloat16* __restrict__ x, int M, int H, int k,
                                                     const int32_t* __restrict__ pos, uint8_t* __restrict__ xq,
                                                     uint8_t* __restrict__ xs, int xs_ld) {
  const int nb = H / 32;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)M * nb) return;
  const int t = (int)(i / nb), b = (int)(i % nb);
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H + 32 * b);
  uint32_t w[16];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 r = __ldg(src + c);
    w[4 * c] = r.x;
    w[4 * c + 1] = r.y;
    w[4 * c + 2] = r.z;
    w[4 * c + 3] = r.w;
  }
  float v[32];  // bf16 -> fp32 is exact: the bits moved up by 16
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    v[2 * e] = __uint_as_float(w[e] << 16);
    v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
  float am = 0.0f;
#pragma unroll
  for (int e = 0; e < 32; ++e) am = fmaxf(am, fabsf(v[e]));
  const int s = mxfp8_exponent(am);
  uint32_t o[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (am != 0.0f) {
    const float sc = exp2i(-s);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      o[q] = f32x2_to_e4m3x2(v[4 * q] * sc, v[4 * q + 1] * sc) |
             (f32x2_to_e4m3x2(v[4 * q + 2] * sc, v[4 * q + 3] * sc) << 16);
  }
  for (int j = 0; j < k; ++j) {
    const int gi = __ldg(pos + (size_t)t * k + j);
    if (gi < 0) continue;
    uint4* dst = reinterpret_cast<uint4*>(xq + (size_t)gi * H + 32 * b);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    xs[(size_t)gi * xs_ld + b] = (uint8_t)(s + 127);
  }
}

// Stand-alone MXFP8 quantiser of an fp32 matrix [M][K] (codes [M][K], E8M0 [M][K/32]).
__global__ void __launch_bounds__(256) k_mxfp8_quantize(const float* __restrict__ v, int M, int K,
                                                         uint8_t* __restrict__ q, uint8_t* __restrict__ se) {
  const int lane = threadIdx.x & 31;
  const long long wi = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int nb = K / 32;
  if (wi >= (long long)M * nb) return;
  const int t = (int)(wi / nb), b = (int)(wi % nb);
  const float x = v[(size_t)t * K + 32 * b + lane];
  float am = fabsf(x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int s = mxfp8_exponent(am);
  q[(size_t)t * K + 32 * b + lane] = am == 0.0f ? (uint8_t)0 : e4m3_of(x * exp2i(-s));
  if (lane == 0) se[(size_t)t * nb + b] = (uint8_t)(s + 127);
}

}  // namespace moe
