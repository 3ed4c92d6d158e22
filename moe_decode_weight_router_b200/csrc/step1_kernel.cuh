// step1_kernel.cuh -- the decode step for one token (M = 1): every MoE layer in one
// persistent launch (one block per SM), each block streaming a contiguous share of
// every weight matrix of the layer with a few large bulk copies.
//
// Why the shares are contiguous: the SM's copy engine spends a fixed ~0.25-0.4 us on
// every bulk copy whatever its size, so a layer's 267 KB per SM must travel in a
// handful of copies (about 7 to 10 per block and layer here), not tile by tile.
//
// Per layer, block c owns
//   router rows        [E c/G, E (c+1)/G)           bf16, one copy
//   shared units       [Is c/G, Is (c+1)/G)         gate rows + up rows, two copies
//   shared W2 rows     [H c/G, H (c+1)/G)           one copy
//   routed units       [U c/G, U (c+1)/G)           U = distinct experts x I; per expert
//                                                   segment (at most 2) gate codes, up
//                                                   codes, gate scales, up scales
//   routed W2 rows     [D c/G, D (c+1)/G)           D = distinct experts x H; per
//                                                   segment codes + scales
// Shared memory: region X holds the layer's router + shared-W13 rows, and once those
// are consumed the routed-W2 rows and the shared-W2 rows; region Y the routed-W13
// rows.  One producer warp issues, per layer l: shared W2 (l) as soon as the router and
// shared-W13 rows of l are consumed; routed W13 and W2 (l) once the routing plan is
// built; router + shared W13 (l+1) as soon as routed and shared W2 (l) are consumed,
// so they land while the residual of layer l is exchanged and normalised.
//
// Sources: DGX Spark MoE knowledge card (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
// 三种方法), 事件概述或研究问题 (batch-1 decode bound by weight reads; 8 of 512 experts
// + 1 shared) and 方法/产品要点 item 1 (MXFP4 routed experts).
#pragma once

#include "step_kernel.cuh"

namespace moe {

// Region layout of the one-token kernel (bytes; host and device compute the same).
struct Step1Sizes {
  int nr, ns, no, nu, nw;  // per-block maxima: router rows, shared units, shared-W2 rows,
                           // routed units, routed W2 rows
  uint32_t a_bytes;        // router + shared-W13 rows at X
  uint32_t cr_bytes;       // routed W2 codes + scale supersets at X
  uint32_t cs_off;         // shared W2 rows at X + cs_off
  uint32_t cs_bytes;
  uint32_t x_bytes;
  uint32_t y_bytes;        // routed W13 codes + scale supersets
};
__host__ __device__ inline uint32_t up128(uint32_t b) { return (b + 127u) / 128u * 128u; }
__host__ __device__ inline Step1Sizes step1_sizes(int H, int I, int Is, int E, int k, int G) {
  Step1Sizes z;
  z.nr = (E + G - 1) / G;
  z.ns = (Is + G - 1) / G;
  z.no = Is > 0 ? (H + G - 1) / G : 0;
  z.nu = (k * I + G - 1) / G;
  z.nw = (k * H + G - 1) / G;
  z.a_bytes = up128((uint32_t)(z.nr + 2 * z.ns) * 2u * (uint32_t)H);
  // two segments at most; each scale run widened to 16-byte boundaries (+32 bytes)
  z.cr_bytes = up128((uint32_t)z.nw * (uint32_t)(I / 2) + 16u + (uint32_t)z.nw * (uint32_t)(I / 32) + 2u * 32u);
  z.cs_off = z.cr_bytes;
  z.cs_bytes = up128((uint32_t)z.no * 2u * (uint32_t)Is);
  z.x_bytes = z.a_bytes > z.cs_off + z.cs_bytes ? z.a_bytes : z.cs_off + z.cs_bytes;
  z.y_bytes = up128((uint32_t)z.nu * (uint32_t)H + 16u + (uint32_t)z.nu * (uint32_t)(H / 16) + 4u * 32u);
  return z;
}

// Block c's share [a, a + n) of `total` items.
__device__ __forceinline__ void block_share(int total, int& a, int& n) {
  const int c = blockIdx.x, G = gridDim.x;
  a = (int)((long long)total * c / G);
  n = (int)((long long)total * (c + 1) / G) - a;
}

// A range of a (expert slot, index) space split at expert boundaries: at most two
// segments when the range is no longer than one expert.
struct Segs {
  int n;
  int u[2], j0[2], len[2];
};
__device__ __forceinline__ Segs split_segments(int a, int n, int per) {
  Segs s;
  s.n = 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int u = a / per, j = a - u * per;
    const int m = min(n, per - j);
    s.u[t] = u;
    s.j0[t] = j;
    s.len[t] = n > 0 ? m : 0;
    if (n > 0) s.n = t + 1;
    a += m;
    n -= m;
  }
  return s;
}

// A run of scale rows copied as its 16-byte-aligned superset: the copy starts at the
// run's address rounded down and its length is rounded up (every scale tensor is a
// multiple of 16 bytes from a 16-byte-aligned base, so the superset stays inside it).
struct ScaleRun {
  const uint8_t* src;  // aligned start
  uint32_t off;        // offset of the first wanted byte in the copy
  uint32_t len;        // bytes copied (multiple of 16)
};
__device__ __forceinline__ ScaleRun scale_run(const uint8_t* first, uint32_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(first);
  const uintptr_t s = a & ~(uintptr_t)15;
  ScaleRun r;
  r.src = reinterpret_cast<const uint8_t*>(s);
  r.off = (uint32_t)(a - s);
  r.len = bytes ? (r.off + bytes + 15u) & ~15u : 0u;
  return r;
}

// Where the routed W13 rows of a layer sit in region Y: per segment the gate code rows,
// the up code rows, then all scale supersets (gate, up per segment).
struct BLayout {
  Segs sg;
  const uint8_t* gate[2];
  const uint8_t* up[2];
  const uint8_t* gsc[2];
  const uint8_t* usc[2];
  ScaleRun rg[2], ru[2];
  uint32_t dst_codes[2], dst_rg[2], dst_ru[2];  // byte offsets in Y of each copy
  uint32_t total;                               // bytes landing in Y
};
__device__ __forceinline__ BLayout b_layout(const StepParams& p, const LayerPtrs& Lp, const Plan& P, int a, int n,
                                            const uint8_t* Y) {
  const int H = p.H, I = p.I;
  BLayout b;
  b.sg = split_segments(a, n, I);
  uint32_t off = 0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const size_t row = (size_t)P.ids[k < b.sg.n ? b.sg.u[k] : 0] * 2 * I + b.sg.j0[k];
    b.gate[k] = Lp.w13c + row * (H / 2);
    b.up[k] = Lp.w13c + (row + I) * (H / 2);
    b.dst_codes[k] = off;
    off += 2u * (uint32_t)b.sg.len[k] * (uint32_t)(H / 2);
    b.rg[k] = scale_run(Lp.w13s + row * (H / 32), (uint32_t)b.sg.len[k] * (uint32_t)(H / 32));
    b.ru[k] = scale_run(Lp.w13s + (row + I) * (H / 32), (uint32_t)b.sg.len[k] * (uint32_t)(H / 32));
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    b.dst_rg[k] = off;
    off += b.rg[k].len;
    b.dst_ru[k] = off;
    off += b.ru[k].len;
  }
  b.total = off;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    b.gsc[k] = Y + b.dst_rg[k] + b.rg[k].off;
    b.usc[k] = Y + b.dst_ru[k] + b.ru[k].off;
  }
  return b;
}
// Where the routed W2 rows sit in region X: per segment the code rows, then the scale
// supersets.
struct CLayout {
  Segs sg;
  const uint8_t* codes[2];
  ScaleRun rs[2];
  uint32_t dst_codes[2], dst_sc[2];
  uint32_t total;
};
__device__ __forceinline__ CLayout c_layout(const StepParams& p, const LayerPtrs& Lp, const Plan& P, int a, int n) {
  const int H = p.H, I = p.I;
  CLayout c;
  c.sg = split_segments(a, n, H);
  uint32_t off = 0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const size_t row = (size_t)P.ids[k < c.sg.n ? c.sg.u[k] : 0] * H + c.sg.j0[k];
    c.codes[k] = Lp.w2c + row * (I / 2);
    c.dst_codes[k] = off;
    off += (uint32_t)c.sg.len[k] * (uint32_t)(I / 2);
    c.rs[k] = scale_run(Lp.w2s + row * (I / 32), (uint32_t)c.sg.len[k] * (uint32_t)(I / 32));
  }
  off = (off + 15u) & ~15u;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    c.dst_sc[k] = off;
    off += c.rs[k].len;
  }
  c.total = off;
  return c;
}

// One token: bf16 rows (stride 2K bytes) against the bf16 activation xb (row-major),
// lanes along K: lane L takes 16-byte chunks L, L+32, ...  R rows share the activation
// loads; every lane returns the R row sums (exact bf16 products, fp32 sums).
template <int R>
__device__ __forceinline__ void bf16_rows_dot(const uint8_t* const (&rows)[R], const uint8_t* xb, int K,
                                              float (&out)[R]) {
  const int lane = threadIdx.x & 31;
  float a[R][2];
#pragma unroll
  for (int q = 0; q < R; ++q) a[q][0] = a[q][1] = 0.0f;
#pragma unroll 1
  for (int c = lane; c < K / 8; c += 32) {
    const uint4 X = lds128(xb + 16 * c);
    const uint32_t xw[4] = {X.x, X.y, X.z, X.w};
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const uint4 W = lds128(rows[q] + 16 * c);
      const uint32_t ww[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a[q][0] = fma_bf16_lo(ww[j], xw[j], a[q][0]);
        a[q][1] = fma_bf16_hi(ww[j], xw[j], a[q][1]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < R; ++q) {
    float v = a[q][0] + a[q][1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    out[q] = v;
  }
}
// One bf16 row of K against an fp32 activation held as bf16 hi + lo rows.
__device__ __forceinline__ float bf16_row_dot_hilo(const uint8_t* row, const uint8_t* xhi, const uint8_t* xlo, int K) {
  const int lane = threadIdx.x & 31;
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll 1
  for (int c = lane; c < K / 8; c += 32) {
    const uint4 W = lds128(row + 16 * c);
    const uint4 X = lds128(xhi + 16 * c);
    const uint4 Y = lds128(xlo + 16 * c);
    const uint32_t ww[4] = {W.x, W.y, W.z, W.w}, xw[4] = {X.x, X.y, X.z, X.w}, yw[4] = {Y.x, Y.y, Y.z, Y.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a0 = fma_bf16_lo(ww[j], xw[j], a0);
      a1 = fma_bf16_hi(ww[j], xw[j], a1);
      a0 = fma_bf16_lo(ww[j], yw[j], a0);
      a1 = fma_bf16_hi(ww[j], yw[j], a1);
    }
  }
  float v = a0 + a1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The products the one-token kernel calls in its loops.
__device__ __forceinline__ void unit_dot(const uint8_t* gate, const uint8_t* up, const uint8_t* gsc, const uint8_t* usc,
                                      int nb, const uint8_t* xc, int sh, float& g, float& u) {
  const uint8_t* const rows[2] = {gate, up};
  const uint8_t* const scs[2] = {gsc, usc};
  float r[2];
  rows_dot_m1_exact<16, 2>(rows, scs, nb, xc, sh, r);
  g = r[0];
  u = r[1];
}
__device__ __forceinline__ void w2_pair_dot(const uint8_t* ra, const uint8_t* rb, const uint8_t* sa, const uint8_t* sb,
                                         int nb, const uint8_t* xc, int sh, float& va, float& vb) {
  const uint8_t* const rows[2] = {ra, rb};
  const uint8_t* const scs[2] = {sa, sb};
  float r[2];
  rows_dot_m1_exact<8, 2>(rows, scs, nb, xc, sh, r);
  va = r[0];
  vb = r[1];
}
__device__ __forceinline__ float w2_row_dot(const uint8_t* ra, const uint8_t* sa, int nb, const uint8_t* xc, int sh) {
  const uint8_t* const rows[1] = {ra};
  const uint8_t* const scs[1] = {sa};
  float r[1];
  rows_dot_m1_exact<8, 1>(rows, scs, nb, xc, sh, r);
  return r[0];
}
__device__ __forceinline__ void bf16_dot1(const uint8_t* row, const uint8_t* xb, int K, float& v) {
  const uint8_t* const rows[1] = {row};
  float r[1];
  bf16_rows_dot<1>(rows, xb, K, r);
  v = r[0];
}
__device__ __forceinline__ void bf16_dot2(const uint8_t* ra, const uint8_t* rb, const uint8_t* xb, int K, float& va,
                                       float& vb) {
  const uint8_t* const rows[2] = {ra, rb};
  float r[2];
  bf16_rows_dot<2>(rows, xb, K, r);
  va = r[0];
  vb = r[1];
}

__global__ void __launch_bounds__(STEP_THREADS, 1) k_step1(const __grid_constant__ StepParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Plan P;
  __shared__ float s_part[MAX_M * STEP_CONSUMERS];
  __shared__ float s_r[MAX_M];
  __shared__ int s_ash[2];  // f16 shift of each staged routed activation
  __shared__ int32_t s_ids[MAX_SLOTS];
  __shared__ float s_wts[MAX_SLOTS];
  __shared__ float s_amx[MAX_M * STEP_CONSUMERS];
  __shared__ int s_sh[MAX_M];
  __shared__ uint32_t s_wmax[MAX_M * STEP_CONSUMERS];
  __shared__ int s_ncand[MAX_M];
  __shared__ unsigned long long s_cand[MAX_M * TOPK_CAND];
  __shared__ unsigned long long s_sel[MAX_M * 8];
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I, Is = p.Is, L = p.L, E = p.E;
  const unsigned G = gridDim.x;
  const Step1Sizes Z = step1_sizes(H, I, Is, E, p.k, (int)G);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint64_t* fullA = bars + 0;   // router + shared W13 rows landed (X)
  uint64_t* emptyA = bars + 1;  // ... consumed (8 consumer warps)
  uint64_t* fullS = bars + 2;   // shared W2 rows landed (X + cs_off)
  uint64_t* fullB = bars + 3;   // routed W13 rows landed (Y)
  uint64_t* emptyB = bars + 4;  // ... consumed
  uint64_t* fullC = bars + 5;   // routed W2 rows landed (X)
  uint64_t* emptyX = bars + 6;  // routed and shared W2 rows consumed: X free for the next layer
  uint64_t* plan_bar = bars + 7;
  uint64_t* hinit_bar = bars + 8;
  uint64_t* fullB1 = bars + 9;  // second halves of the routed W13 code rows landed (Y)
  uint8_t* X = smem + STEP_FIXED;
  uint8_t* Y = X + Z.x_bytes;
  uint8_t* act = Y + Z.y_bytes;
  const uint32_t xss = padded_stride(2u * H);
  const uint32_t ass = padded_stride(2u * I);
  uint8_t* xb16 = act;        // bf16 x row
  uint8_t* xf16 = act + xss;  // f16 x row, chunk-major
  uint8_t* shi = act;         // shared-W2 phase: a_shared as bf16 hi, lo (x is dead by then)
  uint8_t* slo = act + padded_stride(2u * Is);
  uint8_t* afc = act;         // routed-W2 phase: f16 routed a of the range's experts [2][ass]

  int r0, nr, s0, ns, o0, no;  // this block's router rows, shared units, shared-W2 rows
  block_share(E, r0, nr);
  block_share(Is, s0, ns);
  if (Is > 0)
    block_share(H, o0, no);
  else
    o0 = no = 0;

  if (tid == 0) {
    mbar_init(fullA, 1);
    mbar_init(emptyA, STEP_CONSUMERS);
    mbar_init(fullS, 1);
    mbar_init(fullB, 1);
    mbar_init(fullB1, 1);
    mbar_init(emptyB, STEP_CONSUMERS);
    mbar_init(fullC, 1);
    mbar_init(emptyX, STEP_CONSUMERS);
    mbar_init(plan_bar, 1);
    mbar_init(hinit_bar, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  // ---------------- producer ----------------
  if (warp == STEP_CONSUMERS) {
    if (lane != 0) return;  // one thread issues every copy of the block
    const uint64_t pol = policy_evict_first();
    int issued[6] = {0, 0, 0, 0, 0, 0};  // phases armed per full barrier: A, S, B, C (for the drain)
    auto issue_a = [&](const LayerPtrs& Lp) {
      const uint32_t ra = (uint32_t)nr * 2u * H, sa = (uint32_t)ns * 2u * H;
      mbar_arrive_expect_tx(fullA, ra + 2u * sa);
      if (ra) bulk_g2s(X, Lp.wr + (size_t)r0 * H, ra, fullA, pol);
      if (sa) {
        bulk_g2s(X + (size_t)Z.nr * 2 * H, Lp.sw13 + (size_t)s0 * H, sa, fullA, pol);
        bulk_g2s(X + (size_t)(Z.nr + Z.ns) * 2 * H, Lp.sw13 + (size_t)(Is + s0) * H, sa, fullA, pol);
      }
      ++issued[0];
    };
    bool ok = true;
    if (L > 0) issue_a(p.layer[0]);
    for (int l = 0; l < L && ok; ++l) {
      const LayerPtrs& Lp = p.layer[l];
      const uint32_t par = (uint32_t)(l & 1);
      // shared W2 rows once the router and shared-W13 rows of this layer are consumed
      if (!(ok = ring_wait(emptyA, par, p.status, &s_abort))) break;
      {
        const uint32_t b = (uint32_t)no * 2u * Is;
        mbar_arrive_expect_tx(fullS, b);
        if (b) bulk_g2s(X + Z.cs_off, Lp.sw2 + (size_t)o0 * Is, b, fullS, pol);
        ++issued[1];
      }
      stamp(p, l, 12);
      // the consumers' slice copy of h (ordered before their arrive by a block
      // barrier) is published here, off their critical path: fence, then count
      if (!(ok = ring_wait(hinit_bar, par, p.status, &s_abort))) break;
      signal_counter(p.ctr + (size_t)l * CTR_PER_LAYER + CTR_HINIT);
      if (!(ok = ring_wait(plan_bar, par, p.status, &s_abort))) break;
      stamp(p, l, 13);
      // routed W13 into Y (free: the previous layer's were consumed before its plan)
      if (l > 0 && !(ok = ring_wait(emptyB, (uint32_t)((l - 1) & 1), p.status, &s_abort))) break;
      int a, n;
      block_share(P.n_unique * I, a, n);
      const BLayout B = b_layout(p, Lp, P, a, n, Y);
      {
        // scales and the first half of every segment's code rows complete fullB, the
        // second halves fullB1, so the first units compute while the rest lands
        uint32_t b0 = 0, b1 = 0;
        for (int k = 0; k < B.sg.n; ++k) {
          const uint32_t h = (uint32_t)((B.sg.len[k] + 1) / 2) * (uint32_t)(H / 2);
          const uint32_t cb = (uint32_t)B.sg.len[k] * (uint32_t)(H / 2);
          b0 += 2u * h + B.rg[k].len + B.ru[k].len;
          b1 += 2u * (cb - h);
        }
        mbar_arrive_expect_tx(fullB, b0);
        mbar_arrive_expect_tx(fullB1, b1);
        for (int k = 0; k < B.sg.n; ++k) {
          bulk_g2s(Y + B.dst_rg[k], B.rg[k].src, B.rg[k].len, fullB, pol);
          bulk_g2s(Y + B.dst_ru[k], B.ru[k].src, B.ru[k].len, fullB, pol);
        }
        for (int k = 0; k < B.sg.n; ++k) {
          const uint32_t h = (uint32_t)((B.sg.len[k] + 1) / 2) * (uint32_t)(H / 2);
          const uint32_t cb = (uint32_t)B.sg.len[k] * (uint32_t)(H / 2);
          bulk_g2s(Y + B.dst_codes[k], B.gate[k], h, fullB, pol);
          bulk_g2s(Y + B.dst_codes[k] + cb, B.up[k], h, fullB, pol);
        }
        for (int k = 0; k < B.sg.n; ++k) {
          const uint32_t h = (uint32_t)((B.sg.len[k] + 1) / 2) * (uint32_t)(H / 2);
          const uint32_t cb = (uint32_t)B.sg.len[k] * (uint32_t)(H / 2);
          if (cb > h) {
            bulk_g2s(Y + B.dst_codes[k] + h, B.gate[k] + h, cb - h, fullB1, pol);
            bulk_g2s(Y + B.dst_codes[k] + cb + h, B.up[k] + h, cb - h, fullB1, pol);
          }
        }
      }
      ++issued[2];
      // routed W2 into X (the router and shared-W13 rows there are consumed)
      block_share(P.n_unique * H, a, n);
      const CLayout C = c_layout(p, Lp, P, a, n);
      mbar_arrive_expect_tx(fullC, C.total);
      for (int k = 0; k < C.sg.n; ++k) {
        bulk_g2s(X + C.dst_codes[k], C.codes[k], (uint32_t)C.sg.len[k] * (uint32_t)(I / 2), fullC, pol);
        bulk_g2s(X + C.dst_sc[k], C.rs[k].src, C.rs[k].len, fullC, pol);
      }
      ++issued[3];
      stamp(p, l, 14);
      // the next layer's router and shared-W13 rows once X is free again
      if (l + 1 < L) {
        if (!(ok = ring_wait(emptyX, par, p.status, &s_abort))) break;
        issue_a(p.layer[l + 1]);
        stamp(p, l, 15);
      }
    }
    // every copy issued lands before the block may exit
    if (issued[0]) drain_wait(fullA, (uint32_t)((issued[0] - 1) & 1));
    if (issued[1]) drain_wait(fullS, (uint32_t)((issued[1] - 1) & 1));
    if (issued[2]) {
      drain_wait(fullB, (uint32_t)((issued[2] - 1) & 1));
      drain_wait(fullB1, (uint32_t)((issued[2] - 1) & 1));
    }
    if (issued[3]) drain_wait(fullC, (uint32_t)((issued[3] - 1) & 1));
    return;
  }
  if (warp > STEP_CONSUMERS) return;

  // ---------------- consumers ----------------
  unsigned* ctr = p.ctr;
  int slice_q0, slice_n;
  block_share(H / 4, slice_q0, slice_n);
  const int nr_w = nr;  // router rows on warps 0.., shared units after them
  for (int l = 0; l < L; ++l) {
    unsigned* lc = ctr + (size_t)l * CTR_PER_LAYER;
    const uint32_t par = (uint32_t)(l & 1);
    float* hout = p.h + (size_t)(l & 1) * H;
    const float* hin = p.h + (size_t)((l + 1) & 1) * H;  // layer l-1's buffer
    stamp(p, l, 0);
    if (l > 0) {
      if (tid == 0) wait_counter(ctr + (size_t)(l - 1) * CTR_PER_LAYER + CTR_H, G, p.status, &s_abort);
      csync();
    }
    stamp(p, l, 1);
    if (tid == 0) blk_stamp(p, l, 0);
    stage_layer_input<true>(p, l, hin, hout, xb16, xf16, xss, s_part, s_amx, s_r, s_sh, slice_q0,
                            slice_q0 + slice_n);
    if (tid == 0) mbar_arrive(hinit_bar);
    stamp(p, l, 2);
    if (tid == 0) blk_stamp(p, l, 1);
    if (blockIdx.x == 0 && (p.x_trace || p.h_trace)) {
      for (int e = tid; e < H; e += 32 * STEP_CONSUMERS) {
        const __nv_bfloat16 xv = *reinterpret_cast<const __nv_bfloat16*>(xb16 + 2 * e);
        const float hv = l == 0 ? __bfloat162float(p.x_in[e]) : __ldcg(hin + e);
        if (p.x_trace) p.x_trace[(size_t)l * H + e] = xv;
        if (p.h_trace) p.h_trace[(size_t)l * H + e] = hv;
      }
    }

    // ---- router rows and shared units: task j on warp j % 8 ----
    {
      const bool ready = warp_ring_wait(fullA, par, p.status, &s_abort);
      if (lane == 0 && warp == 0) blk_stamp(p, l, 15);
      const uint32_t tag = (uint32_t)l + 1u;
      for (int j = warp; j < nr_w + ns; j += STEP_CONSUMERS) {
        if (j < nr_w) {
          float v = 0.0f;
          if (ready) bf16_dot1(X + (size_t)j * 2 * H, xb16, H, v);
          if (lane == 0) {
            st_tagged(p.logits + r0 + j, v, tag);
            blk_stamp(p, l, 2);
          }
        } else {
          const int s = j - nr_w;
          float vg = 0.0f, vu = 0.0f;
          if (ready) bf16_dot2(X + (size_t)(Z.nr + s) * 2 * H, X + (size_t)(Z.nr + Z.ns + s) * 2 * H, xb16, H, vg, vu);
          if (lane == 0) st_tagged(p.a_shared + s0 + s, silu_f32(vg) * vu, tag);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(emptyA);
    }
    stamp(p, l, 3);
    if (tid == 0) blk_stamp(p, l, 3);

    // ---- top-k and plan (every block, identical; polls the tagged logits) ----
    stamp(p, l, 4);
    step_topk<true>(p, l, P, s_ids, s_wts, s_wmax, s_ncand, s_cand, s_sel, &s_abort);
    if (tid == 0) mbar_arrive(plan_bar);
    stamp(p, l, 5);
    if (tid == 0) blk_stamp(p, l, 4);

    // ---- shared activation as bf16 hi + lo (over the dead bf16 x), while the routed
    //      W13 rows land; every slice of h initialised before the accumulations ----
    if (Is > 0) {
      for (int e = tid; e < Is / 8; e += 32 * STEP_CONSUMERS) {
        const unsigned long long* w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = p.a_shared + 8 * e + j;
        float a8[8];
        if (!await_tagged(w, 8, (uint32_t)l + 1u, a8, p.status, &s_abort)) {
#pragma unroll
          for (int j = 0; j < 8; ++j) a8[j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const __nv_bfloat16 hi = __float2bfloat16_rn(a8[j]);
          const __nv_bfloat16 lo = __float2bfloat16_rn(a8[j] - __bfloat162float(hi));
          *reinterpret_cast<__nv_bfloat16*>(shi + 2 * (8 * e + j)) = hi;
          *reinterpret_cast<__nv_bfloat16*>(slo + 2 * (8 * e + j)) = lo;
        }
      }
    }
    if (tid == 0) wait_counter(lc + CTR_HINIT, G, p.status, &s_abort);  // every slice of h initialised
    csync();

    // ---- routed W13 + SwiGLU: units round-robin over the 16 half-warps ----
    {
      int a, n;
      block_share(P.n_unique * I, a, n);
      const BLayout B = b_layout(p, p.layer[l], P, a, n, Y);
      // the (at most two) segments as scalars: no indexed struct in the loop
      const int nseg = B.sg.n;
      const int len0 = B.sg.len[0], len1 = nseg > 1 ? B.sg.len[1] : 0;
      const int hf0 = (len0 + 1) / 2, hf1 = (len1 + 1) / 2;  // first halves (landing first)
      const uint8_t* code0 = Y + B.dst_codes[0];
      const uint8_t* code1 = Y + (nseg > 1 ? B.dst_codes[1] : 0u);
      const uint32_t cb0 = (uint32_t)len0 * (uint32_t)(H / 2), cb1 = (uint32_t)len1 * (uint32_t)(H / 2);
      const uint8_t* gs0 = B.gsc[0];
      const uint8_t* gs1 = nseg > 1 ? B.gsc[1] : B.gsc[0];
      const uint8_t* us0 = B.usc[0];
      const uint8_t* us1 = nseg > 1 ? B.usc[1] : B.usc[0];
      const int eu0 = B.sg.u[0], eu1 = nseg > 1 ? B.sg.u[1] : 0;
      const int ej0 = B.sg.j0[0], ej1 = nseg > 1 ? B.sg.j0[1] : 0;
      const int hw = 2 * warp + (lane >> 4);
      const int nmine = hw < n ? (n - 1 - hw) / 16 + 1 : 0;
      const int nw = max(__shfl_sync(0xffffffffu, nmine, 0), __shfl_sync(0xffffffffu, nmine, 16));
      int done0 = 0, done1 = 0;  // units of each segment finished by this half-warp
      bool got0 = false, got1 = false, ready = true;
      for (int m = 0; m < nw; ++m) {
        const int q = hw + 16 * m;
        const bool live = q < n;
        const int qq = live ? q : 0;
        const bool s1 = qq >= len0;
        const int jj = s1 ? qq - len0 : qq;       // unit within its segment
        const bool second = jj >= (s1 ? hf1 : hf0);  // in the second half of its code rows
        // the warp waits for the halves either of its half-warps needs
        const bool need1 = __any_sync(0xffffffffu, live && second);
        if (!got0) {
          ready = warp_ring_wait(fullB, par, p.status, &s_abort) && ready;
          got0 = true;
          if (lane == 0 && warp == 0) blk_stamp(p, l, 13);
        }
        if (need1 && !got1) {
          ready = warp_ring_wait(fullB1, par, p.status, &s_abort) && ready;
          got1 = true;
        }
        const uint8_t* gate = (s1 ? code1 : code0) + (size_t)jj * (H / 2);
        float r[2] = {0.0f, 0.0f};
        if (ready)
          unit_dot(gate, gate + (s1 ? cb1 : cb0), (s1 ? gs1 : gs0) + (size_t)jj * (H / 32),
                   (s1 ? us1 : us0) + (size_t)jj * (H / 32), H / 32, xf16, s_sh[0], r[0], r[1]);
        if (live) {
          if ((lane & 15) == 0)
            p.a_routed[(size_t)(s1 ? eu1 : eu0) * I + (s1 ? ej1 : ej0) + jj] = silu_f32(r[0]) * r[1];
          if (s1)
            ++done1;
          else
            ++done0;
        }
      }
      __syncwarp();
      // per segment: the warp's finished units, counted towards the expert's I
      const int d0 = __shfl_sync(0xffffffffu, done0, 0) + __shfl_sync(0xffffffffu, done0, 16);
      const int d1 = __shfl_sync(0xffffffffu, done1, 0) + __shfl_sync(0xffffffffu, done1, 16);
      if (lane == 0 && (d0 > 0 || d1 > 0)) {
        __threadfence();
        if (d0 > 0) atomicAdd(lc + CTR_EXP + eu0, (unsigned)d0);
        if (d1 > 0) atomicAdd(lc + CTR_EXP + eu1, (unsigned)d1);
      }
      // the barriers must be passed before the region is released (a warp with no
      // units still waits, so the phase it releases is the current one)
      if (!got0) warp_ring_wait(fullB, par, p.status, &s_abort);
      if (!got1) warp_ring_wait(fullB1, par, p.status, &s_abort);
      if (lane == 0) mbar_arrive(emptyB);
    }
    stamp(p, l, 8);
    if (tid == 0) blk_stamp(p, l, 6);

    // ---- shared W2 rows, accumulated into h (activation staged after the top-k) ----
    stamp(p, l, 6);
    if (no > 0) {
      const bool ready = warp_ring_wait(fullS, par, p.status, &s_abort);
      for (int j = warp; j < no; j += STEP_CONSUMERS) {
        const float v = ready ? bf16_row_dot_hilo(X + Z.cs_off + (size_t)j * 2 * Is, shi, slo, Is) : 0.0f;
        if (lane == 0) atomicAdd(hout + o0 + j, v);
      }
    }
    stamp(p, l, 7);
    if (tid == 0) blk_stamp(p, l, 5);
    csync();  // x and the shared halves are dead: the routed-W2 activations take the region

    // ---- routed W2 (weighted), accumulated into h ----
    {
      int a, n;
      block_share(P.n_unique * H, a, n);
      const CLayout C = c_layout(p, p.layer[l], P, a, n);
      // warp k stages the activation of segment k's expert once its W13 units are
      // complete everywhere: f16, chunk-major, with its own power-of-two shift
      if (warp < C.sg.n) {
        const int u = C.sg.u[warp];
        if (lane == 0) wait_counter(lc + CTR_EXP + u, (unsigned)I, p.status, &s_abort);
        __syncwarp();
        uint8_t* dst = afc + (size_t)warp * ass;
        const float4* src = reinterpret_cast<const float4*>(p.a_routed + (size_t)u * I);
        float4 v[8];  // I <= 1024: at most 8 float4 per lane
        float amax = 0.0f;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int c4 = lane + 32 * jj;
          v[jj] = c4 < I / 4 ? __ldcg(src + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
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
            *reinterpret_cast<uint2*>(dst + chunk_major_off(4 * c4, I / 32)) = u2;
          }
        }
        if (lane == 0) s_ash[warp] = sh;
      }
      csync();
      // rows round-robin over 32 row slots of 8 lanes, two rows of a slot at a time;
      // the (at most two) segments as scalars
      const int len0 = C.sg.len[0];
      const bool two = C.sg.n > 1;
      const uint8_t* cd0 = X + C.dst_codes[0];
      const uint8_t* cd1 = X + (two ? C.dst_codes[1] : 0u);
      const uint8_t* sc0 = X + C.dst_sc[0] + C.rs[0].off;
      const uint8_t* sc1 = two ? X + C.dst_sc[1] + C.rs[1].off : sc0;
      const int oj0 = C.sg.j0[0], oj1 = two ? C.sg.j0[1] : 0;
      const float wt0 = n > 0 ? P.w[C.sg.u[0]][0] : 0.0f, wt1 = two ? P.w[C.sg.u[1]][0] : 0.0f;
      const int sh0 = s_ash[0], sh1 = two ? s_ash[1] : 0;
      const int rs = 4 * warp + (lane >> 3);
      const int nmine = rs < n ? (n - 1 - rs) / 32 + 1 : 0;
      int nw = max(nmine, __shfl_xor_sync(0xffffffffu, nmine, 8));
      nw = max(nw, __shfl_xor_sync(0xffffffffu, nw, 16));
      const bool ready = warp_ring_wait(fullC, par, p.status, &s_abort);
      if (lane == 0 && warp == 0) blk_stamp(p, l, 14);
      for (int m = 0; m < nw; m += 2) {
        const int qa = rs + 32 * m, qb = qa + 32;
        const bool la = qa < n, lb = qb < n;
        const int ra = la ? qa : 0, rb = lb ? qb : 0;
        const bool ka = ra >= len0, kb = rb >= len0;
        const int ja = ka ? ra - len0 : ra, jb = kb ? rb - len0 : rb;
        float r[2] = {0.0f, 0.0f};
        const uint8_t* rowa = (ka ? cd1 : cd0) + (size_t)ja * (I / 2);
        const uint8_t* rowb = (kb ? cd1 : cd0) + (size_t)jb * (I / 2);
        const uint8_t* sca = (ka ? sc1 : sc0) + (size_t)ja * (I / 32);
        const uint8_t* scb = (kb ? sc1 : sc0) + (size_t)jb * (I / 32);
        if (ready) {
          if (__all_sync(0xffffffffu, ka == kb)) {  // both rows of one expert: one set of activation loads
            w2_pair_dot(rowa, rowb, sca, scb, I / 32, afc + (ka ? ass : 0u), ka ? sh1 : sh0, r[0], r[1]);
          } else {
            r[0] = w2_row_dot(rowa, sca, I / 32, afc + (ka ? ass : 0u), ka ? sh1 : sh0);
            r[1] = w2_row_dot(rowb, scb, I / 32, afc + (kb ? ass : 0u), kb ? sh1 : sh0);
          }
        }
        if ((lane & 7) == 0) {
          const float wa = ka ? wt1 : wt0, wb = kb ? wt1 : wt0;
          if (la && wa != 0.0f) atomicAdd(hout + (ka ? oj1 : oj0) + ja, r[0] * wa);
          if (lb && wb != 0.0f) atomicAdd(hout + (kb ? oj1 : oj0) + jb, r[1] * wb);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(emptyX);
    }
    stamp(p, l, 10);
    csync();
    if (tid == 0) blk_stamp(p, l, 7);
    if (tid == 0) signal_counter(lc + CTR_H);
    stamp(p, l, 11);
  }

  // ---- LM-head input: bf16(RMSNorm(h_L)) by block 0 ----
  if (blockIdx.x != 0) return;
  if (tid == 0) wait_counter(ctr + (size_t)(L - 1) * CTR_PER_LAYER + CTR_H, G, p.status, &s_abort);
  csync();
  const float* hf = p.h + (size_t)((L - 1) & 1) * H;
  float ss = 0.0f;
  for (int c = tid; c < H / 4; c += 32 * STEP_CONSUMERS) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(hf) + c);
    ss = fmaf(v.x, v.x, ss);
    ss = fmaf(v.y, v.y, ss);
    ss = fmaf(v.z, v.z, ss);
    ss = fmaf(v.w, v.w, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) s_part[warp] = ss;
  csync();
  if (tid == 0) {
    float t = 0.0f;
    for (int w = 0; w < STEP_CONSUMERS; ++w) t += s_part[w];
    s_r[0] = 1.0f / sqrtf(t / (float)H + p.eps);
  }
  csync();
  for (int e = tid; e < H; e += 32 * STEP_CONSUMERS) {
    const float hv = __ldcg(hf + e);
    const __nv_bfloat16 v = __float2bfloat16_rn(hv * s_r[0]);
    p.x_final[e] = v;
    if (p.x_trace) p.x_trace[(size_t)L * H + e] = v;
    if (p.h_trace) p.h_trace[(size_t)L * H + e] = hv;
  }
}

}  // namespace moe
