// sq_linear_tc.cu -- the decode linear layer on the tensor cores (sm_100a).
//
// Page: "1-bit量化不是玄学，以往掉点是机制问题" (m.lqnn.cn/news/241359),
// section 2.3: the 1-bit trunk product and the high-bit residual product are
// computed side by side and summed; section 3.3: all of it in one kernel.
//
// Same results as sq_linear.cu (bit-exact integer accumulators, fp32 y); the
// default decode kernel for group size 128, up to 8 tokens per pass:
//   * residual: four int8 MMAs (mma.sync m16n8k32, one token per column) per
//     128-channel group give the exact group accumulators R_g of 16 rows,
//     promoted once per group with the group scales;
//   * trunk: each lane expands its sign bits (and mask bits) four at a time
//     to 0/1 bytes and runs the same int8 MMAs against the same activation
//     codes: P = sum_{m and b} xq and S = sum_m xq (an all-ones operand
//     without a mask) accumulate in MMA fragments across a row's tiles, and
//     T = 2P - S.  (A binary AND/popcount MMA would read the bits directly,
//     but on sm_100 it is emulated at ~69 instructions per m16n8k128, ten
//     times the int8 MMA, while expanding a nibble costs ~3.)
// The MMA's reduction order over k is free, so each lane feeds the MMAs the
// 32 contiguous channels it loaded with one 256-bit load, and takes the
// matching 32 bytes of activation codes: no reshuffling of the stream.
// Tile = 16 rows x 128 channels (one group); work = tiles in row-block-major
// order split evenly over the warps; every lane ends a row block holding the
// finished sums of its two rows and two tokens, so no reduction is needed;
// a row block shared by warps is finished by its last contributor from
// per-warp partials, summed in warp order (deterministic); the fence and the
// arrival counts wait until the warp's stream has drained.
#include <stdint.h>

#include <algorithm>
#include <cstdint>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBps = 2;       // CTAs per SM
constexpr int kTileK = 128;   // channels per tile (= group size)
constexpr int kTileRows = 16;
constexpr int kDepth = 3;     // tiles in flight per warp
constexpr int kCols = 8;      // tokens per pass (MMA N)

struct Params {
  const uint32_t* sign;
  const uint32_t* mask;
  const float* alpha;
  const int8_t* res;
  const float* scale;
  int N, K, K16, ng, sign_stride, res_stride, scale_stride;
  int tpr;          // tiles per row block = ceil(K16 / 128)
  int T;            // total tiles = ceil(N / 16) * tpr
  int warps_total;  // warps that own tiles: min(gridDim.x * kWarps, T); the rest idle
  int M;            // tokens in this pass (<= 8)
  const int8_t* xq;
  const float* sx;
  const float* xout;
  const int32_t* idx;
  int n_out;
  float* y;
  int32_t* T_out;
  int32_t* R_out;
  float* ws_part;
  int32_t* ws_cnt;
  int pdl;
};

__device__ __forceinline__ int warp_begin(int w, const Params& p) {
  return (int)((int64_t)w * p.T / p.warps_total);
}
__device__ __forceinline__ int tile_owner(int g, const Params& p) {
  return (int)(((int64_t)(g + 1) * p.warps_total + p.T - 1) / p.T) - 1;
}

__device__ __forceinline__ void mma_s8(int (&c)[4], int a0, int a1, int a2, int a3, int b0, int b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 32 bytes (full) or 16 bytes + zeros, 32-byte aligned when V8 and full.
// Codes are streamed once (no L1 allocation); activation codes are reused by
// every row (cached).
template <bool V8, bool STREAM>
__device__ __forceinline__ void ld32(int* v, const int8_t* p, bool full) {
  if (V8 && full) {
    if (STREAM)
      asm volatile("ld.global.nc.L1::no_allocate.v8.s32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                     "=r"(v[6]), "=r"(v[7])
                   : "l"(p));
    else
      asm volatile("ld.global.nc.v8.s32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                     "=r"(v[6]), "=r"(v[7])
                   : "l"(p));
  } else {
    const int4 a = ldg_nc_v4(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    if (full) {
      const int4 b = ldg_nc_v4(p + 16);
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      v[4] = v[5] = v[6] = v[7] = 0;
    }
  }
}

// One tile as seen by one lane: rows r0 = 16*rb + gid and r1 = r0 + 8,
// channels [128*g + 32*tid4, +32).
template <bool MASK>
struct Tile {
  int a0[8], a1[8];   // codes of r0, r1
  uint32_t s0, s1;    // sign words
  float c0, c1;       // group scales
};
template <>
struct Tile<true> {
  int a0[8], a1[8];
  uint32_t s0, s1;
  uint32_t mw0, mw1;  // mask words
  float c0, c1;
};

template <bool MASK>
__device__ __forceinline__ uint32_t tile_mask(const Tile<MASK>& t, int r);
template <>
__device__ __forceinline__ uint32_t tile_mask<false>(const Tile<false>&, int) { return 0xFFFFFFFFu; }
template <>
__device__ __forceinline__ uint32_t tile_mask<true>(const Tile<true>& t, int r) { return r ? t.mw1 : t.mw0; }

template <bool MASK, bool V8>
__device__ __forceinline__ void load_tile(Tile<MASK>& t, const Params& p, int rb, int g, int gid,
                                          int tid4, bool live) {
  const int r0 = rb * kTileRows + gid, r1 = r0 + 8;
  const int k = g * kTileK + tid4 * 32;
  const bool kin = live && k < p.K16;
  const bool full = k + 32 <= p.K16;
  // the group scale promotes this lane's accumulator columns, which sum the
  // whole group: every lane of a live tile loads it, also a lane whose own 32
  // channels lie past the padded row end
  t.c0 = live && r0 < p.N ? __ldg(p.scale + (int64_t)r0 * p.scale_stride + g) : 0.0f;
  t.c1 = live && r1 < p.N ? __ldg(p.scale + (int64_t)r1 * p.scale_stride + g) : 0.0f;
  if (kin && r0 < p.N) {
    ld32<V8, true>(t.a0, p.res + (int64_t)r0 * p.res_stride + k, full);
    t.s0 = __ldg(p.sign + (int64_t)r0 * p.sign_stride + (k >> 5));
    if constexpr (MASK) t.mw0 = __ldg(p.mask + (int64_t)r0 * p.sign_stride + (k >> 5));
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) t.a0[i] = 0;
    t.s0 = 0;
    if constexpr (MASK) t.mw0 = 0;
  }
  if (kin && r1 < p.N) {
    ld32<V8, true>(t.a1, p.res + (int64_t)r1 * p.res_stride + k, full);
    t.s1 = __ldg(p.sign + (int64_t)r1 * p.sign_stride + (k >> 5));
    if constexpr (MASK) t.mw1 = __ldg(p.mask + (int64_t)r1 * p.sign_stride + (k >> 5));
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) t.a1[i] = 0;
    t.s1 = 0;
    if constexpr (MASK) t.mw1 = 0;
  }
}

__device__ __forceinline__ int pick_word(const int* q, int w) {
  const int a = (w & 1) ? q[1] : q[0], b = (w & 1) ? q[3] : q[2];
  const int c = (w & 1) ? q[5] : q[4], d = (w & 1) ? q[7] : q[6];
  const int ab = (w & 2) ? b : a, cd = (w & 2) ? d : c;
  return (w & 4) ? cd : ab;
}

// Row-block accumulators of one lane: rows (gid, gid + 8) x tokens
// (2*tid4, 2*tid4 + 1), in MMA accumulator order (r0t0, r0t1, r1t0, r1t1).
struct Acc {
  int P[4], S[4];           // trunk sums: sum_{m and b} xq, sum_m xq
  float F[4], Ut[4], Ur[4]; // sum_g s_g R_g; outlier terms (trunk, residual)
};

__device__ __forceinline__ void acc_zero(Acc& a) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a.P[i] = 0;
    a.S[i] = 0;
    a.F[i] = 0.0f;
    a.Ut[i] = 0.0f;
    a.Ur[i] = 0.0f;
  }
}

template <bool MASK, bool EMIT, bool V8>
__global__ void __launch_bounds__(kThreads, kBps) k_linear_tc(const Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  // shared: omask[nw32] u32 | obase[nw32] i32 | xo[M][n_pad] f32 | sx[M] f32
  const int nw32 = (p.K16 + 31) >> 5;
  uint32_t* omask = reinterpret_cast<uint32_t*>(smem);
  int* obase = reinterpret_cast<int*>(omask + nw32);
  const int n_pad = (p.n_out + 3) & ~3;
  float* xo_s = reinterpret_cast<float*>(obase + nw32);
  float* sx_s = xo_s + p.M * n_pad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid4 = lane & 3;
  const int gw = blockIdx.x * kWarps + warp;
  // every owning warp has >= 1 tile, so the owners of a row block are consecutive
  const int t0 = gw < p.warps_total ? warp_begin(gw, p) : p.T;
  const int t1 = gw < p.warps_total ? warp_begin(gw + 1, p) : p.T;

  // ---- prefetch the first kDepth tiles (weights only; allowed before the wait)
  Tile<MASK> buf[kDepth];
  int irb = t0 / p.tpr, ig = t0 - irb * p.tpr;
#pragma unroll
  for (int d = 0; d < kDepth; ++d) {
    load_tile<MASK, V8>(buf[d], p, irb, ig, gid, tid4, t0 + d < t1);
    if (++ig == p.tpr) {
      ig = 0;
      ++irb;
    }
  }

  if (p.pdl) pdl_wait();

  for (int i = threadIdx.x; i < nw32; i += kThreads) omask[i] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < p.n_out; i += kThreads) {
    const int j = p.idx[i];
    if (j >= 0 && j < p.K) {
      atomicOr(&omask[j >> 5], 1u << (j & 31));
      if (i == 0 || (p.idx[i - 1] >> 5) != (j >> 5)) obase[j >> 5] = i;
    }
    for (int t = 0; t < p.M; ++t) xo_s[t * n_pad + i] = p.xout[(int64_t)t * p.n_out + i];
  }
  if (threadIdx.x < p.M) sx_s[threadIdx.x] = p.sx[threadIdx.x];
  __syncthreads();
  if (p.pdl) pdl_launch_dependents();

  // tokens of this lane's accumulator columns
  const int tk0 = 2 * tid4, tk1 = 2 * tid4 + 1;
  Acc acc;
  acc_zero(acc);
  int crb = t0 / p.tpr, cg = t0 - crb * p.tpr;
  bool rb_head = (cg == 0);  // the current row block started inside this range
  bool have_head = false;
  int head_rb = -1;

  for (int g = t0; g < t1; g += kDepth) {
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      if (g + d < t1) {
        Tile<MASK>& tl = buf[d];
        const int k = cg * kTileK + tid4 * 32;
        const bool kin = k < p.K16;
        // activation codes of token gid (the MMA column this lane feeds)
        int xw[8];
        if (gid < p.M && kin) {
          ld32<V8, false>(xw, p.xq + (int64_t)gid * p.K16 + k, k + 32 <= p.K16);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) xw[i] = 0;
        }
        const uint32_t tm0 = tile_mask<MASK>(tl, 0), tm1 = tile_mask<MASK>(tl, 1);
        const uint32_t pb0 = tl.s0 & tm0, pb1 = tl.s1 & tm1;
        int R[4] = {0, 0, 0, 0};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          // residual codes of channels 8m..8m+7 of this lane's 32
          mma_s8(R, tl.a0[2 * m], tl.a1[2 * m], tl.a0[2 * m + 1], tl.a1[2 * m + 1], xw[2 * m],
                 xw[2 * m + 1]);
          // trunk bits of the same channels, as 0/1 bytes
          const int e0 = expand_nibble(pb0 >> (8 * m)), e0h = expand_nibble(pb0 >> (8 * m + 4));
          const int e1 = expand_nibble(pb1 >> (8 * m)), e1h = expand_nibble(pb1 >> (8 * m + 4));
          mma_s8(acc.P, e0, e1, e0h, e1h, xw[2 * m], xw[2 * m + 1]);
          if (MASK) {
            const int f0 = expand_nibble(tm0 >> (8 * m)), f0h = expand_nibble(tm0 >> (8 * m + 4));
            const int f1 = expand_nibble(tm1 >> (8 * m)), f1h = expand_nibble(tm1 >> (8 * m + 4));
            mma_s8(acc.S, f0, f1, f0h, f1h, xw[2 * m], xw[2 * m + 1]);
          } else {
            mma_s8(acc.S, 0x01010101, 0x01010101, 0x01010101, 0x01010101, xw[2 * m], xw[2 * m + 1]);
          }
        }
        // promote the group accumulators: R[0..1] row r0, R[2..3] row r1
        acc.F[0] = fmaf(tl.c0, (float)R[0], acc.F[0]);
        acc.F[1] = fmaf(tl.c0, (float)R[1], acc.F[1]);
        acc.F[2] = fmaf(tl.c1, (float)R[2], acc.F[2]);
        acc.F[3] = fmaf(tl.c1, (float)R[3], acc.F[3]);
        if (EMIT) {
          const int r0 = crb * kTileRows + gid, r1 = r0 + 8;
          if (tk0 < p.M) {
            if (r0 < p.N) p.R_out[((int64_t)tk0 * p.N + r0) * p.ng + cg] = R[0];
            if (r1 < p.N) p.R_out[((int64_t)tk0 * p.N + r1) * p.ng + cg] = R[2];
          }
          if (tk1 < p.M) {
            if (r0 < p.N) p.R_out[((int64_t)tk1 * p.N + r0) * p.ng + cg] = R[1];
            if (r1 < p.N) p.R_out[((int64_t)tk1 * p.N + r1) * p.ng + cg] = R[3];
          }
        }
        // outlier channels of this tile (the same for every row): the lane
        // holding the channel forms the dequantized weight of its two rows;
        // the four lanes of its row group take it by shuffle
        const int wbase = (cg * kTileK) >> 5;
        const uint32_t om = kin ? omask[wbase + tid4] : 0u;
        uint32_t any = __ballot_sync(0xffffffffu, om != 0u) & 0xFu;  // lanes 0..3 = chunks 0..3
        while (any) {
          const int src = __ffs(any) - 1;
          any &= any - 1;
          uint32_t bits = __shfl_sync(0xffffffffu, om, src);
          int pos = __shfl_sync(0xffffffffu, kin ? obase[wbase + tid4] : 0, src);
          while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1;
            float w0 = 0.0f, w1 = 0.0f, t0w = 0.0f, t1w = 0.0f;
            if (tid4 == src) {
              const int q0 = (int)(int8_t)(pick_word(tl.a0, bit >> 2) >> (8 * (bit & 3)));
              const int q1 = (int)(int8_t)(pick_word(tl.a1, bit >> 2) >> (8 * (bit & 3)));
              t0w = ((tm0 >> bit) & 1u) ? (((tl.s0 >> bit) & 1u) ? 1.0f : -1.0f) : 0.0f;
              t1w = ((tm1 >> bit) & 1u) ? (((tl.s1 >> bit) & 1u) ? 1.0f : -1.0f) : 0.0f;
              w0 = tl.c0 * (float)q0;
              w1 = tl.c1 * (float)q1;
            }
            const int owner = gid * 4 + src;
            w0 = __shfl_sync(0xffffffffu, w0, owner);
            w1 = __shfl_sync(0xffffffffu, w1, owner);
            t0w = __shfl_sync(0xffffffffu, t0w, owner);
            t1w = __shfl_sync(0xffffffffu, t1w, owner);
            // (an index list that is not strictly ascending cannot push pos
            // past the staged values)
            if (pos >= 0 && pos < p.n_out) {
              const float x0 = tk0 < p.M ? xo_s[tk0 * n_pad + pos] : 0.0f;
              const float x1 = tk1 < p.M ? xo_s[tk1 * n_pad + pos] : 0.0f;
              acc.Ut[0] = fmaf(t0w, x0, acc.Ut[0]);
              acc.Ut[1] = fmaf(t0w, x1, acc.Ut[1]);
              acc.Ut[2] = fmaf(t1w, x0, acc.Ut[2]);
              acc.Ut[3] = fmaf(t1w, x1, acc.Ut[3]);
              acc.Ur[0] = fmaf(w0, x0, acc.Ur[0]);
              acc.Ur[1] = fmaf(w0, x1, acc.Ur[1]);
              acc.Ur[2] = fmaf(w1, x0, acc.Ur[2]);
              acc.Ur[3] = fmaf(w1, x1, acc.Ur[3]);
            }
            ++pos;
          }
        }

        // refill this slot with the tile kDepth ahead
        const bool live = g + d + kDepth < t1;
        load_tile<MASK, V8>(buf[d], p, irb, ig, gid, tid4, live);
        if (live && ++ig == p.tpr) {
          ig = 0;
          ++irb;
        }

        // end of a row block, or end of this warp's range
        if (cg == p.tpr - 1 || g + d + 1 == t1) {
          const int r0 = crb * kTileRows + gid, r1 = r0 + 8;
          int T[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) T[i] = 2 * acc.P[i] - acc.S[i];
          if (EMIT) {
            if (tk0 < p.M && r0 < p.N) atomicAdd(&p.T_out[(int64_t)tk0 * p.N + r0], T[0]);
            if (tk1 < p.M && r0 < p.N) atomicAdd(&p.T_out[(int64_t)tk1 * p.N + r0], T[1]);
            if (tk0 < p.M && r1 < p.N) atomicAdd(&p.T_out[(int64_t)tk0 * p.N + r1], T[2]);
            if (tk1 < p.M && r1 < p.N) atomicAdd(&p.T_out[(int64_t)tk1 * p.N + r1], T[3]);
          }
          if (rb_head && cg == p.tpr - 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = (i < 2) ? r0 : r1, tk = (i & 1) ? tk1 : tk0;
              if (row < p.N && tk < p.M) {
                const float al = __ldg(p.alpha + row);
                p.y[(int64_t)tk * p.N + row] =
                    fmaf(sx_s[tk], fmaf(al, (float)T[i], acc.F[i]), fmaf(al, acc.Ut[i], acc.Ur[i]));
              }
            }
          } else {
            // shared row block: slot 0 if this range started inside it (its
            // head), else slot 1 (its tail: the range ends inside it)
            const int slot = rb_head ? 1 : 0;
            if (!rb_head) {
              have_head = true;
              head_rb = crb;
            }
            float4* part = reinterpret_cast<float4*>(p.ws_part) + (((size_t)gw * 2 + slot) * 32 + lane) * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              part[i] = make_float4(__int_as_float(T[i]), acc.F[i], acc.Ut[i], acc.Ur[i]);
          }
          acc_zero(acc);
          if (g + d + 1 < t1) rb_head = true;
        }
        if (++cg == p.tpr) {
          cg = 0;
          ++crb;
        }
      }
    }
  }

  // ---- arrival counts for shared row blocks; the last contributor finishes
  const int last_rb = (t1 - 1) / p.tpr;
  const bool tail_partial = t1 > t0 && (t1 % p.tpr) != 0;
  if (!have_head && !tail_partial) return;
  __threadfence();
  __syncwarp();
  for (int which = 0; which < 2; ++which) {
    const int rb = which == 0 ? head_rb : last_rb;
    if (which == 0 && !have_head) continue;
    if (which == 1 && (!tail_partial || (have_head && last_rb == head_rb))) continue;
    const int w_first = tile_owner(rb * p.tpr, p);
    const int w_last = tile_owner(rb * p.tpr + p.tpr - 1, p);
    int prev = 0;
    if (lane == 0) prev = atomicAdd(&p.ws_cnt[rb], 1);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != w_last - w_first) continue;
    __threadfence();
    // sum the parts in warp order (the same lane layout in every part)
    int Tt[4] = {0, 0, 0, 0};
    float Ft[4] = {0, 0, 0, 0}, Ut[4] = {0, 0, 0, 0}, Ur[4] = {0, 0, 0, 0};
    for (int w = w_first; w <= w_last; ++w) {
      const int sl = warp_begin(w, p) > rb * p.tpr ? 0 : 1;  // head part or tail part
      const float4* pb =
          reinterpret_cast<const float4*>(p.ws_part) + (((size_t)w * 2 + sl) * 32 + lane) * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldcg(pb + i);
        Tt[i] += __float_as_int(v.x);
        Ft[i] += v.y;
        Ut[i] += v.z;
        Ur[i] += v.w;
      }
    }
    const int r0 = rb * kTileRows + gid, r1 = r0 + 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = (i < 2) ? r0 : r1, tk = (i & 1) ? tk1 : tk0;
      if (row < p.N && tk < p.M) {
        const float al = __ldg(p.alpha + row);
        p.y[(int64_t)tk * p.N + row] = fmaf(sx_s[tk], fmaf(al, (float)Tt[i], Ft[i]), fmaf(al, Ut[i], Ur[i]));
      }
    }
    if (lane == 0) p.ws_cnt[rb] = 0;
  }
}

template <bool MASK, bool EMIT, bool V8>
cudaError_t launch_one(const Params& p, int grid, int smem, bool pdl, cudaStream_t stream) {
  auto* fn = k_linear_tc<MASK, EMIT, V8>;
  cudaError_t e = ensure_smem_attr((const void*)fn, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace

size_t linear_tc_part_bytes(int sm_count) {
  // per warp: two slots of 32 lanes x 4 (row, token) cells x 4 floats
  return (size_t)sm_count * kBps * kWarps * 2 * 32 * 4 * 4 * sizeof(float);
}

bool linear_tc_supported(const sq_packed_weight& w) { return w.group_size == kTileK; }

cudaError_t launch_linear_tc(const sq_packed_weight& w, int M, const int8_t* xq, const float* sx,
                             const float* x_out, const int32_t* idx, int n_out, float* y,
                             int32_t* T_out, int32_t* R_out, void* workspace, size_t part_bytes,
                             int sm_count, bool pdl, cudaStream_t stream) {
  if (M < 1 || M > kCols) return cudaErrorInvalidValue;
  Params p;
  p.sign = w.sign_bits;
  p.mask = w.mask_bits;
  p.alpha = w.alpha;
  p.res = w.res_q;
  p.scale = w.res_scale;
  p.N = w.N;
  p.K = w.K;
  p.K16 = w.res_stride;
  p.ng = (int)ceil_div(w.K, w.group_size);
  p.sign_stride = w.sign_stride;
  p.res_stride = w.res_stride;
  p.scale_stride = w.scale_stride;
  p.tpr = (int)ceil_div(w.res_stride, kTileK);
  const int64_t T = ceil_div(w.N, kTileRows) * (int64_t)p.tpr;
  if (T >= INT32_MAX) return cudaErrorInvalidValue;
  p.T = (int)T;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count * kBps,
                                                                ceil_div(T, 2 * kWarps)));
  p.warps_total = (int)std::min<int64_t>(blocks * kWarps, T);
  p.M = M;
  p.xq = xq;
  p.sx = sx;
  p.xout = x_out;
  p.idx = idx;
  p.n_out = n_out;
  p.y = y;
  p.T_out = T_out;
  p.R_out = R_out;
  p.ws_part = reinterpret_cast<float*>(workspace);
  p.ws_cnt = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(workspace) + part_bytes);
  p.pdl = pdl ? 1 : 0;
  const int nw32 = (int)ceil_div(w.res_stride, 32);
  const int n_pad = (int)round_up(n_out, 4);
  const int smem = (int)round_up((int64_t)nw32 * 8 + (int64_t)M * n_pad * 4 + M * 4 + 16, 16);
  const bool v8 = (w.res_stride % 32) == 0 && (reinterpret_cast<uintptr_t>(w.res_q) % 32) == 0 &&
                  (reinterpret_cast<uintptr_t>(xq) % 32) == 0;
  const bool mask = w.mask_bits != nullptr;
  const bool emit = T_out != nullptr;
  const int grid = (int)blocks;
  if (mask) {
    if (emit) return v8 ? launch_one<true, true, true>(p, grid, smem, pdl, stream)
                        : launch_one<true, true, false>(p, grid, smem, pdl, stream);
    return v8 ? launch_one<true, false, true>(p, grid, smem, pdl, stream)
              : launch_one<true, false, false>(p, grid, smem, pdl, stream);
  }
  if (emit) return v8 ? launch_one<false, true, true>(p, grid, smem, pdl, stream)
                      : launch_one<false, true, false>(p, grid, smem, pdl, stream);
  return v8 ? launch_one<false, false, true>(p, grid, smem, pdl, stream)
            : launch_one<false, false, false>(p, grid, smem, pdl, stream);
}

}  // namespace sq
