// sq_linear.cu -- fused separated-quantization decode linear layer (sm_100a).
//
// Page: "1-bit量化不是玄学，以往掉点是机制问题" (m.lqnn.cn/news/241359):
//   section 2.3  the 1-bit trunk path by bit operations and the high-bit
//                residual path by integer products, results summed;
//   section 3.1  decode reads every weight once per token: bandwidth bound;
//   section 3.3  dequantization, trunk, residual and the sum fused in ONE
//                kernel, intermediates kept in registers / shared memory;
//   section 2.2  outlier channels at full precision against the weight.
// For token t and row r (m = trunk mask bit, b = sign bit, q = residual code):
//   T   = sum_j m*(2b-1)*xq_j = 2*sum_{m&b} xq - sum_m xq     exact int32
//   R_g = sum_{j in g} q_j*xq_j                                exact int32
//   U   = sum_i What[r][idx_i]*x_out_i, What = m*(+-alpha) + s_g*q
//   y   = sx*(alpha*T + sum_g s_g*R_g) + U
//
// Design (B200): the layer moves 1.156 bytes per weight and does a few
// integer operations per byte, so it is an HBM stream whose instruction
// budget is tight (~70 warp-instructions per KiB of codes at 7 TB/s).
// Measured on this part, plain wide loads with enough bytes in flight reach
// ~7.1 TB/s, while a ring of bulk asynchronous copies into shared memory
// sustains only about one stage per ~0.55 us per CTA (it needs >= 32 KB
// stages, too coarse to balance the small layers).  So:
//   * the weight is cut into 1024-channel pieces of one row; lane l of a warp
//     owns channels [32l, 32l+32) of a piece: one 256-bit load of codes, one
//     sign word, one group scale (a lane never spans two groups, G >= 32);
//   * each warp streams a contiguous range of pieces (split evenly over all
//     warps) through a register ring of kDepth pieces in flight, pointers
//     advanced incrementally;
//   * the trunk bits are expanded four at a time to 0/1 bytes and dotted
//     with xq by dp4a; the residual codes are dotted by dp4a and scaled once
//     per lane and piece; sum xq comes precomputed per piece;
//   * outlier channels are taken from the lane's own registers;
//   * a row shared by two warps is finished by its last contributor from
//     per-warp partials, summed in warp order (deterministic, no spin-wait).
// With programmatic dependent launch each warp issues its first weight loads
// before the previous kernel has finished; every other input is read, and
// every output written, only after it has completed.
#include <stdint.h>

#include <algorithm>
#include <cstdint>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kPiece = 1024;  // channels per piece: 32 per lane
// Pieces in flight per warp and CTAs per SM, per tokens per pass.
constexpr int kDepth1 = 5, kBps1 = 2;
constexpr int kDepth2 = 4, kBps2 = 2;
constexpr int kDepth4 = 3, kBps4 = 2;
constexpr int kBlocksPerSm = 2;  // the largest of the kBps*

int blocks_per_sm(int M) { return M == 1 ? kBps1 : (M == 2 ? kBps2 : kBps4); }

struct Params {
  const uint32_t* sign;
  const uint32_t* mask;
  const float* alpha;
  const int8_t* res;
  const float* scale;
  int N, K, K16, log2G, ng, sign_stride, res_stride, scale_stride;
  int xs;            // row stride of xq (roundup(K, 128))
  int ppr;          // pieces per row = ceil(K16 / 1024)
  int P;            // total pieces = N * ppr (< 2^31)
  int warps_total;  // warps that own pieces: min(gridDim.x * kWarps, P); the rest idle
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
  int32_t* status;
  int pdl;
};

// One piece as seen by one lane: 32 codes, 32 sign bits (32 mask bits), the
// lane's group scale.
struct Piece {
  int q[8];
  uint32_t b;
  uint32_t m;
  float s;
};

__device__ __forceinline__ int warp_begin(int w, const Params& p) {
  return (int)((int64_t)w * p.P / p.warps_total);
}
// warp that owns piece g
__device__ __forceinline__ int piece_owner(int g, const Params& p) {
  return (int)(((int64_t)(g + 1) * p.warps_total + p.P - 1) / p.P) - 1;
}

__device__ __forceinline__ void ld32B_v4x2(int* v, const int8_t* p) {
  const int4 a = ldg_nc_v4(p), b = ldg_nc_v4(p + 16);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// 32 streamed bytes (read once): 32-byte aligned when V8, else 16.
template <bool V8>
__device__ __forceinline__ void ld32B_stream(int* v, const int8_t* p) {
  if (V8) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.s32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "l"(p));
  } else {
    ld32B_v4x2(v, p);
  }
}

// 32 bytes of activation codes: reused by every row, so they stay in L1.
template <bool V8>
__device__ __forceinline__ void ld32B_cached(int* v, const int8_t* p) {
  if (V8) {
    asm volatile("ld.global.nc.v8.s32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "l"(p));
  } else {
    ld32B_v4x2(v, p);
  }
}

// Streaming position of one lane: row, piece in row, and its pointers.
struct Cursor {
  int row, pc;
  const int8_t* res;
  const uint32_t* sign;
  const uint32_t* mask;
  const float* scale;
};

__device__ __forceinline__ void cursor_seek(Cursor& c, const Params& p, int row, int pc, int lane) {
  c.row = row;
  c.pc = pc;
  const int k = pc * kPiece + lane * 32;
  c.res = p.res + (int64_t)row * p.res_stride + k;
  c.sign = p.sign + (int64_t)row * p.sign_stride + (k >> 5);
  c.mask = p.mask + (int64_t)row * p.sign_stride + (k >> 5);  // unused without a mask
  c.scale = p.scale + (int64_t)row * p.scale_stride + (k >> p.log2G);
}

__device__ __forceinline__ void cursor_next(Cursor& c, const Params& p, int lane) {
  if (++c.pc == p.ppr) {
    cursor_seek(c, p, c.row + 1, 0, lane);
  } else {
    c.res += kPiece;
    c.sign += kPiece / 32;
    c.mask += kPiece / 32;
    c.scale += kPiece >> p.log2G;
  }
}

template <bool MASK, bool V8>
__device__ __forceinline__ void load_piece(Piece& pc, const Cursor& c, const Params& p, int lane,
                                           bool live) {
  const int k = c.pc * kPiece + lane * 32;
  if (live && k < p.K16) {
    if (k + 32 <= p.K16) {
      ld32B_stream<V8>(pc.q, c.res);
    } else {  // last 16 bytes of a row whose stride is 16 mod 32
      const int4 a = ldg_nc_v4(c.res);
      pc.q[0] = a.x; pc.q[1] = a.y; pc.q[2] = a.z; pc.q[3] = a.w;
      pc.q[4] = pc.q[5] = pc.q[6] = pc.q[7] = 0;
    }
    pc.b = __ldg(c.sign);
    pc.m = MASK ? __ldg(c.mask) : 0xFFFFFFFFu;
    pc.s = __ldg(c.scale);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) pc.q[i] = 0;
    pc.b = 0;
    pc.m = 0;
    pc.s = 0.0f;
  }
}

__device__ __forceinline__ int pick_word(const int* q, int w) {
  // register select (no dynamically indexed local array)
  const int a = (w & 1) ? q[1] : q[0], b = (w & 1) ? q[3] : q[2];
  const int c = (w & 1) ? q[5] : q[4], d = (w & 1) ? q[7] : q[6];
  const int ab = (w & 2) ? b : a, cd = (w & 2) ? d : c;
  return (w & 4) ? cd : ab;
}

template <int M, int D, int BPS, bool MASK, bool EMIT, bool V8>
__global__ void __launch_bounds__(kThreads, BPS) k_linear(const Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  // shared: Sx[M][ppr] i32 | omask[nw] u32 (outlier bits per 32 channels) |
  //         obase[nw] i32 (first outlier of the word) | xo[M][n_pad] f32 | sx[M] f32
  const int nw = (p.K16 + 31) >> 5;
  int* sx_sum = reinterpret_cast<int*>(smem);
  uint32_t* omask = reinterpret_cast<uint32_t*>(sx_sum + M * p.ppr);
  int* obase = reinterpret_cast<int*>(omask + nw);
  const int n_pad = (p.n_out + 3) & ~3;
  float* xo_s = reinterpret_cast<float*>(obase + nw);
  float* sx_s = xo_s + M * n_pad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;
  // every owning warp has >= 1 piece, so the owners of a row are consecutive
  const int g0 = gw < p.warps_total ? warp_begin(gw, p) : p.P;
  const int g1 = gw < p.warps_total ? warp_begin(gw + 1, p) : p.P;

  // ---- prefetch the first D pieces (weights only; allowed before the wait)
  Piece buf[D];
  Cursor ic;
  cursor_seek(ic, p, g0 / p.ppr, g0 % p.ppr, lane);
#pragma unroll
  for (int d = 0; d < D; ++d) {
    load_piece<MASK, V8>(buf[d], ic, p, lane, g0 + d < g1);
    if (g0 + d + 1 < g1) cursor_next(ic, p, lane);
  }

  if (p.pdl) pdl_wait();

  // ---- per-block tables (after the previous kernel completed) -------------
  for (int i = threadIdx.x; i < nw; i += kThreads) omask[i] = 0u;
  for (int i = threadIdx.x; i < M * p.ppr; i += kThreads) sx_sum[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < p.n_out; i += kThreads) {
    const int j = p.idx[i];
    if (j >= 0 && j < p.K) {
      atomicOr(&omask[j >> 5], 1u << (j & 31));
      // the first outlier of each 32-channel word (the list is ascending)
      if (i == 0 || (p.idx[i - 1] >> 5) != (j >> 5)) obase[j >> 5] = i;
    }
#pragma unroll
    for (int t = 0; t < M; ++t) xo_s[t * n_pad + i] = p.xout[(int64_t)t * p.n_out + i];
  }
  if (threadIdx.x < M) sx_s[threadIdx.x] = p.sx[threadIdx.x];
  if (!MASK) {  // per-piece sums of xq for T = 2*P - S
    const int nseg = p.K16 >> 4;
    for (int t = 0; t < M; ++t)
      for (int seg = threadIdx.x; seg < nseg; seg += kThreads) {
        const int4 x = ldg_nc_v4(p.xq + (int64_t)t * p.xs + seg * 16);
        int s = __dp4a(x.x, 0x01010101, 0);
        s = __dp4a(x.y, 0x01010101, s);
        s = __dp4a(x.z, 0x01010101, s);
        s = __dp4a(x.w, 0x01010101, s);
        atomicAdd(&sx_sum[t * p.ppr + (seg >> 6)], s);
      }
  }
  __syncthreads();
  if (p.pdl) pdl_launch_dependents();

  // ---- main loop -----------------------------------------------------------
  int accP[M], accS[M];
  float accF[M], accUt[M], accUr[M];
#pragma unroll
  for (int t = 0; t < M; ++t) {
    accP[t] = 0;
    accS[t] = 0;
    accF[t] = 0.0f;
    accUt[t] = 0.0f;
    accUr[t] = 0.0f;
  }
  int crow = g0 / p.ppr;
  int cc = g0 - crow * p.ppr;
  float row_alpha = (g0 < g1) ? __ldg(p.alpha + crow) : 0.0f;
  bool row_head = (cc == 0);  // the current row started inside this warp's range
  const int8_t* xq_lane = p.xq + lane * 32;

  for (int g = g0; g < g1; g += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (g + d < g1) {
        Piece& pc = buf[d];
        const int k = cc * kPiece + lane * 32;
        const bool act = k < p.K16;
        const uint32_t mb = pc.b & pc.m;
        int e[8], f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          e[i] = expand_nibble(mb >> (4 * i));
          if (MASK) f[i] = expand_nibble(pc.m >> (4 * i));
        }
#pragma unroll
        for (int t = 0; t < M; ++t) {
          int x[8];
          if (act) {
            const int8_t* xp = xq_lane + (int64_t)t * p.xs + cc * kPiece;
            if (k + 32 <= p.K16) {
              ld32B_cached<V8>(x, xp);
            } else {
              const int4 a = ldg_nc_v4(xp);
              x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
              x[4] = x[5] = x[6] = x[7] = 0;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = 0;
          }
          int R = 0, Pt = accP[t];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            R = __dp4a(pc.q[i], x[i], R);
            Pt = __dp4a(e[i], x[i], Pt);
          }
          accP[t] = Pt;
          if (MASK) {
            int St = accS[t];
#pragma unroll
            for (int i = 0; i < 8; ++i) St = __dp4a(f[i], x[i], St);
            accS[t] = St;
          }
          accF[t] = fmaf(pc.s, (float)R, accF[t]);
          if (EMIT) {
            const int sh = p.log2G - 5;  // lanes per group = 2^sh
            for (int o = 1; o < (1 << sh); o <<= 1) R += __shfl_xor_sync(0xffffffffu, R, o);
            if (act && (lane & ((1 << sh) - 1)) == 0)
              p.R_out[((int64_t)t * p.N + crow) * p.ng + (k >> p.log2G)] = R;
          }
        }
        if (!MASK && lane == 0) {
#pragma unroll
          for (int t = 0; t < M; ++t) accS[t] += sx_sum[t * p.ppr + cc];
        }
        // outlier channels among this lane's 32
        uint32_t om = act ? omask[k >> 5] : 0u;
        if (om) {
          int pos = obase[k >> 5];
          do {
            const int bit = __ffs(om) - 1;
            om &= om - 1;
            const int qv = (int)(int8_t)(pick_word(pc.q, bit >> 2) >> (8 * (bit & 3)));
            const bool in_trunk = (pc.m >> bit) & 1u;
            const float sgn = ((pc.b >> bit) & 1u) ? 1.0f : -1.0f;
            const float rq = pc.s * (float)qv;
            // (an index list that is not strictly ascending cannot push pos
            // past the staged values)
            if (pos >= 0 && pos < p.n_out) {
#pragma unroll
              for (int t = 0; t < M; ++t) {
                const float xv = xo_s[t * n_pad + pos];
                if (in_trunk) accUt[t] = fmaf(sgn, xv, accUt[t]);
                accUr[t] = fmaf(rq, xv, accUr[t]);
              }
            }
            ++pos;
          } while (om);
        }

        // refill this slot with the piece D ahead
        const bool live = g + d + D < g1;
        load_piece<MASK, V8>(buf[d], ic, p, lane, live);
        if (live) cursor_next(ic, p, lane);

        // end of a row, or end of this warp's range
        if (cc == p.ppr - 1 || g + d + 1 == g1) {
#pragma unroll
          for (int t = 0; t < M; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              accP[t] += __shfl_xor_sync(0xffffffffu, accP[t], o);
              if (MASK) accS[t] += __shfl_xor_sync(0xffffffffu, accS[t], o);
              accF[t] += __shfl_xor_sync(0xffffffffu, accF[t], o);
              accUt[t] += __shfl_xor_sync(0xffffffffu, accUt[t], o);
              accUr[t] += __shfl_xor_sync(0xffffffffu, accUr[t], o);
            }
          }
          if (lane == 0) {
            int T[M];
#pragma unroll
            for (int t = 0; t < M; ++t) {
              T[t] = 2 * accP[t] - accS[t];
              if (EMIT) atomicAdd(&p.T_out[(int64_t)t * p.N + crow], T[t]);
            }
            if (row_head && cc == p.ppr - 1) {
#pragma unroll
              for (int t = 0; t < M; ++t) {
                const float inner = fmaf(row_alpha, (float)T[t], accF[t]);
                p.y[(int64_t)t * p.N + crow] =
                    fmaf(sx_s[t], inner, fmaf(row_alpha, accUt[t], accUr[t]));
              }
            } else {
              // publish this warp's part of the row; the last arrival sums
              // every part in warp order and writes y
              const int slot = row_head ? 1 : 0;  // 0: head row of the range, 1: tail row
              float* part = p.ws_part + (((size_t)gw * 2 + slot) * M) * 4;
#pragma unroll
              for (int t = 0; t < M; ++t) {
                part[t * 4 + 0] = __int_as_float(T[t]);
                part[t * 4 + 1] = accF[t];
                part[t * 4 + 2] = accUt[t];
                part[t * 4 + 3] = accUr[t];
              }
              __threadfence();
              const int w_first = piece_owner(crow * p.ppr, p);
              const int w_last = piece_owner(crow * p.ppr + p.ppr - 1, p);
              const int prev = atomicAdd(&p.ws_cnt[crow], 1);
              if (prev == w_last - w_first) {
                __threadfence();
                int Tt[M];
                float Ft[M], Ut[M], Ur[M];
#pragma unroll
                for (int t = 0; t < M; ++t) {
                  Tt[t] = 0;
                  Ft[t] = 0.0f;
                  Ut[t] = 0.0f;
                  Ur[t] = 0.0f;
                }
                for (int w = w_first; w <= w_last; ++w) {
                  // a contributor whose range starts inside the row published
                  // it as its head row (slot 0), any other as its tail (slot 1)
                  const int sl = warp_begin(w, p) > crow * p.ppr ? 0 : 1;
                  const float* pb = p.ws_part + (((size_t)w * 2 + sl) * M) * 4;
#pragma unroll
                  for (int t = 0; t < M; ++t) {
                    Tt[t] += __float_as_int(__ldcg(pb + t * 4 + 0));
                    Ft[t] += __ldcg(pb + t * 4 + 1);
                    Ut[t] += __ldcg(pb + t * 4 + 2);
                    Ur[t] += __ldcg(pb + t * 4 + 3);
                  }
                }
#pragma unroll
                for (int t = 0; t < M; ++t) {
                  const float inner = fmaf(row_alpha, (float)Tt[t], Ft[t]);
                  p.y[(int64_t)t * p.N + crow] = fmaf(sx_s[t], inner, fmaf(row_alpha, Ut[t], Ur[t]));
                }
                p.ws_cnt[crow] = 0;
              }
            }
          }
#pragma unroll
          for (int t = 0; t < M; ++t) {
            accP[t] = 0;
            accS[t] = 0;
            accF[t] = 0.0f;
            accUt[t] = 0.0f;
            accUr[t] = 0.0f;
          }
          if (g + d + 1 < g1) {
            row_alpha = __ldg(p.alpha + crow + 1);
            row_head = true;
          }
        }
        if (++cc == p.ppr) {
          cc = 0;
          ++crow;
        }
      }
    }
  }
}

template <int M, int D, int BPS, bool MASK, bool EMIT, bool V8>
cudaError_t launch_one(const Params& p, const LinearPlan& plan, bool pdl, cudaStream_t stream) {
  auto* fn = k_linear<M, D, BPS, MASK, EMIT, V8>;
  cudaError_t e = ensure_smem_attr((const void*)fn, plan.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

template <bool MASK, bool EMIT, bool V8>
cudaError_t dispatch_m(int M, const Params& p, const LinearPlan& plan, bool pdl, cudaStream_t st) {
  switch (M) {
    case 1: return launch_one<1, kDepth1, kBps1, MASK, EMIT, V8>(p, plan, pdl, st);
    case 2: return launch_one<2, kDepth2, kBps2, MASK, EMIT, V8>(p, plan, pdl, st);
    case 3: return launch_one<3, kDepth4, kBps4, MASK, EMIT, V8>(p, plan, pdl, st);
    case 4: return launch_one<4, kDepth4, kBps4, MASK, EMIT, V8>(p, plan, pdl, st);
    default: return cudaErrorInvalidValue;
  }
}

template <bool MASK, bool EMIT>
cudaError_t dispatch_v8(bool v8, int M, const Params& p, const LinearPlan& plan, bool pdl,
                        cudaStream_t st) {
  return v8 ? dispatch_m<MASK, EMIT, true>(M, p, plan, pdl, st)
            : dispatch_m<MASK, EMIT, false>(M, p, plan, pdl, st);
}

int log2_exact(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

}  // namespace

bool plan_linear(const sq_packed_weight& w, int M, int n_out, int sm_count, LinearPlan* plan) {
  if (M < 1 || M > kMaxTokensPerPass || sm_count < 1) return false;
  LinearPlan pl;
  pl.M = M;
  const int64_t K16 = round_up(w.K, 16);
  const int64_t ppr = ceil_div(K16, kPiece);
  const int64_t P = (int64_t)w.N * ppr;
  if (P >= INT32_MAX) return false;
  // about two pieces per warp at least, at most blocks_per_sm(M) CTAs per SM
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count * blocks_per_sm(M),
                                                                ceil_div(P, 2 * kWarps)));
  pl.grid = (int)blocks;
  pl.Kc = kPiece;
  pl.n_c = (int)ppr;
  pl.U = (int)P;
  const int64_t nw = ceil_div(K16, 32);
  const int64_t n_pad = round_up(n_out, 4);
  const int64_t smem = (int64_t)M * ppr * 4 + nw * 4 + nw * 4 + (int64_t)M * n_pad * 4 + M * 4 + 16;
  pl.smem_bytes = (int)round_up(smem, 16);
  pl.ws_part_bytes = linear_part_bytes(sm_count);
  pl.ws_cnt_bytes = (size_t)round_up((int64_t)w.N * 4, 256);
  *plan = pl;
  return true;
}

size_t linear_part_bytes(int sm_count) {
  const size_t core = (size_t)sm_count * kBlocksPerSm * kWarps * 2 * kMaxTokensPerPass * 4 * sizeof(float);
  return (size_t)round_up((int64_t)std::max(core, linear_tc_part_bytes(sm_count)), 256);
}

size_t linear_workspace_bytes(const sq_packed_weight& w, int M, int sm_count) {
  LinearPlan pl;
  if (!plan_linear(w, std::min(std::max(M, 1), kMaxTokensPerPass), 0, sm_count, &pl)) return 0;
  return pl.ws_part_bytes + pl.ws_cnt_bytes;
}

cudaError_t launch_linear(const sq_packed_weight& w, const LinearPlan& plan, const int8_t* xq,
                          const float* sx, const float* x_out, const int32_t* idx, int n_out,
                          float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                          size_t part_bytes, int32_t* status, bool pdl, cudaStream_t stream) {
  Params p;
  p.sign = w.sign_bits;
  p.mask = w.mask_bits;
  p.alpha = w.alpha;
  p.res = w.res_q;
  p.scale = w.res_scale;
  p.N = w.N;
  p.K = w.K;
  p.K16 = w.res_stride;
  p.xs = (int)xq_stride_of(w.K);
  p.log2G = log2_exact(w.group_size);
  p.ng = (int)ceil_div(w.K, w.group_size);
  p.sign_stride = w.sign_stride;
  p.res_stride = w.res_stride;
  p.scale_stride = w.scale_stride;
  p.ppr = plan.n_c;
  p.P = w.N * plan.n_c;
  p.warps_total = std::min(plan.grid * kWarps, p.P);
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
  p.status = status;
  p.pdl = pdl ? 1 : 0;
  // 256-bit loads need 32-byte aligned rows of codes and of activation codes
  const bool v8 = (w.res_stride % 32) == 0 && (reinterpret_cast<uintptr_t>(w.res_q) % 32) == 0 &&
                  (reinterpret_cast<uintptr_t>(xq) % 32) == 0;
  const bool mask = w.mask_bits != nullptr;
  const bool emit = T_out != nullptr;
  if (mask)
    return emit ? dispatch_v8<true, true>(v8, plan.M, p, plan, pdl, stream)
                : dispatch_v8<true, false>(v8, plan.M, p, plan, pdl, stream);
  return emit ? dispatch_v8<false, true>(v8, plan.M, p, plan, pdl, stream)
              : dispatch_v8<false, false>(v8, plan.M, p, plan, pdl, stream);
}

}  // namespace sq
