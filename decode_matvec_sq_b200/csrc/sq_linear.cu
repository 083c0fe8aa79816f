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
// integer operations per byte, so it is an HBM stream.  Measured on this
// part, plain 128-bit loads with enough bytes in flight reach ~7.1 TB/s,
// while a ring of bulk asynchronous copies sustains only about one stage per
// ~0.55 us per CTA (it needs >= 32 KB stages, too coarse to balance the small
// layers).  So every lane loads its own weight bytes with LDG.128 straight
// into a register ring that keeps kDepth 512-channel pieces in flight per
// warp (~110 KB per SM), the trunk bits are expanded to bytes and dotted with
// dp4a, the residual codes are dotted with dp4a per 16-channel segment and
// scaled once per segment, and the outlier channels are taken from the
// lane's own registers.  Work = 512-channel pieces of the row-major weight,
// split evenly over all warps of a grid of kBlocksPerSm CTAs per SM; a row
// shared by two warps is finished by its last contributor from per-warp
// partials in a fixed order (deterministic, no spin-wait).  With programmatic
// dependent launch each warp issues its first weight loads before the
// previous kernel has finished; every other input is read, and every output
// written, only after it has completed.
#include <stdint.h>

#include <algorithm>
#include <cstdint>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
// Pieces in flight per warp and CTAs per SM, per tokens per pass: keep
// ~100+ KB of weight loads in flight per SM without register spills.
constexpr int kDepth1 = 6, kBps1 = 3;
constexpr int kDepth2 = 4, kBps2 = 3;
constexpr int kDepth4 = 4, kBps4 = 2;
constexpr int kBlocksPerSm = 3;  // the largest of the kBps*

int blocks_per_sm(int M) { return M == 1 ? kBps1 : (M == 2 ? kBps2 : kBps4); }
constexpr int kPiece = 512;  // channels per piece: 16 per lane
constexpr int kMaxPiecesPerRow = (1 << 24) / kPiece;

struct Params {
  const uint32_t* sign;
  const uint32_t* mask;
  const float* alpha;
  const int8_t* res;
  const float* scale;
  int N, K, K16, log2G, ng, sign_stride, res_stride, scale_stride;
  int ppr;          // pieces per row = ceil(K16 / 512)
  int P;            // total pieces = N * ppr (< 2^31)
  int warps_total;  // gridDim.x * kWarps
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

// One 512-channel piece as seen by one lane: 16 codes, 16 sign bits (and 16
// mask bits), the scale of the lane's group.
struct Piece {
  int4 q;
  uint32_t bm;  // sign bits (low 16) and mask bits (high 16)
  float s;
};

__device__ __forceinline__ int warp_begin(int w, const Params& p) {
  return (int)((int64_t)w * p.P / p.warps_total);
}
// warp that owns piece g
__device__ __forceinline__ int piece_owner(int g, const Params& p) {
  return (int)(((int64_t)(g + 1) * p.warps_total + p.P - 1) / p.P) - 1;
}

template <bool MASK>
__device__ __forceinline__ void load_piece(Piece& pc, const Params& p, int row, int c, int lane,
                                           bool live) {
  const int k = c * kPiece + lane * 16;
  if (live && k < p.K16) {
    pc.q = ldg_nc_v4(p.res + (int64_t)row * p.res_stride + k);
    const uint16_t* sg = reinterpret_cast<const uint16_t*>(p.sign + (int64_t)row * p.sign_stride);
    pc.bm = __ldg(sg + (k >> 4));
    if (MASK)
      pc.bm |= (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(p.mask + (int64_t)row * p.sign_stride) +
                               (k >> 4)) << 16;
    pc.s = __ldg(p.scale + (int64_t)row * p.scale_stride + (k >> p.log2G));
  } else {
    pc.q = make_int4(0, 0, 0, 0);
    pc.bm = 0;
    pc.s = 0.0f;
  }
}

template <int M, int D, int BPS, bool MASK, bool EMIT>
__global__ void __launch_bounds__(kThreads, BPS) k_linear(const Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  // shared layout: Sx[M][ppr] int, omask[roundup(K16/16, 2)] u16 (outlier
  //                channel bits per 16-channel segment), idx[n_pad] int,
  //                xo[M][n_pad] f32, sx[M] f32
  const int nseg = p.K16 >> 4;
  const int nseg2 = (nseg + 1) & ~1;
  int* sx_sum = reinterpret_cast<int*>(smem);
  uint16_t* omask = reinterpret_cast<uint16_t*>(sx_sum + M * p.ppr);
  const int n_pad = (p.n_out + 3) & ~3;
  int* idx_s = reinterpret_cast<int*>(omask + nseg2);
  float* xo_s = reinterpret_cast<float*>(idx_s + n_pad);
  float* sx_s = xo_s + M * n_pad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;
  const int g0 = warp_begin(gw, p), g1 = warp_begin(gw + 1, p);

  // ---- prefetch the first D pieces (weights only; allowed before the wait)
  Piece buf[D];
  int irow = g0 / p.ppr;
  int ic = (int)(g0 - irow * p.ppr);
#pragma unroll
  for (int d = 0; d < D; ++d) {
    load_piece<MASK>(buf[d], p, irow, ic, lane, g0 + d < g1);
    if (++ic == p.ppr) {
      ic = 0;
      ++irow;
    }
  }

  if (p.pdl) pdl_wait();

  // ---- per-block tables (after the previous kernel completed) -------------
  for (int i = threadIdx.x; i < nseg2; i += kThreads) omask[i] = 0;
  for (int i = threadIdx.x; i < M * p.ppr; i += kThreads) sx_sum[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < p.n_out; i += kThreads) {
    const int j = p.idx[i];
    idx_s[i] = j;
    if (j >= 0 && j < p.K) atomicOr(reinterpret_cast<unsigned int*>(omask) + (j >> 5), 1u << (j & 31));
#pragma unroll
    for (int t = 0; t < M; ++t) xo_s[t * n_pad + i] = p.xout[(int64_t)t * p.n_out + i];
  }
  if (threadIdx.x < M) sx_s[threadIdx.x] = p.sx[threadIdx.x];
  // per-piece sums of xq (for T = 2*P - S without a mask)
  if (!MASK) {
    for (int t = 0; t < M; ++t)
      for (int seg = threadIdx.x; seg < nseg; seg += kThreads) {
        const int4 x = ldg_nc_v4(p.xq + (int64_t)t * p.K16 + seg * 16);
        int s = __dp4a(x.x, 0x01010101, 0);
        s = __dp4a(x.y, 0x01010101, s);
        s = __dp4a(x.z, 0x01010101, s);
        s = __dp4a(x.w, 0x01010101, s);
        atomicAdd(&sx_sum[t * p.ppr + (seg >> 5)], s);
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
  int cc = (int)(g0 - crow * p.ppr);
  float row_alpha = (g0 < g1) ? __ldg(p.alpha + crow) : 0.0f;
  bool row_head = true;  // the current row started inside this warp's range?
  row_head = (cc == 0);

  for (int g = g0; g < g1; g += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (g + d < g1) {
        Piece& pc = buf[d];
        const int seg = cc * 32 + lane;  // 16-channel segment index in the row
        const int k = seg * 16;
        const bool act = k < p.K16;
        const uint32_t pb_ = pc.bm & 0xFFFFu, pm_ = MASK ? (pc.bm >> 16) : 0xFFFFu;
        const uint32_t mb = pb_ & pm_;
        const int e0 = expand_nibble(mb), e1 = expand_nibble(mb >> 4), e2 = expand_nibble(mb >> 8),
                  e3 = expand_nibble(mb >> 12);
        int f0 = 0, f1 = 0, f2 = 0, f3 = 0;
        if (MASK) {
          f0 = expand_nibble(pm_);
          f1 = expand_nibble(pm_ >> 4);
          f2 = expand_nibble(pm_ >> 8);
          f3 = expand_nibble(pm_ >> 12);
        }
#pragma unroll
        for (int t = 0; t < M; ++t) {
          int4 x = make_int4(0, 0, 0, 0);
          if (act) x = ldg_nc_v4(p.xq + (int64_t)t * p.K16 + k);
          int R = __dp4a(pc.q.x, x.x, 0);
          R = __dp4a(pc.q.y, x.y, R);
          R = __dp4a(pc.q.z, x.z, R);
          R = __dp4a(pc.q.w, x.w, R);
          accF[t] = fmaf(pc.s, (float)R, accF[t]);
          accP[t] = __dp4a(e0, x.x, __dp4a(e1, x.y, __dp4a(e2, x.z, __dp4a(e3, x.w, accP[t]))));
          if (MASK) accS[t] = __dp4a(f0, x.x, __dp4a(f1, x.y, __dp4a(f2, x.z, __dp4a(f3, x.w, accS[t]))));
          if (EMIT) {
            const int sh = p.log2G - 4;  // segments per group = 2^sh
            for (int o = 1; o < (1 << sh); o <<= 1) R += __shfl_xor_sync(0xffffffffu, R, o);
            if (act && (lane & ((1 << sh) - 1)) == 0)
              p.R_out[((int64_t)t * p.N + crow) * p.ng + (k >> p.log2G)] = R;
          }
        }
        if (!MASK && lane == 0) {
#pragma unroll
          for (int t = 0; t < M; ++t) accS[t] += sx_sum[t * p.ppr + cc];
        }
        // outlier channels among this lane's 16
        uint32_t om = act ? omask[seg] : 0u;
        if (om) {
          // position of the segment's first outlier in the ascending list
          int pos = 0, hi = p.n_out;
          while (pos < hi) {
            const int mid = (pos + hi) >> 1;
            if (idx_s[mid] < k)
              pos = mid + 1;
            else
              hi = mid;
          }
          do {
            const int bit = __ffs(om) - 1;
            om &= om - 1;
            const int wsel = bit >> 2;
            const int word = wsel == 0 ? pc.q.x : (wsel == 1 ? pc.q.y : (wsel == 2 ? pc.q.z : pc.q.w));
            const int qv = (int)(int8_t)(word >> (8 * (bit & 3)));
            const bool in_trunk = MASK ? ((pm_ >> bit) & 1u) : true;
            const float sgn = ((pb_ >> bit) & 1u) ? 1.0f : -1.0f;
            const float rq = pc.s * (float)qv;
#pragma unroll
            for (int t = 0; t < M; ++t) {
              // (an index list that is not strictly ascending cannot push
              // pos past the staged values)
              const float xv = pos < p.n_out ? xo_s[t * n_pad + pos] : 0.0f;
              if (in_trunk) accUt[t] = fmaf(sgn, xv, accUt[t]);
              accUr[t] = fmaf(rq, xv, accUr[t]);
            }
            ++pos;
          } while (om);
        }

        // refill this slot with the piece D ahead
        load_piece<MASK>(buf[d], p, irow, ic, lane, g + d + D < g1);
        if (++ic == p.ppr) {
          ic = 0;
          ++irow;
        }

        // end of a row, or end of this warp's range
        const bool row_end = (cc == p.ppr - 1) || (g + d + 1 == g1);
        if (row_end) {
#pragma unroll
          for (int t = 0; t < M; ++t) {
            for (int o = 16; o > 0; o >>= 1) {
              accP[t] += __shfl_xor_sync(0xffffffffu, accP[t], o);
              accS[t] += __shfl_xor_sync(0xffffffffu, accS[t], o);
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
            const bool whole = row_head && cc == p.ppr - 1;
            if (whole) {
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

template <int M, int D, int BPS, bool MASK, bool EMIT>
cudaError_t launch_one(const Params& p, const LinearPlan& plan, bool pdl, cudaStream_t stream) {
  auto* fn = k_linear<M, D, BPS, MASK, EMIT>;
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

template <bool MASK, bool EMIT>
cudaError_t dispatch_m(int M, const Params& p, const LinearPlan& plan, bool pdl, cudaStream_t st) {
  switch (M) {
    case 1: return launch_one<1, kDepth1, kBps1, MASK, EMIT>(p, plan, pdl, st);
    case 2: return launch_one<2, kDepth2, kBps2, MASK, EMIT>(p, plan, pdl, st);
    case 3: return launch_one<3, kDepth4, kBps4, MASK, EMIT>(p, plan, pdl, st);
    case 4: return launch_one<4, kDepth4, kBps4, MASK, EMIT>(p, plan, pdl, st);
    default: return cudaErrorInvalidValue;
  }
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
  if (ppr > kMaxPiecesPerRow) return false;
  const int64_t P = (int64_t)w.N * ppr;
  if (P >= INT32_MAX) return false;
  // at least ~4 pieces per warp, at most kBlocksPerSm CTAs per SM
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count * blocks_per_sm(M),
                                                                ceil_div(P, 4 * kWarps)));
  pl.grid = (int)blocks;
  pl.Kc = kPiece;
  pl.n_c = (int)ppr;
  pl.U = (int)std::min<int64_t>(P, INT32_MAX);
  const int nseg = (int)(K16 / 16);
  const int n_pad = (int)round_up(n_out, 4);
  size_t smem = (size_t)M * ppr * 4 + (size_t)round_up(nseg, 2) * 2 + (size_t)n_pad * 4 +
                (size_t)M * n_pad * 4 + (size_t)M * 4 + 16;
  pl.smem_bytes = (int)round_up((int64_t)smem, 16);
  // workspace: [partial sums, sized for the largest grid on this device]
  //            [per-row arrival counters]; the first area does not depend on
  //            the weight, so one workspace can serve weights of any N
  pl.ws_part_bytes = (size_t)sm_count * kBlocksPerSm * kWarps * 2 * kMaxTokensPerPass * 4 * sizeof(float);
  pl.ws_cnt_bytes = (size_t)round_up((int64_t)w.N * 4, 256);
  *plan = pl;
  return true;
}

size_t linear_workspace_bytes(const sq_packed_weight& w, int M, int sm_count) {
  LinearPlan pl;
  if (!plan_linear(w, std::min(std::max(M, 1), kMaxTokensPerPass), 0, sm_count, &pl)) return 0;
  return pl.ws_part_bytes + pl.ws_cnt_bytes;
}

cudaError_t launch_linear(const sq_packed_weight& w, const LinearPlan& plan, const int8_t* xq,
                          const float* sx, const float* x_out, const int32_t* idx, int n_out,
                          float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                          int32_t* status, bool pdl, cudaStream_t stream) {
  Params p;
  p.sign = w.sign_bits;
  p.mask = w.mask_bits;
  p.alpha = w.alpha;
  p.res = w.res_q;
  p.scale = w.res_scale;
  p.N = w.N;
  p.K = w.K;
  p.K16 = w.res_stride;
  p.log2G = log2_exact(w.group_size);
  p.ng = (int)ceil_div(w.K, w.group_size);
  p.sign_stride = w.sign_stride;
  p.res_stride = w.res_stride;
  p.scale_stride = w.scale_stride;
  p.ppr = plan.n_c;
  p.P = w.N * plan.n_c;
  p.warps_total = plan.grid * kWarps;
  p.xq = xq;
  p.sx = sx;
  p.xout = x_out;
  p.idx = idx;
  p.n_out = n_out;
  p.y = y;
  p.T_out = T_out;
  p.R_out = R_out;
  p.ws_part = reinterpret_cast<float*>(workspace);
  p.ws_cnt = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(workspace) + plan.ws_part_bytes);
  p.status = status;
  p.pdl = pdl ? 1 : 0;
  const bool mask = w.mask_bits != nullptr;
  const bool emit = T_out != nullptr;
  if (mask)
    return emit ? dispatch_m<true, true>(plan.M, p, plan, pdl, stream)
                : dispatch_m<true, false>(plan.M, p, plan, pdl, stream);
  return emit ? dispatch_m<false, true>(plan.M, p, plan, pdl, stream)
              : dispatch_m<false, false>(plan.M, p, plan, pdl, stream);
}

}  // namespace sq
