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
//   y   = sx*(alpha*T + sum_g s_g*R_g) + sum_i What[r][idx_i]*x_out_i
//
// Design (B200): the kernel is HBM bound (1.156 bytes per weight), so it is
// a streaming pipeline.  One producer warp moves the packed rows into a ring
// of shared-memory stages with bulk asynchronous copies (cp.async.bulk,
// mbarrier completion, L2 evict-first); eight consumer warps, one per row of
// an 8-row block, expand the sign bits to bytes and accumulate both dot
// products with dp4a, reading xq through the read-only path (it is reused by
// every row).  Work = (8-row block, K chunk) units, split evenly over one CTA
// per SM; a row block split between CTAs is finished by its last contributor
// from per-CTA partials in a fixed order (deterministic).  With programmatic
// dependent launch the producer streams weights before the previous kernel
// has finished; consumers touch inputs and outputs only after it completes.
#include <stdint.h>

#include <algorithm>
#include <cstdint>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kConsumerWarps = kRowsPerBlock;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kChunkMax = 2048;         // channels per unit (multiple of 512)
constexpr int kStageBudget = 160 * 1024;
constexpr int kMaxStages = 8;

struct Params {
  const uint32_t* sign;
  const uint32_t* mask;
  const float* alpha;
  const int8_t* res;
  const float* scale;
  int N, K, K16, log2G, ng, sign_stride, res_stride, scale_stride;
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
  int Kc, n_c, U, grid, S, stage_bytes, off_sign, off_mask, off_scale, off_alpha, hdr_bytes;
  int pdl;
};

__device__ __forceinline__ int unit_begin(int b, const Params& p) {
  return (int)((int64_t)b * p.U / p.grid);
}
// CTA that owns unit u.
__device__ __forceinline__ int unit_owner(int u, const Params& p) {
  return (int)(((int64_t)(u + 1) * p.grid + p.U - 1) / p.U) - 1;
}

template <int M, bool MASK, bool EMIT>
__global__ void __launch_bounds__(kThreads, 1) k_linear(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + p.S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + p.S);
  int* chunk_lo = reinterpret_cast<int*>(empty + p.S) + 4;
  int* idx_s = chunk_lo + ((p.n_c + 1 + 3) & ~3);
  float* xo_s = reinterpret_cast<float*>(idx_s + ((p.n_out + 3) & ~3));
  float* sx_s = xo_s + M * ((p.n_out + 3) & ~3);
  uint8_t* stages = smem + p.hdr_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int u_begin = unit_begin(cta, p), u_end = unit_begin(cta + 1, p);
  const int n_units = u_end - u_begin;
  const int n_pad = (p.n_out + 3) & ~3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------ producer ------------------------------
    const uint64_t policy = l2_evict_first_policy();
    const int per_row = MASK ? 4 : 3;
    const int scale_per_chunk = p.Kc >> p.log2G;
    bool waited = p.pdl == 0;
    int issued = 0;
    bool failed = false;
    for (int i = 0; i < n_units; ++i) {
      const int s = i % p.S;
      if (i >= p.S) {
        if (!waited) {
          pdl_wait();
          waited = true;
        }
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], ((i / p.S) - 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok || *abort_flag) {
          failed = !ok;
          break;
        }
      }
      const int u = u_begin + i;
      const int rb = u / p.n_c, c = u - rb * p.n_c;
      const int row0 = rb * kRowsPerBlock;
      const int rows = min(kRowsPerBlock, p.N - row0);
      const int k0 = c * p.Kc;
      const uint32_t res_b = (uint32_t)min(p.Kc, p.K16 - k0);
      const uint32_t sign_b = 4u * (uint32_t)min(p.Kc / 32, p.sign_stride - k0 / 32);
      const uint32_t scale_b = 4u * (uint32_t)min(scale_per_chunk, p.scale_stride - c * scale_per_chunk);
      const uint32_t alpha_b = (uint32_t)((rows * 4 + 15) & ~15);
      const uint32_t total = (uint32_t)rows * (res_b + sign_b * (MASK ? 2u : 1u) + scale_b) + alpha_b;
      uint8_t* st = stages + (size_t)s * p.stage_bytes;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], total);
      __syncwarp();
      const int ncopies = rows * per_row + 1;
      for (int ci = lane; ci < ncopies; ci += 32) {
        if (ci == ncopies - 1) {
          bulk_g2s(st + p.off_alpha, p.alpha + row0, alpha_b, &full[s], policy);
          continue;
        }
        const int r = ci / per_row, kind = ci - r * per_row;
        const int64_t row = row0 + r;
        if (kind == 0) {
          bulk_g2s(st + r * p.Kc, p.res + row * p.res_stride + k0, res_b, &full[s], policy);
        } else if (kind == 1) {
          bulk_g2s(st + p.off_sign + r * (p.Kc / 8), p.sign + row * p.sign_stride + k0 / 32,
                   sign_b, &full[s], policy);
        } else if (kind == 2) {
          bulk_g2s(st + p.off_scale + r * scale_per_chunk * 4,
                   p.scale + row * p.scale_stride + (int64_t)c * scale_per_chunk, scale_b, &full[s],
                   policy);
        } else {
          bulk_g2s(st + p.off_mask + r * (p.Kc / 8), p.mask + row * p.sign_stride + k0 / 32,
                   sign_b, &full[s], policy);
        }
      }
      ++issued;
    }
    if (failed || *abort_flag) {
      // do not leave copies in flight into shared memory: wait (bounded) for
      // the latest phase of every stage that was issued
      if (failed) {
        set_status(p.status, SQ_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (lane == 0)
        for (int i = max(0, issued - p.S); i < issued; ++i)
          (void)mbar_wait(&full[i % p.S], (i / p.S) & 1);
    }
    return;
  }

  // ------------------------------- consumers --------------------------------
  if (p.pdl) pdl_wait();
  const int ctid = threadIdx.x;  // 0 .. 255
  for (int i = ctid; i < p.n_out; i += kConsumerWarps * 32) {
    idx_s[i] = p.idx[i];
#pragma unroll
    for (int t = 0; t < M; ++t) xo_s[t * n_pad + i] = p.xout[(int64_t)t * p.n_out + i];
  }
  for (int c = ctid; c <= p.n_c; c += kConsumerWarps * 32) {
    // first outlier channel >= c*Kc (lower bound over the ascending list)
    int lo = 0, hi = p.n_out;
    const int key = c * p.Kc;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (p.idx[mid] < key)
        lo = mid + 1;
      else
        hi = mid;
    }
    chunk_lo[c] = lo;
  }
  if (ctid < M) sx_s[ctid] = p.sx[ctid];
  named_sync(1, kConsumerWarps * 32);
  if (p.pdl) pdl_launch_dependents();

  int accP[M], accS[M];
  float accF[M], accU[M];
#pragma unroll
  for (int t = 0; t < M; ++t) {
    accP[t] = 0;
    accS[t] = 0;
    accF[t] = 0.0f;
    accU[t] = 0.0f;
  }
  float row_alpha = 0.0f;
  const int scale_per_chunk = p.Kc >> p.log2G;
  const int seg_per_group_log2 = p.log2G - 4;  // 16-channel segments per group

  for (int i = 0; i < n_units; ++i) {
    const int s = i % p.S;
    bool ok = true;
    if (lane == 0) ok = mbar_wait(&full[s], (i / p.S) & 1);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      set_status(p.status, SQ_ERR_TIMEOUT);
      *abort_flag = 1;
      return;
    }
    if (*abort_flag) return;
    const int u = u_begin + i;
    const int rb = u / p.n_c, c = u - rb * p.n_c;
    const int row = rb * kRowsPerBlock + warp;
    const bool valid = row < p.N;
    const int k0 = c * p.Kc;
    const int kc_len = min(p.Kc, p.K16 - k0);
    const int nseg = kc_len >> 4;
    const uint8_t* st = stages + (size_t)s * p.stage_bytes;
    if (valid) {
      const int4* rres = reinterpret_cast<const int4*>(st + warp * p.Kc);
      const uint16_t* rsg = reinterpret_cast<const uint16_t*>(st + p.off_sign + warp * (p.Kc / 8));
      const uint16_t* rmk = reinterpret_cast<const uint16_t*>(st + p.off_mask + warp * (p.Kc / 8));
      const float* rsc = reinterpret_cast<const float*>(st + p.off_scale) + warp * scale_per_chunk;
      row_alpha = reinterpret_cast<const float*>(st + p.off_alpha)[warp];
      const int8_t* xbase = p.xq + k0;
      for (int it = 0; it * 32 < nseg; ++it) {
        const int seg = it * 32 + lane;
        const bool act = seg < nseg;
        int4 q = make_int4(0, 0, 0, 0);
        uint32_t b = 0, m = 0xFFFFu;
        float sg = 0.0f;
        if (act) {
          q = rres[seg];
          b = rsg[seg];
          if (MASK) m = rmk[seg];
          sg = rsc[seg >> seg_per_group_log2];
        }
        const uint32_t mb = b & m;
        const int e0 = expand_nibble(mb), e1 = expand_nibble(mb >> 4), e2 = expand_nibble(mb >> 8),
                  e3 = expand_nibble(mb >> 12);
        int f0 = 0x01010101, f1 = 0x01010101, f2 = 0x01010101, f3 = 0x01010101;
        if (MASK) {
          f0 = expand_nibble(m);
          f1 = expand_nibble(m >> 4);
          f2 = expand_nibble(m >> 8);
          f3 = expand_nibble(m >> 12);
        }
#pragma unroll
        for (int t = 0; t < M; ++t) {
          int4 x = make_int4(0, 0, 0, 0);
          if (act) x = ldg_nc_v4(xbase + (int64_t)t * p.K16 + seg * 16);
          int R = __dp4a(q.x, x.x, 0);
          R = __dp4a(q.y, x.y, R);
          R = __dp4a(q.z, x.z, R);
          R = __dp4a(q.w, x.w, R);
          accF[t] = fmaf(sg, (float)R, accF[t]);
          accP[t] = __dp4a(e0, x.x, __dp4a(e1, x.y, __dp4a(e2, x.z, __dp4a(e3, x.w, accP[t]))));
          accS[t] = __dp4a(f0, x.x, __dp4a(f1, x.y, __dp4a(f2, x.z, __dp4a(f3, x.w, accS[t]))));
          if (EMIT) {
            // exact per-group accumulator: sum over the lanes of this group
            for (int o = 1; o < (1 << seg_per_group_log2); o <<= 1)
              R += __shfl_xor_sync(0xffffffffu, R, o);
            if (act && (lane & ((1 << seg_per_group_log2) - 1)) == 0) {
              const int g = (k0 + seg * 16) >> p.log2G;
              p.R_out[((int64_t)t * p.N + row) * p.ng + g] = R;
            }
          }
        }
      }
      // outlier channels inside this chunk, at full precision
      const int o_lo = chunk_lo[c], o_hi = chunk_lo[c + 1];
      for (int oi = o_lo + lane; oi < o_hi; oi += 32) {
        const int j = idx_s[oi] - k0;
        if (j < 0 || j >= kc_len) continue;
        const int qv = (int)reinterpret_cast<const int8_t*>(rres)[j];
        const uint32_t bit = (reinterpret_cast<const uint32_t*>(rsg)[j >> 5] >> (j & 31)) & 1u;
        uint32_t mbit = 1u;
        if (MASK) mbit = (reinterpret_cast<const uint32_t*>(rmk)[j >> 5] >> (j & 31)) & 1u;
        const float trunk = mbit ? (bit ? row_alpha : -row_alpha) : 0.0f;
        const float what = fmaf(rsc[j >> p.log2G], (float)qv, trunk);
#pragma unroll
        for (int t = 0; t < M; ++t) accU[t] = fmaf(what, xo_s[t * n_pad + oi], accU[t]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if (c == p.n_c - 1 || i == n_units - 1) {
      // the row block ends here for this CTA: reduce over the warp
#pragma unroll
      for (int t = 0; t < M; ++t) {
        for (int o = 16; o > 0; o >>= 1) {
          accP[t] += __shfl_xor_sync(0xffffffffu, accP[t], o);
          accS[t] += __shfl_xor_sync(0xffffffffu, accS[t], o);
          accF[t] += __shfl_xor_sync(0xffffffffu, accF[t], o);
          accU[t] += __shfl_xor_sync(0xffffffffu, accU[t], o);
        }
      }
      if (valid && lane == 0) {
        int T[M];
#pragma unroll
        for (int t = 0; t < M; ++t) {
          T[t] = 2 * accP[t] - accS[t];
          if (EMIT) atomicAdd(&p.T_out[(int64_t)t * p.N + row], T[t]);
        }
        const bool whole = rb * p.n_c >= u_begin && (rb + 1) * p.n_c <= u_end;
        if (whole) {
#pragma unroll
          for (int t = 0; t < M; ++t)
            p.y[(int64_t)t * p.N + row] = fmaf(sx_s[t], fmaf(row_alpha, (float)T[t], accF[t]), accU[t]);
        } else {
          // partial row: publish, the last contributor finishes in CTA order
          const int slot = (rb == u_begin / p.n_c) ? 0 : 1;
          float* part = p.ws_part + (((size_t)cta * 2 + slot) * kRowsPerBlock + warp) * (M * 4);
#pragma unroll
          for (int t = 0; t < M; ++t) {
            part[t * 4 + 0] = __int_as_float(T[t]);
            part[t * 4 + 1] = accF[t];
            part[t * 4 + 2] = accU[t];
          }
          __threadfence();
          const int b_first = unit_owner(rb * p.n_c, p);
          const int b_last = unit_owner(min((rb + 1) * p.n_c, p.U) - 1, p);
          const int prev = atomicAdd(&p.ws_cnt[row], 1);
          if (prev == b_last - b_first) {
            __threadfence();
            int Tt[M];
            float Ft[M], Ut[M];
#pragma unroll
            for (int t = 0; t < M; ++t) {
              Tt[t] = 0;
              Ft[t] = 0.0f;
              Ut[t] = 0.0f;
            }
            for (int b = b_first; b <= b_last; ++b) {
              const int sl = (rb == unit_begin(b, p) / p.n_c) ? 0 : 1;
              const float* pb = p.ws_part + (((size_t)b * 2 + sl) * kRowsPerBlock + warp) * (M * 4);
#pragma unroll
              for (int t = 0; t < M; ++t) {
                Tt[t] += __float_as_int(__ldcg(pb + t * 4 + 0));
                Ft[t] += __ldcg(pb + t * 4 + 1);
                Ut[t] += __ldcg(pb + t * 4 + 2);
              }
            }
#pragma unroll
            for (int t = 0; t < M; ++t)
              p.y[(int64_t)t * p.N + row] = fmaf(sx_s[t], fmaf(row_alpha, (float)Tt[t], Ft[t]), Ut[t]);
            p.ws_cnt[row] = 0;
          }
        }
      }
#pragma unroll
      for (int t = 0; t < M; ++t) {
        accP[t] = 0;
        accS[t] = 0;
        accF[t] = 0.0f;
        accU[t] = 0.0f;
      }
    }
  }
}

template <int M, bool MASK, bool EMIT>
cudaError_t launch_one(const Params& p, const LinearPlan& plan, bool pdl, cudaStream_t stream) {
  auto* fn = k_linear<M, MASK, EMIT>;
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
    case 1: return launch_one<1, MASK, EMIT>(p, plan, pdl, st);
    case 2: return launch_one<2, MASK, EMIT>(p, plan, pdl, st);
    case 3: return launch_one<3, MASK, EMIT>(p, plan, pdl, st);
    case 4: return launch_one<4, MASK, EMIT>(p, plan, pdl, st);
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
  pl.Kc = (int)std::min<int64_t>(kChunkMax, round_up(K16, 512));
  pl.n_c = (int)ceil_div(K16, pl.Kc);
  pl.n_rb = (int)ceil_div(w.N, kRowsPerBlock);
  const int64_t U = (int64_t)pl.n_rb * pl.n_c;
  if (U > INT32_MAX / 2) return false;
  pl.U = (int)U;
  pl.grid = (int)std::min<int64_t>(U, sm_count);
  const int R = kRowsPerBlock;
  const bool mask = w.mask_bits != nullptr;
  int off = R * pl.Kc;
  pl.off_sign = off;
  off += R * (pl.Kc / 8);
  pl.off_mask = off;
  if (mask) off += R * (pl.Kc / 8);
  pl.off_scale = off;
  off += R * (pl.Kc / w.group_size) * 4;
  pl.off_alpha = off;
  off += R * 4;
  pl.stage_bytes = (int)round_up(off, 128);
  const int n_pad = (int)round_up(n_out, 4);
  int hdr = 16 * kMaxStages + 16 + (int)round_up(pl.n_c + 1, 4) * 4 + n_pad * 4 + M * n_pad * 4 + 16;
  pl.hdr_bytes = (int)round_up(hdr, 128);
  pl.S = std::max(2, std::min(kMaxStages, kStageBudget / pl.stage_bytes));
  pl.smem_bytes = pl.hdr_bytes + pl.S * pl.stage_bytes;
  pl.ws_cnt_bytes = (size_t)round_up((int64_t)w.N * 4, 256);
  pl.ws_part_bytes = (size_t)pl.grid * 2 * R * kMaxTokensPerPass * 4 * sizeof(float);
  *plan = pl;
  return true;
}

size_t linear_workspace_bytes(const sq_packed_weight& w, int M, int sm_count) {
  LinearPlan pl;
  if (!plan_linear(w, std::min(std::max(M, 1), kMaxTokensPerPass), 0, sm_count, &pl)) return 0;
  return pl.ws_cnt_bytes + pl.ws_part_bytes;
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
  p.xq = xq;
  p.sx = sx;
  p.xout = x_out;
  p.idx = idx;
  p.n_out = n_out;
  p.y = y;
  p.T_out = T_out;
  p.R_out = R_out;
  p.ws_cnt = reinterpret_cast<int32_t*>(workspace);
  p.ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + plan.ws_cnt_bytes);
  p.status = status;
  p.Kc = plan.Kc;
  p.n_c = plan.n_c;
  p.U = plan.U;
  p.grid = plan.grid;
  p.S = plan.S;
  p.stage_bytes = plan.stage_bytes;
  p.off_sign = plan.off_sign;
  p.off_mask = plan.off_mask;
  p.off_scale = plan.off_scale;
  p.off_alpha = plan.off_alpha;
  p.hdr_bytes = plan.hdr_bytes;
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
