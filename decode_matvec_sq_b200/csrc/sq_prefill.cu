// sq_prefill.cu -- the separated-quantization linear layer for many tokens
// (prefill) on the 5th-generation tensor cores: tcgen05.mma kind::i8 with the
// accumulators in tensor memory, operands staged by TMA.
//
// Page: "1-bit量化不是玄学，以往掉点是机制问题" (m.lqnn.cn/news/241359),
// section 2.3: the trunk product and the residual product side by side,
// summed; at prefill the activation matrix is a dense operand, so both are
// int8 GEMMs: xq [M][K] against the trunk as +-1 (0 outside the mask) bytes
// and against the residual codes.
//
// Same results as the decode kernels: exact int32 T and R_g, fp32 y.
//   CTA tile: 128 tokens (MMA M, one TMEM lane each) x 64 weight rows (MMA N),
//   looping over the 128-channel groups g (MMA K = 32, four per group).
//   Warp 0 (one lane): TMA loads of the activation codes, residual codes and
//     sign / mask words of group g into a 3-stage ring (128-byte swizzle).
//   Warps 2-3: expand the sign (and mask) bits of the stage into +-1 / 0
//     bytes, written in the same swizzled K-major layout.
//   Warp 1 (one lane): four MMAs of the residual into accumulator R[g % 2]
//     and four of the trunk into T (accumulating over all K).
//   Warps 4-7: read R[g % 2] (tcgen05.ld), promote it with the group scales
//     (F += s_g * R_g) and free the buffer; at the end read T and write
//     y = sx * (alpha * T + F) + sum_i What[r][idx_i] * x_out[i].
// Two CTAs share an SM (256 of the 512 TMEM columns each), so one CTA's
// epilogue overlaps the other's MMAs.  Every wait is bounded: a wait that
// runs out sets SQ_ERR_TIMEOUT in the status word and the CTA winds down.
// Winding down drains the asynchronous work first: the TMA producer waits
// (bounded) until every stage it requested has landed, and the MMA issuer
// commits to a last barrier and waits (bounded) until its MMAs are done, so
// no copy still writes shared memory and no MMA still writes tensor memory
// when the CTA frees it and exits.
#include <stdint.h>

#include <algorithm>

#include "sq_internal.h"
#include "sq_tcgen05.cuh"

namespace sq {
namespace {

constexpr int BM = 128;        // tokens per CTA
constexpr int BN = 64;         // weight rows per CTA
constexpr int BK = 128;        // channels per group
constexpr int kStages = 3;
constexpr int kThreads = 256;  // 8 warps
constexpr uint32_t kTmemCols = 256;  // T [0,64), R0 [64,128), R1 [128,192), R2 [192,256)
constexpr int kAccBufs = 3;          // residual accumulators: the MMAs run two groups ahead

constexpr int kBytesA = BM * BK;  // 16 KB
constexpr int kBytesB = BN * BK;  // 8 KB
constexpr int kBytesE = BN * BK;  // 8 KB
constexpr int kBytesBits = BN * 16;  // 4 words per row
constexpr int kOffA = 0, kOffB = kOffA + kBytesA, kOffE = kOffB + kBytesB;
constexpr int kOffS = kOffE + kBytesE, kOffM = kOffS + kBytesBits;
constexpr int kStageBytes = kOffM + kBytesBits;  // 34 KB, a multiple of 1024
static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");

// small shared state after the stages
struct Aux {
  uint64_t full[kStages], tready[kStages], empty[kStages];
  uint64_t accf[kAccBufs], acce[kAccBufs], tdone;
  uint64_t sready[8];  // group scales of group g written (slot g % 8)
  uint32_t tmem_base;
  int abort;
  __align__(16) float scl[8][BN];  // group scales of the CTA's rows, ring of 8 groups
  float alpha[BN];
};
constexpr int kSmemBytes = kStages * kStageBytes + (int)sizeof(Aux) + 1024;  // + alignment slack

struct Params {
  int M, N, K, nk;  // nk = ceil(K / 128) groups
  const float* alpha;
  const float* scale;
  int scale_stride;
  const int8_t* res;  // row layout, for the outlier weights
  int res_stride;
  const uint32_t* sign;
  const uint32_t* mask;
  int sign_stride;
  const float* sx;
  const float* xout;
  const int32_t* idx;
  int n_out;
  float* y;
  int32_t* T_out;
  int32_t* R_out;
  int32_t* status;
  uint64_t wait_ns;  // limit of every bounded wait
  int skip_group;    // failure injection for tests: this group's operands are never requested (-1: none)
};

// D (s32) += A (s8, K-major) * B (s8, K-major), M = 128, N = 64.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc ? 1 : 0));
}

using tc05::fence_after;
using tc05::fence_before;
using tc05::make_map;
using tc05::mma_commit;
using tc05::sw128_desc;
using tc05::tma_load_2d;
using tc05::tmem_ld32;

// int32 -> float for |r| < 2^22 (group sums are below 2^21, trunk sums below
// 2^22 for K < 33000): the integer lands in the mantissa of 1.5 * 2^23.
__device__ __forceinline__ float small_int_to_float(int r) {
  return __fsub_rn(__int_as_float(r + 0x4B400000), 12582912.0f);
}

__device__ __forceinline__ void named_sync_epi() {
  asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
}

// Waits on an mbarrier phase; on a timeout records it and asks the CTA to stop.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Aux* aux,
                                              const Params& p) {
  if (mbar_wait(bar, parity, p.wait_ns)) return true;
  set_status(p.status, SQ_ERR_TIMEOUT);
  atomicExch(&aux->abort, 1);
  return false;
}
__device__ __forceinline__ bool aborted(const Aux* aux) {
  return *reinterpret_cast<const volatile int*>(&aux->abort) != 0;
}

// +-1 (or 0 outside the mask) bytes of channels 4n .. 4n+3 from the nibble of
// sign bits (and mask bits): byte = 0x01 if b, 0xFF if not, 0 if m = 0.
template <bool MASK>
__device__ __forceinline__ uint32_t trunk_bytes(uint32_t snib, uint32_t mnib) {
  const uint32_t eb = ((snib & 0xFu) * 0x00204081u) & 0x01010101u;  // 0/1 per byte
  uint32_t pm = ~(eb * 0xFEu);                                      // 0x01 / 0xFF
  if (MASK) pm &= (((mnib & 0xFu) * 0x00204081u) & 0x01010101u) * 0xFFu;
  return pm;
}

template <bool MASK, bool EMIT>
__global__ void __launch_bounds__(kThreads, 2)
    k_prefill(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmM,
              const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Aux* aux = reinterpret_cast<Aux*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt_m = (p.M + BM - 1) / BM;
  const int m0 = (blockIdx.x % nt_m) * BM, n0 = (blockIdx.x / nt_m) * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&aux->full[s], 1);
      mbar_init(&aux->tready[s], 64);
      mbar_init(&aux->empty[s], 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&aux->accf[b], 1);
      mbar_init(&aux->acce[b], 128);
    }
    mbar_init(&aux->tdone, 1);
    for (int g = 0; g < 8; ++g) mbar_init(&aux->sready[g], 64);
    aux->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&aux->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x >= 128 && threadIdx.x < 128 + BN) {
    const int n = n0 + threadIdx.x - 128;
    aux->alpha[threadIdx.x - 128] = n < p.N ? __ldg(p.alpha + n) : 0.0f;
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = aux->tmem_base;

  if (warp == 0) {
    // ---- TMA producer
    if (lane == 0) {
      int last_use[kStages];  // the last use of each stage requested (-1: none)
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_use[s] = -1;
      for (int kb = 0; kb < p.nk; ++kb) {
        const int s = kb % kStages;
        const uint32_t use = (uint32_t)(kb / kStages);
        if (kb >= kStages && !wait_or_abort(&aux->empty[s], (use & 1u) ^ 1u, aux, p)) break;
        if (aborted(aux)) break;
        if (kb == p.skip_group) continue;  // (tests only) never requested: its waits run out
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&aux->full[s],
                              kBytesA + kBytesB + kBytesBits + (MASK ? kBytesBits : 0));
        tma_load_2d(st + kOffA, &tmA, kb * BK, m0, &aux->full[s]);
        tma_load_2d(st + kOffB, &tmB, kb * BK, n0, &aux->full[s]);
        tma_load_2d(st + kOffS, &tmS, kb * 4, n0, &aux->full[s]);
        if (MASK) tma_load_2d(st + kOffM, &tmM, kb * 4, n0, &aux->full[s]);
        last_use[s] = (int)use;
      }
      // winding down after a timeout: every requested stage must have landed
      // before the CTA's shared memory is released
      if (aborted(aux)) {
#pragma unroll
        for (int s = 0; s < kStages; ++s)
          if (last_use[s] >= 0) (void)mbar_wait(&aux->full[s], (uint32_t)last_use[s] & 1u, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      for (int kb = 0; kb < p.nk; ++kb) {
        const int s = kb % kStages, b = kb % kAccBufs;
        const uint32_t use = (uint32_t)(kb / kStages);
        if (!wait_or_abort(&aux->full[s], use & 1u, aux, p)) break;
        if (!wait_or_abort(&aux->tready[s], use & 1u, aux, p)) break;
        if (kb >= kAccBufs &&
            !wait_or_abort(&aux->acce[b], ((uint32_t)(kb / kAccBufs) & 1u) ^ 1u, aux, p))
          break;
        fence_after();
        const uint32_t st = smem_u32(smem + s * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk) {
          const uint64_t da = sw128_desc(st + kOffA + kk * 32);
          const uint64_t db = sw128_desc(st + kOffB + kk * 32);
          const uint64_t de = sw128_desc(st + kOffE + kk * 32);
          mma_i8(tmem + 64 + 64 * b, da, db, kk > 0);
          mma_i8(tmem, da, de, kb > 0 || kk > 0);
        }
        mma_commit(&aux->empty[s]);
        mma_commit(&aux->accf[b]);
      }
      mma_commit(&aux->tdone);
      // winding down after a timeout: the MMAs issued must be done before the
      // tensor memory is freed (in a normal run the epilogue waited for this)
      if (aborted(aux)) (void)mbar_wait(&aux->tdone, 0u, p.wait_ns);
    }
  } else if (warp < 4) {
    // ---- trunk expansion: one weight row per thread; the same thread puts
    // its row's group scale in the scale ring (loaded two groups ahead)
    const int r = threadIdx.x - 64;
    const bool srow = n0 + r < p.N;
    const float* srow_p = p.scale + (int64_t)(srow ? n0 + r : 0) * p.scale_stride;
    float s_cur = srow ? __ldg(srow_p) : 0.0f;
    float s_next = (srow && p.nk > 1) ? __ldg(srow_p + 1) : 0.0f;
    for (int kb = 0; kb < p.nk; ++kb) {
      const int s = kb % kStages;
      aux->scl[kb & 7][r] = s_cur;
      s_cur = s_next;
      s_next = (srow && kb + 2 < p.nk) ? __ldg(srow_p + kb + 2) : 0.0f;
      mbar_arrive(&aux->sready[kb & 7]);
      if (!wait_or_abort(&aux->full[s], (uint32_t)(kb / kStages) & 1u, aux, p)) break;
      uint8_t* st = smem + s * kStageBytes;
      const uint4 sw = *reinterpret_cast<const uint4*>(st + kOffS + r * 16);
      uint4 mw = make_uint4(0u, 0u, 0u, 0u);
      if (MASK) mw = *reinterpret_cast<const uint4*>(st + kOffM + r * 16);
      const uint32_t sv[4] = {sw.x, sw.y, sw.z, sw.w};
      const uint32_t mv[4] = {mw.x, mw.y, mw.z, mw.w};
      uint8_t* row = st + kOffE + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = channels 16c .. 16c+15
        const uint32_t s16 = sv[c >> 1] >> (16 * (c & 1));
        const uint32_t m16 = mv[c >> 1] >> (16 * (c & 1));
        uint4 v;
        v.x = trunk_bytes<MASK>(s16, m16);
        v.y = trunk_bytes<MASK>(s16 >> 4, m16 >> 4);
        v.z = trunk_bytes<MASK>(s16 >> 8, m16 >> 8);
        v.w = trunk_bytes<MASK>(s16 >> 12, m16 >> 12);
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) * 16)) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&aux->tready[s]);
    }
  } else {
    // ---- epilogue: one token (TMEM lane) per thread
    const int et = threadIdx.x - 128;
    const int lb = 32 * (warp & 3);  // TMEM lanes of this warp
    const int t = m0 + lb + lane;
    float F[BN];
#pragma unroll
    for (int n = 0; n < BN; ++n) F[n] = 0.0f;
    const int ng = p.nk;
    (void)et;
    // Whether a warp reads TMEM is decided per warp (tcgen05.ld is
    // warp-collective); after a timeout the rest is skipped.
    for (int kb = 0; kb < p.nk; ++kb) {
      const int b = kb % kAccBufs;
      const float4* scl4 = reinterpret_cast<const float4*>(aux->scl[kb & 7]);
      bool ok = !aborted(aux) &&
                wait_or_abort(&aux->sready[kb & 7], (uint32_t)(kb >> 3) & 1u, aux, p) &&
                wait_or_abort(&aux->accf[b], (uint32_t)(kb / kAccBufs) & 1u, aux, p);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        int r[32];
        tmem_ld32(tmem + ((uint32_t)lb << 16) + 64 + 64 * b + 32 * h, r);
        if (h == 1) {
          fence_before();
          mbar_arrive(&aux->acce[b]);
        }
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 sc = scl4[8 * h + i4];
          const int i = 4 * i4;
          F[32 * h + i] = fmaf(sc.x, small_int_to_float(r[i]), F[32 * h + i]);
          F[32 * h + i + 1] = fmaf(sc.y, small_int_to_float(r[i + 1]), F[32 * h + i + 1]);
          F[32 * h + i + 2] = fmaf(sc.z, small_int_to_float(r[i + 2]), F[32 * h + i + 2]);
          F[32 * h + i + 3] = fmaf(sc.w, small_int_to_float(r[i + 3]), F[32 * h + i + 3]);
        }
        if (EMIT && t < p.M) {
          for (int i = 0; i < 32; ++i) {
            const int n = n0 + 32 * h + i;
            if (n < p.N) p.R_out[((int64_t)t * p.N + n) * ng + kb] = r[i];
          }
        }
      }
    }
    bool fin = !aborted(aux) && wait_or_abort(&aux->tdone, 0u, aux, p);
    named_sync_epi();  // a timeout anywhere is now visible to all epilogue threads
    fin = fin && !aborted(aux);
    if (__any_sync(0xffffffffu, !fin)) fin = false;
    named_sync_epi();
    fin = !aborted(aux) && fin;
    if (fin) {
      fence_after();
      const float sxt = t < p.M ? __ldg(p.sx + t) : 0.0f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        int r[32];
        tmem_ld32(tmem + ((uint32_t)lb << 16) + 32 * h, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int n = 32 * h + i;
          F[n] = sxt * fmaf(aux->alpha[n], (float)r[i], F[n]);
        }
        if (EMIT && t < p.M) {
          for (int i = 0; i < 32; ++i) {
            const int n = n0 + 32 * h + i;
            if (n < p.N) p.T_out[(int64_t)t * p.N + n] = r[i];
          }
        }
      }
      // outlier channels: y += sum_i What[n][idx_i] * x_out[t][i], What from
      // the packed row (the dequantized weight); table in the free stage memory
      // Thread et builds row nn = et % 64 of the table for the outliers
      // i = et / 64 (mod 2), eight at a time: their channel indices first,
      // then all their weight words, so that each batch costs two memory
      // round trips instead of two per entry.
      float* wo = reinterpret_cast<float*>(smem);  // [64 outliers][BN]
      static_assert(BN == 64, "two epilogue threads per weight row");
      const int nn = et & (BN - 1), n = n0 + nn;
      const bool live_row = n < p.N;
      const int64_t nr = live_row ? n : 0;
      for (int i0 = 0; i0 < p.n_out; i0 += 64) {
        const int ni = min(64, p.n_out - i0);
        named_sync_epi();
        for (int ib = et >> 6; ib < ni; ib += 16) {
          int jj[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) jj[u] = ib + 2 * u < ni ? __ldg(p.idx + i0 + ib + 2 * u) : -1;
          uint32_t sg[8], mk[8];
          float sc[8];
          int rs[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const bool ok = live_row && jj[u] >= 0 && jj[u] < p.K;
            const int jc = ok ? jj[u] : 0;
            sg[u] = ok ? __ldg(p.sign + nr * p.sign_stride + (jc >> 5)) : 0u;
            mk[u] = (ok && MASK) ? __ldg(p.mask + nr * p.sign_stride + (jc >> 5)) : 0u;
            sc[u] = ok ? __ldg(p.scale + nr * p.scale_stride + (jc >> 7)) : 0.0f;
            rs[u] = ok ? (int)__ldg(p.res + nr * p.res_stride + jc) : 0;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = ib + 2 * u, j = jj[u];
            if (i >= ni) break;
            float w = 0.0f;
            if (live_row && j >= 0 && j < p.K) {
              const uint32_t bit = 1u << (j & 31);
              const bool sgn = (sg[u] & bit) != 0;
              const bool m = MASK ? (mk[u] & bit) != 0 : true;
              const float al = aux->alpha[nn];
              const float tr = m ? (sgn ? al : -al) : 0.0f;
              w = fmaf(sc[u], (float)rs[u], tr);
            }
            wo[i * BN + nn] = w;
          }
        }
        named_sync_epi();
        if (t < p.M) {
          for (int i = 0; i < ni; ++i) {
            const float xv = __ldg(p.xout + (int64_t)t * p.n_out + i0 + i);
#pragma unroll
            for (int n = 0; n < BN; ++n) F[n] = fmaf(wo[i * BN + n], xv, F[n]);
          }
        }
      }
      if (t < p.M) {
        float* yr = p.y + (int64_t)t * p.N + n0;
        if (n0 + BN <= p.N && (p.N & 3) == 0) {
#pragma unroll
          for (int n = 0; n < BN; n += 4)
            *reinterpret_cast<float4*>(yr + n) = make_float4(F[n], F[n + 1], F[n + 2], F[n + 3]);
        } else {
          for (int n = 0; n < BN; ++n)
            if (n0 + n < p.N) yr[n] = F[n];
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

template <bool MASK, bool EMIT>
cudaError_t launch_prefill_t(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& s,
                             const CUtensorMap& m, const Params& p, int grid, cudaStream_t stream) {
  auto* fn = k_prefill<MASK, EMIT>;
  cudaError_t e = ensure_smem_attr((const void*)fn, kSmemBytes);
  if (e != cudaSuccess) return e;
  fn<<<grid, kThreads, kSmemBytes, stream>>>(a, b, s, m, p);
  return cudaGetLastError();
}

}  // namespace

bool prefill_supported(const sq_packed_weight& w) {
  return w.layout == SQ_LAYOUT_ROWS && w.group_size == BK && tc05::encode_fn() != nullptr;
}

cudaError_t launch_prefill(const sq_packed_weight& w, int M, const int8_t* xq, const float* sx,
                           const float* x_out, const int32_t* idx, int n_out, float* y,
                           int32_t* T_out, int32_t* R_out, int32_t* status, cudaStream_t stream,
                           uint64_t wait_ns, int skip_group) {
  if (!prefill_supported(w) || M < 1) return cudaErrorInvalidValue;
  const int64_t K128 = xq_stride_of(w.K);
  CUtensorMap ma, mb, ms, mm;
  if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K128, (uint64_t)M,
                (uint64_t)K128, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.res_q, (uint64_t)w.res_stride,
                (uint64_t)w.N, (uint64_t)w.res_stride, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT32, w.sign_bits, (uint64_t)w.sign_stride,
                (uint64_t)w.N, (uint64_t)w.sign_stride * 4, 4, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (w.mask_bits) {
    if (!make_map(&mm, CU_TENSOR_MAP_DATA_TYPE_UINT32, w.mask_bits, (uint64_t)w.sign_stride,
                  (uint64_t)w.N, (uint64_t)w.sign_stride * 4, 4, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    mm = ms;
  }
  Params p;
  p.M = M;
  p.N = w.N;
  p.K = w.K;
  p.nk = (int)ceil_div(w.K, BK);
  p.alpha = w.alpha;
  p.scale = w.res_scale;
  p.scale_stride = w.scale_stride;
  p.res = w.res_q;
  p.res_stride = w.res_stride;
  p.sign = w.sign_bits;
  p.mask = w.mask_bits;
  p.sign_stride = w.sign_stride;
  p.sx = sx;
  p.xout = x_out;
  p.idx = idx;
  p.n_out = n_out;
  p.y = y;
  p.T_out = T_out;
  p.R_out = R_out;
  p.status = status;
  p.wait_ns = wait_ns;
  p.skip_group = skip_group;
  const int64_t grid = ceil_div(M, BM) * ceil_div(w.N, BN);
  if (grid >= INT32_MAX) return cudaErrorInvalidValue;
  const bool mask = w.mask_bits != nullptr, emit = T_out != nullptr;
  if (mask)
    return emit ? launch_prefill_t<true, true>(ma, mb, ms, mm, p, (int)grid, stream)
                : launch_prefill_t<true, false>(ma, mb, ms, mm, p, (int)grid, stream);
  return emit ? launch_prefill_t<false, true>(ma, mb, ms, mm, p, (int)grid, stream)
              : launch_prefill_t<false, false>(ma, mb, ms, mm, p, (int)grid, stream);
}

}  // namespace sq
