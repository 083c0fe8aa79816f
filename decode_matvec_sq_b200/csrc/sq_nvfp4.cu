// sq_nvfp4.cu -- the prefill path of format separation: NVFP4 weights and
// activations multiplied on the 5th-generation tensor cores with block
// scaling (tcgen05.mma kind::mxf4nvf4, 16-element UE4M3 scales).
//
// Page: the ISTA-DASLab news page on separated quantization (paragraphs 2-4):
// prefill uses the hardware's native quantized compute (NVFP4) while decode
// keeps its own low-bit weight-only format.  The page names the format
// without defining it; the reading taken is the format the Blackwell tensor
// cores consume:
//   E2M1 elements (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; sign in bit 3; two
//   per byte, the lower channel in the low nibble), blocks of 16 channels with
//   one UE4M3 scale s_b, and a binary32 second-level scale g = amax / (6*448)
//   per weight tensor and per activation row (token).
//   s_b = RNE_ue4m3(amax_b / (6 g)), q = RNE_e2m1(x / (s_b g)) saturating at
//   6, ties to the even code, +0 for a zero result; g = 0 or s_b = 0 -> 0.
//   y[t][n] = g_w g_x[t] sum_b s_w[n][b] s_x[t][b] sum_{j in b} e(qw) e(qx).
//
// Quantizer decisions are exact: the block scale rounds the binary64
// quotient amax_b / (6 g) (6 g is exact in binary64, and a quotient of a
// 24-bit by a 26-bit significand that is not a rounding midpoint lies more
// than 2^-32 of itself from one, far beyond binary64 rounding); the element
// code compares |x| with the seven E2M1 midpoints times s_b g, each product
// exact in binary64.
//
// GEMM: CTA tile 128 tokens (MMA M, one TMEM lane each) x 128 weight rows
// (MMA N), stages of 256 channels (128 bytes a row, 128-byte swizzle).
//   warp 0 (one lane): TMA of both code tiles, bulk copies of both scale
//     chunks (2 KB each) into a 3-stage ring;
//   warp 1 (one lane): per stage, tcgen05.cp of the 4 + 4 scale chunks into
//     this stage's scale columns of tensor memory, then 4 block-scaled MMAs
//     (K = 64 each) into the fp32 accumulator;
//   warps 2-5: y = g_w g_x[t] * D read back with tcgen05.ld.
// Two CTAs share an SM (256 TMEM columns each).  Every wait is bounded: a
// wait that runs out sets SQ_ERR_TIMEOUT and the CTA drains its copies and
// MMAs before it frees its tensor memory.
#include <stdint.h>

#include "sq_internal.h"
#include "sq_tcgen05.cuh"

namespace sq {
namespace {

using tc05::fence_after;
using tc05::fence_before;

constexpr int BM = 128;          // tokens per CTA (MMA M)
constexpr int BN = 128;          // weight rows per CTA (MMA N)
constexpr int kStageK = 256;     // channels per stage
constexpr int kRowBytes = kStageK / 2;  // code bytes per row per stage
constexpr int kStages = 3;
constexpr int kThreads = 192;    // 6 warps
constexpr uint32_t kTmemCols = 256;  // D [0,128); stage s scales: A at 128+32s, B at 144+32s

constexpr int kBytesA = BM * kRowBytes;  // 16 KB
constexpr int kBytesB = BN * kRowBytes;  // 16 KB
constexpr int kBytesSf = 4 * 512;        // 4 chunks of 128 rows x 4 scales
constexpr int kOffA = 0, kOffB = kBytesA, kOffSa = kOffB + kBytesB, kOffSb = kOffSa + kBytesSf;
constexpr int kStageBytes = kOffSb + kBytesSf;  // 36 KB
static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");

struct Aux {
  uint64_t full[kStages], empty[kStages], tdone;
  uint32_t tmem_base;
  int abort;
};
constexpr int kSmemBytes = kStages * kStageBytes + (int)sizeof(Aux) + 1024;

struct Params {
  int M, N, nk;  // nk = stages = K256 / 256
  int sf_chunks;  // 64-channel scale chunks per 128-row block
  const uint8_t* sfa;  // activation scale chunks
  const uint8_t* sfb;  // weight scale chunks
  const float* gx;     // [M]
  const float* gw;     // [1]
  float* y;
  int32_t* status;
  uint64_t wait_ns;
};

// D (f32) += A (E2M1, K-major) * B (E2M1, K-major) with UE4M3 block scales
// of 16; M = 128, N = 128, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t sfa,
                                        uint32_t sfb, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc ? 1 : 0), "r"(sfa), "r"(sfb));
}

// 32 rows x 16 bytes of shared memory into tensor-memory lanes 0-31 of 4
// columns, replicated into all four lane quarters.
__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

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

__global__ void __launch_bounds__(kThreads, 2)
    k_nvfp4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Aux* aux = reinterpret_cast<Aux*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt_m = (p.M + BM - 1) / BM;
  const int mt = blockIdx.x % nt_m, nt = blockIdx.x / nt_m;
  const int m0 = mt * BM, n0 = nt * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&aux->full[s], 1);
      mbar_init(&aux->empty[s], 1);
    }
    mbar_init(&aux->tdone, 1);
    aux->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tc05::tmem_alloc(&aux->tmem_base, kTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = aux->tmem_base;

  if (warp == 0) {
    // ---- producer
    if (lane == 0) {
      int last_use[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_use[s] = -1;
      const uint8_t* sfa = p.sfa + (int64_t)mt * p.sf_chunks * 512;
      const uint8_t* sfb = p.sfb + (int64_t)nt * p.sf_chunks * 512;
      for (int kb = 0; kb < p.nk; ++kb) {
        const int s = kb % kStages;
        const uint32_t use = (uint32_t)(kb / kStages);
        if (kb >= kStages && !wait_or_abort(&aux->empty[s], (use & 1u) ^ 1u, aux, p)) break;
        if (aborted(aux)) break;
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&aux->full[s], kStageBytes);
        tc05::tma_load_2d(st + kOffA, &tmA, kb * kRowBytes, m0, &aux->full[s]);
        tc05::tma_load_2d(st + kOffB, &tmB, kb * kRowBytes, n0, &aux->full[s]);
        tc05::bulk_load(st + kOffSa, sfa + (int64_t)kb * kBytesSf, kBytesSf, &aux->full[s]);
        tc05::bulk_load(st + kOffSb, sfb + (int64_t)kb * kBytesSf, kBytesSf, &aux->full[s]);
        last_use[s] = (int)use;
      }
      if (aborted(aux)) {
#pragma unroll
        for (int s = 0; s < kStages; ++s)
          if (last_use[s] >= 0) (void)mbar_wait(&aux->full[s], (uint32_t)last_use[s] & 1u, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---- scale copies and MMAs
    if (lane == 0) {
      for (int kb = 0; kb < p.nk; ++kb) {
        const int s = kb % kStages;
        const uint32_t use = (uint32_t)(kb / kStages);
        if (!wait_or_abort(&aux->full[s], use & 1u, aux, p)) break;
        fence_after();
        const uint32_t st = smem_u32(smem + s * kStageBytes);
        const uint32_t ta = tmem + 128 + 32 * s, tb = ta + 16;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          sf_copy(ta + 4 * kk, tc05::rows16_desc(st + kOffSa + 512 * kk));
          sf_copy(tb + 4 * kk, tc05::rows16_desc(st + kOffSb + 512 * kk));
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_fp4(tmem, tc05::sw128_desc(st + kOffA + 32 * kk), tc05::sw128_desc(st + kOffB + 32 * kk),
                  ta + 4 * kk, tb + 4 * kk, kb > 0 || kk > 0);
        tc05::mma_commit(&aux->empty[s]);
      }
      tc05::mma_commit(&aux->tdone);
      if (aborted(aux)) (void)mbar_wait(&aux->tdone, 0u, p.wait_ns);
    }
  } else {
    // ---- epilogue: one token (TMEM lane) per thread
    const int lb = 32 * (warp & 3);
    const int t = m0 + lb + lane;
    bool ok = wait_or_abort(&aux->tdone, 0u, aux, p);
    ok = __all_sync(0xffffffffu, ok) && !aborted(aux);
    if (ok) {
      fence_after();
      const float sc = (t < p.M ? __ldg(p.gx + t) : 0.0f) * __ldg(p.gw);
      float* yr = p.y + (int64_t)t * p.N + n0;
      const bool full_row = n0 + BN <= p.N && (p.N & 3) == 0;
#pragma unroll
      for (int h = 0; h < BN / 32; ++h) {
        int r[32];
        tc05::tmem_ld32(tmem + ((uint32_t)lb << 16) + 32 * h, r);
        if (t < p.M) {
          if (full_row) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(yr + 32 * h + i) =
                  make_float4(sc * __int_as_float(r[i]), sc * __int_as_float(r[i + 1]),
                              sc * __int_as_float(r[i + 2]), sc * __int_as_float(r[i + 3]));
          } else {
            for (int i = 0; i < 32; ++i)
              if (n0 + 32 * h + i < p.N) yr[32 * h + i] = sc * __int_as_float(r[i]);
          }
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tc05::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- quantizers ------------------------------------------------------------------

// Nearest UE4M3 code of q >= 0 (a binary64 value), ties to the even code,
// saturating at 448 (code 126).
__device__ __forceinline__ uint32_t ue4m3_rne(double q) {
  if (!(q > 0.0)) return 0u;
  if (q >= 448.0) return 126u;
  if (q < 0.015625) return (uint32_t)rint(q * 512.0);  // subnormals m * 2^-9 (8 = 2^-6)
  const uint64_t bits = (uint64_t)__double_as_longlong(q);
  int e = (int)((bits >> 52) & 0x7FF) - 1023;  // -6 .. 8
  const uint64_t man = bits & ((1ull << 52) - 1);
  uint32_t m = (uint32_t)(man >> 49);
  const uint64_t rem = man & ((1ull << 49) - 1), half = 1ull << 48;
  if (rem > half || (rem == half && (m & 1u))) ++m;
  if (m == 8u) {
    m = 0u;
    ++e;
  }
  const uint32_t code = ((uint32_t)(e + 7) << 3) | m;
  return code > 126u ? 126u : code;
}

__device__ __forceinline__ double ue4m3_val(uint32_t c) {
  const int e = (int)(c >> 3), m = (int)(c & 7u);
  return e == 0 ? (double)m * 0x1p-9 : ldexp(1.0 + (double)m * 0.125, e - 7);
}

// E2M1 code of x against the step s_b * g: the number of midpoints below
// |x| (a midpoint reached exactly counts when the code above it is even).
struct E2m1Thresholds {
  double t[7];
};
__device__ __forceinline__ E2m1Thresholds e2m1_thresholds(double step) {
  E2m1Thresholds th;
  th.t[0] = 0.25 * step;
  th.t[1] = 0.75 * step;
  th.t[2] = 1.25 * step;
  th.t[3] = 1.75 * step;
  th.t[4] = 2.5 * step;
  th.t[5] = 3.5 * step;
  th.t[6] = 5.0 * step;
  return th;
}
__device__ __forceinline__ uint32_t e2m1_code(float x, const E2m1Thresholds& th) {
  const double a = fabs((double)x);
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) c += (i & 1) ? (a >= th.t[i] ? 1u : 0u) : (a > th.t[i] ? 1u : 0u);
  return (c != 0u && x < 0.0f) ? (c | 8u) : c;
}

// Byte offset of the scale of (row r, 16-channel block b) in the chunked
// layout: chunk (r / 128, b / 4) of 512 bytes, then row r % 32 at 16 bytes,
// word (r % 128) / 32, byte b % 4.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int sf_chunks) {
  return ((r >> 7) * sf_chunks + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

__device__ __forceinline__ float absmax_reduce(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  v = red[0];
  __syncthreads();
  return v;
}

// amax of a whole tensor: atomicMax on the bit pattern of |x| (non-negative
// floats order like their bits).  Non-finite entries set SQ_ERR_NONFINITE.
__global__ void k_nvfp4_amax(const float* __restrict__ X, int64_t n, uint32_t* amax_bits,
                             int32_t* status) {
  __shared__ float red[32];
  float a = 0.0f;
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = __ldg(X + i);
    if (!isfinite(v)) bad = true;
    a = fmaxf(a, fabsf(v));
  }
  if (bad) set_status(status, SQ_ERR_NONFINITE);
  a = absmax_reduce(a, red);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(a));
}

// One CTA per row (rows_pad of them): every 16-channel block of the row up to
// K256.  PER_ROW: g from the row's own amax (written to g[r]); else g from
// the tensor amax in amax_bits (written to g[0] by CTA 0).
template <bool PER_ROW>
__global__ void __launch_bounds__(256) k_nvfp4_quantize(const float* __restrict__ X, int rows, int K,
                                                        int code_stride, int sf_chunks,
                                                        uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales, float* g,
                                                        const uint32_t* amax_bits, int32_t* status) {
  __shared__ float red[32];
  const int r = blockIdx.x;
  const bool live = r < rows;
  const float* x = X + (int64_t)(live ? r : 0) * K;
  const int nb = code_stride / 8;  // 16-channel blocks up to K256
  float gr;
  if (PER_ROW) {
    float a = 0.0f;
    bool bad = false;
    if (live)
      for (int j = threadIdx.x; j < K; j += blockDim.x) {
        const float v = __ldg(x + j);
        if (!isfinite(v)) bad = true;
        a = fmaxf(a, fabsf(v));
      }
    if (bad) set_status(status, SQ_ERR_NONFINITE);
    a = absmax_reduce(a, red);
    gr = live ? __double2float_rn((double)a / 2688.0) : 0.0f;
    if (threadIdx.x == 0) g[r] = gr;
  } else {
    gr = __double2float_rn((double)__uint_as_float(*amax_bits) / 2688.0);
    if (r == 0 && threadIdx.x == 0) g[0] = gr;
  }
  const double gd = (double)gr;
  uint8_t* crow = codes + (int64_t)r * code_stride;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    const int j0 = 16 * b;
    float v[16];
    if (live && j0 + 16 <= K && (K & 3) == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(x + j0) + i);
        v[4 * i] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = (live && j0 + i < K) ? __ldg(x + j0 + i) : 0.0f;
    }
    float ab = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) ab = fmaxf(ab, fabsf(v[i]));
    const uint32_t sc = gr == 0.0f ? 0u : ue4m3_rne((double)ab / (6.0 * gd));
    const double step = ue4m3_val(sc) * gd;
    uint32_t w0 = 0u, w1 = 0u;
    if (step != 0.0) {
      const E2m1Thresholds th = e2m1_thresholds(step);
#pragma unroll
      for (int i = 0; i < 8; ++i) w0 |= e2m1_code(v[i], th) << (4 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i) w1 |= e2m1_code(v[8 + i], th) << (4 * i);
    }
    *reinterpret_cast<uint2*>(crow + 8 * b) = make_uint2(w0, w1);
    scales[sf_offset(r, b, sf_chunks)] = (uint8_t)sc;
  }
}

}  // namespace

cudaError_t launch_nvfp4_quantize(const float* X, const sq_nvfp4_matrix& out, int32_t* status,
                                  cudaStream_t stream) {
  const int nb = out.code_stride / 8;
  const int threads = nb >= 256 ? 256 : (nb >= 128 ? 128 : 64);
  if (out.per_row) {
    k_nvfp4_quantize<true><<<out.rows_pad, threads, 0, stream>>>(
        X, out.rows, out.K, out.code_stride, out.sf_chunks, out.codes, out.scales, out.g, nullptr,
        status);
    return cudaGetLastError();
  }
  uint32_t* amax = reinterpret_cast<uint32_t*>(out.g + 1);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)out.rows * out.K;
  const int64_t want = (n + 255) / 256;
  const int grid = (int)(want < 4096 ? want : 4096);
  k_nvfp4_amax<<<grid, 256, 0, stream>>>(X, n, amax, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_nvfp4_quantize<false><<<out.rows_pad, threads, 0, stream>>>(
      X, out.rows, out.K, out.code_stride, out.sf_chunks, out.codes, out.scales, out.g, amax,
      status);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_gemm(const sq_nvfp4_matrix& w, const sq_nvfp4_matrix& x, float* y,
                              int32_t* status, cudaStream_t stream, uint64_t wait_ns) {
  if (w.K != x.K || w.code_stride != x.code_stride || w.per_row || !x.per_row)
    return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!tc05::make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, x.codes, (uint64_t)x.code_stride,
                      (uint64_t)x.rows_pad, (uint64_t)x.code_stride, kRowBytes, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tc05::make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)w.code_stride,
                      (uint64_t)w.rows_pad, (uint64_t)w.code_stride, kRowBytes, BN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Params p;
  p.M = x.rows;
  p.N = w.rows;
  p.nk = w.code_stride / kRowBytes;
  p.sf_chunks = w.sf_chunks;
  p.sfa = x.scales;
  p.sfb = w.scales;
  p.gx = x.g;
  p.gw = w.g;
  p.y = y;
  p.status = status;
  p.wait_ns = wait_ns;
  const int64_t grid = (int64_t)(x.rows_pad / BM) * (w.rows_pad / BN);
  if (grid < 1 || grid >= INT32_MAX) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr((const void*)k_nvfp4_gemm, kSmemBytes);
  if (e != cudaSuccess) return e;
  k_nvfp4_gemm<<<(int)grid, kThreads, kSmemBytes, stream>>>(ma, mb, p);
  return cudaGetLastError();
}

}  // namespace sq
