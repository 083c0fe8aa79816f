// sq_act.cu -- outlier calibration and the per-token activation split.
//
// Page: "1-bit量化不是玄学，以往掉点是机制问题" (m.lqnn.cn/news/241359),
// section 2.2: outlier channels are found once, their indices cached and
// looked up at run time; they stay at high precision while the remaining
// channels are quantized to INT8.  Per-token runtime scale: visual guide to
// LLM quantization, "动态量化" section.  Quantizer: symmetric absmax with
// s = absmax/127 and q = round(x/s) in [-127, 127] (2048ai.net section 三.1).
//
// Built with -fmad=false.
#include <stdint.h>

#include <algorithm>

#include "sq_common.cuh"
#include "sq_internal.h"
#include "sq_quant.cuh"

namespace sq {
namespace {

constexpr int kActThreads = 1024;
constexpr int kCalThreads = 1024;

// One CTA per token; with W warps, warp w handles the 32-channel chunks
// w, w + W, ... with one channel per lane, keeping up to REGS of them in
// registers between the absmax pass and the code pass (one global round
// trip; chunks past W * REGS are read again).  A few tokens: 1024 threads
// each (latency); many: CTAs sized to the row so that several fit an SM.

__device__ __forceinline__ bool outlier_bit(const uint32_t* is_out, int j) {
  return (is_out[j >> 5] >> (j & 31)) & 1u;
}

template <int REGS>
__global__ void __launch_bounds__(kActThreads) k_quantize_act(
    const float* __restrict__ x, int M, int K, int Kx, const int32_t* __restrict__ idx, int n_out,
    int8_t* __restrict__ xq, float* __restrict__ sx, float* __restrict__ x_out,
    int32_t* __restrict__ status, int pdl) {
  extern __shared__ uint32_t is_out[];  // ceil(K/32) words
  __shared__ float warp_max[kActThreads / 32];
  if (pdl) {
    pdl_launch_dependents();
    pdl_wait();
  }
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const int nchunk = (K + 31) >> 5;
  const float* xt = x + (int64_t)t * K;
  // x into registers (issued before anything else)
  float v[REGS];
#pragma unroll
  for (int i = 0; i < REGS; ++i) {
    const int j = (warp + nw * i) * 32 + lane;
    v[i] = j < K ? __ldg(xt + j) : 0.0f;
  }
  for (int i = threadIdx.x; i < nchunk; i += blockDim.x) is_out[i] = 0u;
  __syncthreads();
  bool bad_idx = false;
  for (int i = threadIdx.x; i < n_out; i += blockDim.x) {
    const int j = idx[i];
    const bool ok = j >= 0 && j < K && (i == 0 || idx[i - 1] < j);
    bad_idx |= !ok;
    if (j >= 0 && j < K) atomicOr(&is_out[j >> 5], 1u << (j & 31));
    x_out[(int64_t)t * n_out + i] = (j >= 0 && j < K) ? xt[j] : 0.0f;
  }
  __syncthreads();

  float a = 0.0f;
  bool nonfinite = false;
  const bool big = nchunk > nw * REGS;  // more chunks than registers: re-read x
#pragma unroll
  for (int i = 0; i < REGS; ++i) {
    const int j = (warp + nw * i) * 32 + lane;
    if (j < K) {
      nonfinite |= !isfinite(v[i]);
      if (!outlier_bit(is_out, j)) a = fmaxf(a, fabsf(v[i]));
    }
  }
  if (big) {
    for (int c = warp + nw * REGS; c < nchunk; c += nw) {
      const int j = c * 32 + lane;
      if (j < K) {
        const float u = xt[j];
        nonfinite |= !isfinite(u);
        if (!outlier_bit(is_out, j)) a = fmaxf(a, fabsf(u));
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) warp_max[warp] = a;
  __syncthreads();
  a = lane < nw ? warp_max[lane] : 0.0f;
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));

  const float s = act_scale(a);
  const float rinv = act_rinv(s);
  if (threadIdx.x == 0) sx[t] = s;

  int8_t* qt = xq + (int64_t)t * Kx;
  const bool fast = quantize_fast_ok(s, a);  // one branch per token
  auto emit = [&](int c, float u) {
    const int j = c * 32 + lane;
    int q = 0;
    if (j < K && !outlier_bit(is_out, j)) q = fast ? quantize_fast(u, s, rinv) : quantize_exact(u, s, rinv);
    qt[j] = (int8_t)q;  // j < 32 * nchunk <= Kx
  };
#pragma unroll
  for (int i = 0; i < REGS; ++i) {
    const int c = warp + nw * i;
    if (c < nchunk) emit(c, v[i]);
  }
  if (big) {
    for (int c = warp + nw * REGS; c < nchunk; c += nw) {
      const int j = c * 32 + lane;
      emit(c, j < K ? xt[j] : 0.0f);
    }
  }
  // pad chunks up to the row stride (a multiple of 128 channels)
  for (int c = nchunk + warp; c < (Kx >> 5); c += nw) qt[c * 32 + lane] = 0;
  if (nonfinite) set_status(status, SQ_ERR_NONFINITE);
  if (bad_idx) set_status(status, SQ_ERR_INVALID_ARG);
}

// K % 4 == 0: the same split four channels per lane -- float4 loads, one
// nibble of the outlier bitmap and one 32-bit store of four codes per lane
// and chunk of 128 channels (a warp's 32 lanes); REGS chunks per warp held
// in registers, any further ones read again.  Same codes as k_quantize_act
// (the same quantizer decides them).
template <int REGS>
__global__ void __launch_bounds__(kActThreads) k_quantize_act4(
    const float* __restrict__ x, int M, int K, int Kx, const int32_t* __restrict__ idx, int n_out,
    int8_t* __restrict__ xq, float* __restrict__ sx, float* __restrict__ x_out,
    int32_t* __restrict__ status, int pdl) {
  extern __shared__ uint32_t is_out[];  // ceil(K/32) words
  __shared__ float warp_max[kActThreads / 32];
  if (pdl) {
    pdl_launch_dependents();
    pdl_wait();
  }
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const int K4 = K >> 2, Kx4 = Kx >> 2;
  const int nch = (K4 + 31) >> 5;  // chunks of 128 channels
  const float* xt = x + (int64_t)t * K;
  const float4* xt4 = reinterpret_cast<const float4*>(xt);
  // the first outlier entries and their values, issued with the x loads
  const int j0 = threadIdx.x < n_out ? __ldg(idx + threadIdx.x) : -1;
  const int jq0 = (threadIdx.x < n_out && threadIdx.x > 0) ? __ldg(idx + threadIdx.x - 1) : -1;
  float4 v[REGS];
#pragma unroll
  for (int i = 0; i < REGS; ++i) {
    const int j4 = (warp + nw * i) * 32 + lane;
    v[i] = j4 < K4 ? __ldg(xt4 + j4) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  const float xo0 = (j0 >= 0 && j0 < K) ? __ldg(xt + j0) : 0.0f;
  const int nwords = (K + 31) >> 5;
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) is_out[i] = 0u;
  __syncthreads();
  bool bad_idx = false;
  for (int i = threadIdx.x; i < n_out; i += blockDim.x) {
    const bool first = i < (int)blockDim.x;
    const int j = first ? j0 : idx[i];
    const int jq = first ? jq0 : idx[i - 1];
    const bool ok = j >= 0 && j < K && (i == 0 || jq < j);
    bad_idx |= !ok;
    if (j >= 0 && j < K) atomicOr(&is_out[j >> 5], 1u << (j & 31));
    x_out[(int64_t)t * n_out + i] = first ? xo0 : ((j >= 0 && j < K) ? xt[j] : 0.0f);
  }
  __syncthreads();

  float a = 0.0f;
  bool nonfinite = false;
  const bool big = nch > nw * REGS;
#pragma unroll
  for (int i = 0; i < REGS; ++i) {
    const int j4 = (warp + nw * i) * 32 + lane;
    if (j4 < K4) a = absmax4(v[i], omask_nibble(is_out, j4), a, nonfinite);
  }
  if (big) {
    for (int c = warp + nw * REGS; c < nch; c += nw) {
      const int j4 = c * 32 + lane;
      if (j4 < K4) a = absmax4(xt4[j4], omask_nibble(is_out, j4), a, nonfinite);
    }
  }
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) warp_max[warp] = a;
  __syncthreads();
  a = lane < nw ? warp_max[lane] : 0.0f;
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));

  const float s = act_scale(a);
  const float rinv = act_rinv(s);
  if (threadIdx.x == 0) sx[t] = s;
  uint32_t* qt4 = reinterpret_cast<uint32_t*>(xq + (int64_t)t * Kx);
  const bool fast = quantize_fast_ok(s, a);  // one branch per token
#pragma unroll
  for (int i = 0; i < REGS; ++i) {
    const int j4 = (warp + nw * i) * 32 + lane;
    if (j4 < K4) {
      const uint32_t om = omask_nibble(is_out, j4);
      qt4[j4] = fast ? pack_codes<true>(v[i], om, s, rinv) : pack_codes<false>(v[i], om, s, rinv);
    }
  }
  if (big) {
    for (int c = warp + nw * REGS; c < nch; c += nw) {
      const int j4 = c * 32 + lane;
      if (j4 < K4) qt4[j4] = pack_codes<false>(xt4[j4], omask_nibble(is_out, j4), s, rinv);
    }
  }
  // pad words up to the row stride (a multiple of 128 channels)
  for (int j4 = K4 + threadIdx.x; j4 < Kx4; j4 += blockDim.x) qt4[j4] = 0u;
  if (nonfinite) set_status(status, SQ_ERR_NONFINITE);
  if (bad_idx) set_status(status, SQ_ERR_INVALID_ARG);
}

// ---- calibration: per-channel max |X| over T tokens, top-k ------------------
struct Cand {
  float mag;
  int j;
};

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  return a.mag > b.mag || (a.mag == b.mag && a.j < b.j);
}

__global__ void __launch_bounds__(kCalThreads) k_calibrate(const float* __restrict__ X, int T,
                                                           int K, int k,
                                                           int32_t* __restrict__ idx_out,
                                                           int32_t* __restrict__ status) {
  extern __shared__ float mag[];  // [K] magnitudes, then [K] taken flags
  uint8_t* taken = reinterpret_cast<uint8_t*>(mag + K);
  __shared__ Cand warp_best[kCalThreads / 32];
  __shared__ int counts[kCalThreads];
  bool nonfinite = false;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    float m = 0.0f;
    for (int t = 0; t < T; ++t) {
      const float v = X[(int64_t)t * K + j];
      if (isfinite(v))
        m = fmaxf(m, fabsf(v));
      else
        nonfinite = true;
    }
    mag[j] = m;
    taken[j] = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int round = 0; round < k; ++round) {
    Cand best{-1.0f, 0x7fffffff};
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      Cand c{taken[j] ? -1.0f : mag[j], j};
      if (better(c, best)) best = c;
    }
    for (int o = 16; o > 0; o >>= 1) {
      Cand other{__shfl_xor_sync(0xffffffffu, best.mag, o), __shfl_xor_sync(0xffffffffu, best.j, o)};
      if (better(other, best)) best = other;
    }
    if (lane == 0) warp_best[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
      Cand b = warp_best[0];
      for (int w = 1; w < kCalThreads / 32; ++w)
        if (better(warp_best[w], b)) b = warp_best[w];
      taken[b.j] = 1;
    }
    __syncthreads();
  }
  // ascending compaction: thread i owns channels [i*K/n, (i+1)*K/n)
  const int n = blockDim.x;
  const int j0 = (int)((int64_t)threadIdx.x * K / n), j1 = (int)((int64_t)(threadIdx.x + 1) * K / n);
  int c = 0;
  for (int j = j0; j < j1; ++j) c += taken[j];
  counts[threadIdx.x] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < n; ++i) {
      const int v = counts[i];
      counts[i] = run;
      run += v;
    }
  }
  __syncthreads();
  int pos = counts[threadIdx.x];
  for (int j = j0; j < j1; ++j)
    if (taken[j]) idx_out[pos++] = j;
  if (nonfinite) set_status(status, SQ_ERR_NONFINITE);
}

}  // namespace

namespace {
// Register depths instantiated, and the launch shape for M tokens of K
// channels: at least 2 tokens per SM -> warps = ceil(chunks / 16) (two
// register rounds of 8 or more chunks per warp), else 1024 threads; the
// depth is the smallest instantiated one covering the row, 28 at most.
constexpr int kActDepths[] = {1, 2, 4, 8, 16, 28};

template <int REGS, bool VEC>
cudaError_t launch_act_t(const float* x, int M, int K, int Kx, const int32_t* idx, int n_out,
                         int8_t* xq, float* sx, float* x_out, int32_t* status, bool pdl,
                         int threads, size_t smem, cudaStream_t stream) {
  auto* fn = k_quantize_act<REGS>;
  if constexpr (VEC) fn = k_quantize_act4<REGS>;
  cudaError_t e = ensure_smem_attr((const void*)fn, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, x, M, K, Kx, idx, n_out, xq, sx, x_out, status, pdl ? 1 : 0);
}
}  // namespace

cudaError_t launch_quantize_act(const float* x, int M, int K, const int32_t* idx, int n_out,
                                int8_t* xq, float* sx, float* x_out, int32_t* status, bool pdl,
                                cudaStream_t stream) {
  const int Kx = (int)xq_stride_of(K);
  const size_t smem = (size_t)ceil_div(K, 32) * sizeof(uint32_t);
  // chunks per lane-column: 32 channels (scalar kernel) or 128 (K % 4 == 0)
  const bool vec = (K & 3) == 0;
  const int nchunk = (int)ceil_div(K, vec ? 128 : 32);
  DeviceInfo d;
  const int sms = current_device(&d) ? d.sm_count : 148;
  int warps = 32;
  if (M >= 2 * sms) warps = std::min(32, std::max(1, (int)ceil_div(nchunk, vec ? 4 : 16)));
  const int need = (int)ceil_div(nchunk, warps);
  int regs = kActDepths[5];
  for (int r : kActDepths)
    if (r >= need) {
      regs = r;
      break;
    }
  if (vec) regs = std::min(regs, 8);  // float4 chunks: at most 8 (32 registers) held
  const int threads = 32 * warps;
#define SQ_ACT_LAUNCH(R, V) \
  return launch_act_t<R, V>(x, M, K, Kx, idx, n_out, xq, sx, x_out, status, pdl, threads, smem, stream)
  if (vec) {
    switch (regs) {
      case 1: SQ_ACT_LAUNCH(1, true);
      case 2: SQ_ACT_LAUNCH(2, true);
      case 4: SQ_ACT_LAUNCH(4, true);
      default: SQ_ACT_LAUNCH(8, true);
    }
  }
  switch (regs) {
    case 1: SQ_ACT_LAUNCH(1, false);
    case 2: SQ_ACT_LAUNCH(2, false);
    case 4: SQ_ACT_LAUNCH(4, false);
    case 8: SQ_ACT_LAUNCH(8, false);
    case 16: SQ_ACT_LAUNCH(16, false);
    default: SQ_ACT_LAUNCH(28, false);
  }
#undef SQ_ACT_LAUNCH
}

cudaError_t launch_calibrate(const float* X, int T, int K, int k, int32_t* idx_out,
                             int32_t* status, cudaStream_t stream) {
  const size_t smem = (size_t)K * (sizeof(float) + 1);
  cudaError_t e = ensure_smem_attr((const void*)k_calibrate, (int)smem);
  if (e != cudaSuccess) return e;
  k_calibrate<<<1, kCalThreads, smem, stream>>>(X, T, K, k, idx_out, status);
  return cudaGetLastError();
}

}  // namespace sq
