// sq_pack.cu -- offline decomposition of W into the packed separated form.
//
// Page: "1-bit量化不是玄学，以往掉点是机制问题" (m.lqnn.cn/news/241359):
//   section 2.1  W ~ alpha*sign(W) + W_res,  W_res = W - alpha*sign(W),
//                residual re-quantized to 8 bits; trunk limited to |W| > threshold;
//   section 5.2  threshold from a percentile of |W|;
//   section 5.3  the split is done once, offline, and reused by every inference;
//   section 6.2  one scale and one threshold per output row.
// Quantizer: symmetric absmax, [-127, 127], s = absmax/127, q = round(r/s)
// (visual guide "对称量化以零为中心"; 2048ai.net section 三.1).
//
// Built with -fmad=false: every floating-point step below is a single IEEE
// operation in a fixed order, so the results are identical to any other
// implementation of the same sequence (binary64 sum of |W| in ascending
// channel order, one binary64 division for alpha and for each quotient).
#include <stdint.h>

#include "sq_common.cuh"
#include "sq_internal.h"
#include "sq_layout.h"

namespace sq {
namespace {

constexpr int kPackRows = 128;  // rows per CTA, one thread per row
constexpr int kTile = 32;       // columns per shared-memory tile

// ---- per-row nearest-rank threshold (MSB-first radix select) ---------------
// tau_r = the rank-th smallest |W[r][:]|, rank = ceil(P*K/100).  |W| as the
// float's bit pattern with the sign bit cleared orders like the value.
__global__ void __launch_bounds__(256) k_threshold(const float* __restrict__ W, int N, int K,
                                                   int P, float* __restrict__ tau_out) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_remaining;
  const int row = blockIdx.x;
  if (row >= N) return;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(W + (int64_t)row * K);
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_remaining = (uint32_t)(((int64_t)P * K + 99) / 100);
  }
  uint32_t hi_mask = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      uint32_t key = __ldg(w + j) & 0x7FFFFFFFu;
      if ((key & hi_mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t rem = s_remaining, cum = 0;
      int b = 0;
      for (; b < 255; ++b) {
        if (cum + hist[b] >= rem) break;
        cum += hist[b];
      }
      s_remaining = rem - cum;
      s_prefix = prefix | ((uint32_t)b << shift);
    }
    hi_mask |= 0xFFu << shift;
    __syncthreads();
  }
  if (threadIdx.x == 0) tau_out[row] = __uint_as_float(s_prefix);
}

__device__ __forceinline__ int quantize_q(double r, float s) {
  if (s == 0.0f) return 0;
  double t = r / (double)s;  // IEEE binary64 division
  double q = round(t);       // half away from zero
  q = q > 127.0 ? 127.0 : q;
  q = q < -127.0 ? -127.0 : q;
  return (int)q;
}

// Loads columns [c0, c0 + ncols) of rows [r0, r0 + kPackRows) into tile[row][col].
__device__ __forceinline__ void load_tile(float* tile, int pitch, const float* __restrict__ W,
                                          int N, int K, int r0, int c0, int ncols) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int rr = warp; rr < kPackRows; rr += nwarps) {
    const int row = r0 + rr;
    for (int cc = lane; cc < ncols; cc += 32) {
      const int col = c0 + cc;
      tile[rr * pitch + cc] = (row < N && col < K) ? __ldg(W + (int64_t)row * K + col) : 0.0f;
    }
  }
}

// ---- sign / mask bitplanes, alpha, residual codes and group scales --------
// One thread per row.  TILED writes SQ_LAYOUT_TILES (rows padded to a
// multiple of 16 and channels to a multiple of 128, pads zero); otherwise
// SQ_LAYOUT_ROWS.  ASYM (tiled): asymmetric residual groups with their own
// min / max, scale and zero-point (SQ_LAYOUT_TILES_ASYM).
template <bool TILED, bool ASYM>
__global__ void __launch_bounds__(kPackRows) k_pack(const float* __restrict__ W, int N, int K,
                                                    int P, int G, sq_packed_weight pw,
                                                    int32_t* __restrict__ status) {
  extern __shared__ float tile[];  // [kPackRows][G + 1]
  const int r0 = blockIdx.x * kPackRows;
  const int row = r0 + threadIdx.x;
  const bool valid = row < N;  // a row of W
  // rows written: the rows of W, plus the zero pad rows of the tiled layout
  const bool live = TILED ? row < (int)tiles_rows(N) : valid;
  const int Kp = TILED ? (int)tiles_cols(K) : K;  // channels written
  const int tpr = Kp / kTileK;                    // tiles per row block (tiled)
  const int nwords = (K + 31) / 32;
  const int ng = (K + G - 1) / G;
  const float tau = (valid && P > 0) ? pw.alpha[row] : -1.0f;  // k_threshold wrote it here
  bool nonfinite = false;

  auto store_bits = [&](uint32_t* base, int word, uint32_t bits) {
    if (TILED)
      base[tiled_bits_word(row, word, tpr)] = tiled_bits_from_row_order(bits);
    else
      base[(int64_t)row * pw.sign_stride + word] = bits;
  };

  // pass 1: bits, trunk sum, count
  double sum = 0.0;
  int64_t cnt = 0;
  const int pitch1 = kTile + 1;
  for (int c0 = 0; c0 < Kp; c0 += kTile) {
    if (c0 < K) load_tile(tile, pitch1, W, N, K, r0, c0, kTile);
    __syncthreads();
    if (live) {
      uint32_t sbits = 0, mbits = 0;
      const int ncols = valid ? max(0, min(kTile, K - c0)) : 0;
      for (int j = 0; j < ncols; ++j) {
        const float v = tile[threadIdx.x * pitch1 + j];
        nonfinite |= !isfinite(v);
        if (v >= 0.0f) sbits |= 1u << j;
        const bool m = P < 0 ? true : (fabsf(v) > tau);
        if (m) {
          mbits |= 1u << j;
          sum += fabs((double)v);
          cnt += 1;
        }
      }
      store_bits(pw.sign_bits, c0 / 32, sbits);
      if (pw.mask_bits) store_bits(pw.mask_bits, c0 / 32, mbits);
    }
    __syncthreads();
  }
  float alpha = 0.0f;
  if (valid) alpha = cnt ? (float)(sum / (double)cnt) : 0.0f;
  if (!TILED && valid) {
    for (int w = nwords; w < pw.sign_stride; ++w) {
      pw.sign_bits[(int64_t)row * pw.sign_stride + w] = 0u;
      if (pw.mask_bits) pw.mask_bits[(int64_t)row * pw.sign_stride + w] = 0u;
    }
  }
  __syncthreads();  // every thread has read its tau before alpha overwrites it
  if (live) pw.alpha[row] = alpha;

  // pass 2: residual per group, absmax scale, codes
  const int pitch2 = G + 1;
  for (int g = 0; g < ng; ++g) {
    const int c0 = g * G;
    load_tile(tile, pitch2, W, N, K, r0, c0, G);
    __syncthreads();
    if (live && ASYM) {
      // asymmetric group: s = float((hi - lo) / 255), z = round(-lo/s - 128),
      // code = clip(round(r/s + z), -128, 127), all binary64
      const int ncols = valid ? min(G, K - c0) : 0;
      const float* t = tile + threadIdx.x * pitch2;
      auto resid = [&](int j) {
        const float v = t[j];
        const bool m = P < 0 ? true : (fabsf(v) > tau);
        const double tr = m ? (v >= 0.0f ? (double)alpha : -(double)alpha) : 0.0;
        return (double)v - tr;
      };
      double lo = 0.0, hi = 0.0;
      for (int j = 0; j < ncols; ++j) {
        const double r = resid(j);
        if (j == 0 || r < lo) lo = r;
        if (j == 0 || r > hi) hi = r;
      }
      const float s = ncols > 0 ? (float)((hi - lo) / 255.0) : 0.0f;
      const int32_t z = s == 0.0f ? 0 : (int32_t)round(-lo / (double)s - 128.0);
      pw.res_scale[tiled_scale_index(row, g, tpr)] = s;
      pw.res_zero[tiled_scale_index(row, g, tpr)] = z;
      for (int j0 = 0; j0 < G; j0 += 4) {
        uint32_t word = 0;
        for (int j = j0; j < j0 + 4 && j < ncols; ++j) {
          int q = 0;
          if (s != 0.0f) {
            double v = round(resid(j) / (double)s + (double)z);
            v = v > 127.0 ? 127.0 : v;
            v = v < -128.0 ? -128.0 : v;
            q = (int)v;
          }
          word |= ((uint32_t)(uint8_t)(int8_t)q) << (8 * (j - j0));
        }
        *reinterpret_cast<uint32_t*>(pw.res_q + tiled_code_offset(row, c0 + j0, tpr)) = word;
      }
    } else if (live) {
      const int ncols = valid ? min(G, K - c0) : 0;
      const float* t = tile + threadIdx.x * pitch2;
      double a = 0.0;
      for (int j = 0; j < ncols; ++j) {
        const float v = t[j];
        const bool m = P < 0 ? true : (fabsf(v) > tau);
        const double tr = m ? (v >= 0.0f ? (double)alpha : -(double)alpha) : 0.0;
        const double r = (double)v - tr;
        a = fabs(r) > a ? fabs(r) : a;
      }
      const float s = (float)(a / 127.0);
      if (TILED)
        pw.res_scale[tiled_scale_index(row, g, tpr)] = s;
      else
        pw.res_scale[(int64_t)row * pw.scale_stride + g] = s;
      // tiled: whole 128-channel groups (codes past K are 0)
      const int nwr = TILED ? G : ncols;
      for (int j0 = 0; j0 < nwr; j0 += 4) {
        uint32_t word = 0;
        for (int j = j0; j < j0 + 4 && j < ncols; ++j) {
          const float v = t[j];
          const bool m = P < 0 ? true : (fabsf(v) > tau);
          const double tr = m ? (v >= 0.0f ? (double)alpha : -(double)alpha) : 0.0;
          const int q = quantize_q((double)v - tr, s);
          word |= ((uint32_t)(uint8_t)(int8_t)q) << (8 * (j - j0));
        }
        if (TILED)
          *reinterpret_cast<uint32_t*>(pw.res_q + tiled_code_offset(row, c0 + j0, tpr)) = word;
        else
          *reinterpret_cast<uint32_t*>(pw.res_q + (int64_t)row * pw.res_stride + c0 + j0) = word;
      }
    }
    __syncthreads();
  }
  if (!TILED && valid) {
    // pads: codes K..res_stride (the word loop above already covered up to
    // roundup(K, 4)), scales ng..scale_stride
    int8_t* qrow = pw.res_q + (int64_t)row * pw.res_stride;
    for (int j = (K + 3) / 4 * 4; j < pw.res_stride; j += 4)
      *reinterpret_cast<uint32_t*>(qrow + j) = 0u;
    for (int g = ng; g < pw.scale_stride; ++g)
      pw.res_scale[(int64_t)row * pw.scale_stride + g] = 0.0f;
  }
  if (valid && nonfinite) set_status(status, SQ_ERR_NONFINITE);
}

// ---- sparse residual (SQ_LAYOUT_TILES_SPARSE) -----------------------------------
// m.lqnn.cn section 3.3: residual entries near zero are dropped and the rest
// stored sparsely.  Over a tiled decomposition already written by k_pack
// (sign / mask bits, alpha, dense codes): one CTA per (padded) row re-forms
// r in binary64 exactly as k_pack does, finds theta_r = the rank-th smallest
// |r| (rank = ceil(Ps*K/100)) by an MSB-first radix select on the binary64
// bit patterns (non-negative doubles order like their bits), keeps |r| >
// theta_r and re-quantizes every group from its kept entries.
__global__ void __launch_bounds__(256) k_sparse_residual(const float* __restrict__ W, int N, int K,
                                                         int Ps, sq_packed_weight pw) {
  __shared__ uint32_t hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ uint32_t s_remaining;
  const int row = blockIdx.x;
  const int tpr = (int)(tiles_cols(K) / kTileK);
  const int nw = tpr * 4;  // 32-channel words of a padded row
  if (row >= N) {
    // pad rows of the tiled layout: nothing kept (their codes and scales are 0)
    for (int w = threadIdx.x; w < nw; w += blockDim.x) pw.keep_bits[tiled_bits_word(row, w, tpr)] = 0u;
    return;
  }
  const float alpha = pw.alpha[row];
  const float* wr = W + (int64_t)row * K;
  auto resid = [&](int j) -> double {
    const float v = __ldg(wr + j);
    bool m = true;
    if (pw.mask_bits) m = (pw.mask_bits[tiled_bits_word(row, j >> 5, tpr)] >> tiled_bit_of(j & 31)) & 1u;
    const double tr = m ? (v >= 0.0f ? (double)alpha : -(double)alpha) : 0.0;
    return (double)v - tr;
  };
  if (threadIdx.x == 0) {
    s_prefix = 0ull;
    s_remaining = (uint32_t)(((int64_t)Ps * K + 99) / 100);
  }
  unsigned long long hi_mask = 0ull;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      const unsigned long long key = (unsigned long long)__double_as_longlong(fabs(resid(j)));
      if ((key & hi_mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFull], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t rem = s_remaining, cum = 0;
      int b = 0;
      for (; b < 255; ++b) {
        if (cum + hist[b] >= rem) break;
        cum += hist[b];
      }
      s_remaining = rem - cum;
      s_prefix = prefix | ((unsigned long long)b << shift);
    }
    hi_mask |= 0xFFull << shift;
    __syncthreads();
  }
  const double theta = __longlong_as_double((long long)s_prefix);
  // groups of 128 channels: scale from the kept entries, codes of the kept ones
  for (int g = threadIdx.x; g < tpr; g += blockDim.x) {
    const int c0 = g * kTileK, c1 = min(K, c0 + kTileK);
    double a = 0.0;
    for (int j = c0; j < c1; ++j) {
      const double r = resid(j);
      if (fabs(r) > theta) a = fabs(r) > a ? fabs(r) : a;
    }
    const float sc = (float)(a / 127.0);
    pw.res_scale[tiled_scale_index(row, g, tpr)] = sc;
    for (int j0 = c0; j0 < c0 + kTileK; j0 += 4) {
      uint32_t word = 0;
      for (int j = j0; j < j0 + 4 && j < c1; ++j) {
        const double r = resid(j);
        const int q = fabs(r) > theta ? quantize_q(r, sc) : 0;
        word |= ((uint32_t)(uint8_t)(int8_t)q) << (8 * (j - j0));
      }
      *reinterpret_cast<uint32_t*>(pw.res_q + tiled_code_offset(row, j0, tpr)) = word;
    }
  }
  // keep bits, tiled order
  for (int w = threadIdx.x; w < nw; w += blockDim.x) {
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b) {
      const int j = 32 * w + b;
      if (j < K && fabs(resid(j)) > theta) bits |= 1u << b;
    }
    pw.keep_bits[tiled_bits_word(row, w, tpr)] = tiled_bits_from_row_order(bits);
  }
}

// Packs each tile's kept codes at the start of its 2048-byte slot, one warp
// per tile: lane L in order, row r0's then row r1's kept codes in ascending
// channel order, zero padded to 16 bytes; res_bytes[t] = the padded size.
// Every lane reads its 64 dense bytes before any lane writes (in place).
__global__ void __launch_bounds__(256) k_sparse_compact(int T, sq_packed_weight pw) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const int64_t lt = (int64_t)t * 32 + lane;
  const uint32_t k0 = pw.keep_bits[lt * 2], k1 = pw.keep_bits[lt * 2 + 1];
  uint32_t q[16];
  const uint4* src = reinterpret_cast<const uint4*>(pw.res_q + lt * 64);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 v = src[m];
    q[4 * m] = v.x;
    q[4 * m + 1] = v.y;
    q[4 * m + 2] = v.z;
    q[4 * m + 3] = v.w;
  }
  const int n = __popc(k0) + __popc(k1);
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  __syncwarp();
  uint8_t* dst = reinterpret_cast<uint8_t*>(pw.res_q) + (int64_t)t * 2048;
  int pos = incl - n;
  for (int R = 0; R < 2; ++R) {
    const uint32_t kb = R ? k1 : k0;
    for (int w = 0; w < 8; ++w) {
      // channels 4w .. 4w+3 of the lane's 32: keep bits 8c + w
      const uint32_t nib = (((kb >> w) & 0x01010101u) * 0x01020408u) >> 24;
      const uint32_t word = q[4 * (w >> 1) + 2 * (w & 1) + R];
      for (int c = 0; c < 4; ++c)
        if ((nib >> c) & 1u) dst[pos++] = (uint8_t)(word >> (8 * c));
    }
  }
  const int padded = (total + 15) & ~15;
  for (int b = total + lane; b < padded; b += 32) dst[b] = 0;
  if (lane == 0) pw.res_bytes[t] = padded;
}

// ---- per-layer fallback measure -------------------------------------------------
// m.lqnn.cn section 2.3 (last paragraph): a layer that gains nothing from the
// split falls back to plain 8-bit.  One thread per row: the squared
// reconstruction error of the packed weight (What from its own arrays) and
// of plain symmetric INT8 groups of W, binary64, channels ascending; then one
// thread sums the rows in order.
template <bool TILED, bool ASYM>
__global__ void __launch_bounds__(128) k_row_errors(const float* __restrict__ W, sq_packed_weight pw,
                                                    double* __restrict__ scratch) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  const int N = pw.N, K = pw.K, G = pw.group_size;
  if (row >= N) return;
  const int tpr = (int)(tiles_cols(K) / kTileK);
  const float* wr = W + (int64_t)row * K;
  const double al = (double)pw.alpha[row];
  double e = 0.0;
  for (int j = 0; j < K; ++j) {
    const int g = j / G;
    uint32_t sw, mw = 1u;
    int bit;
    int64_t ci, si;
    if (TILED) {
      const int64_t wi = tiled_bits_word(row, j >> 5, tpr);
      bit = tiled_bit_of(j & 31);
      sw = pw.sign_bits[wi];
      if (pw.mask_bits) mw = pw.mask_bits[wi];
      ci = tiled_code_offset(row, j, tpr);
      si = tiled_scale_index(row, g, tpr);
    } else {
      const int64_t wi = (int64_t)row * pw.sign_stride + (j >> 5);
      bit = j & 31;
      sw = pw.sign_bits[wi];
      if (pw.mask_bits) mw = pw.mask_bits[wi];
      ci = (int64_t)row * pw.res_stride + j;
      si = (int64_t)row * pw.scale_stride + g;
    }
    const bool m = pw.mask_bits ? ((mw >> bit) & 1u) != 0 : true;
    const bool b = ((sw >> bit) & 1u) != 0;
    const double t = m ? (b ? al : -al) : 0.0;
    const int64_t z = ASYM ? (int64_t)pw.res_zero[si] : 0;
    const double what = t + (double)pw.res_scale[si] * (double)((int64_t)pw.res_q[ci] - z);
    const double d = (double)__ldg(wr + j) - what;
    e += d * d;
  }
  double ep = 0.0;
  for (int j0 = 0; j0 < K; j0 += G) {
    const int j1 = min(K, j0 + G);
    double a = 0.0;
    for (int j = j0; j < j1; ++j) {
      const double v = fabs((double)__ldg(wr + j));
      a = v > a ? v : a;
    }
    const float sg = (float)(a / 127.0);
    for (int j = j0; j < j1; ++j) {
      const double w = (double)__ldg(wr + j);
      const double d = w - (double)sg * (double)quantize_q(w, sg);
      ep += d * d;
    }
  }
  scratch[row] = e;
  scratch[N + row] = ep;
}

__global__ void k_sum_errors(const double* __restrict__ scratch, int N, double* __restrict__ err) {
  if (threadIdx.x != 0) return;
  double a = 0.0, b = 0.0;
  for (int r = 0; r < N; ++r) a += scratch[r];
  for (int r = 0; r < N; ++r) b += scratch[N + r];
  err[0] = a;
  err[1] = b;
}

}  // namespace

cudaError_t launch_residual_errors(const float* W, const sq_packed_weight& w, double* err,
                                   double* scratch, int32_t* status, cudaStream_t stream) {
  (void)status;
  const int blocks = (int)ceil_div(w.N, 128);
  if (w.layout == SQ_LAYOUT_TILES_ASYM)
    k_row_errors<true, true><<<blocks, 128, 0, stream>>>(W, w, scratch);
  else if (w.layout == SQ_LAYOUT_TILES)
    k_row_errors<true, false><<<blocks, 128, 0, stream>>>(W, w, scratch);
  else
    k_row_errors<false, false><<<blocks, 128, 0, stream>>>(W, w, scratch);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_sum_errors<<<1, 32, 0, stream>>>(scratch, w.N, err);
  return cudaGetLastError();
}

cudaError_t launch_sparsify_residual(const float* W, int N, int K, int Ps, const sq_packed_weight& pw,
                                     cudaStream_t stream) {
  const int64_t rows = tiles_rows(N);
  k_sparse_residual<<<(int)rows, 256, 0, stream>>>(W, N, K, Ps, pw);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t T = rows / kTileRows * (tiles_cols(K) / kTileK);
  k_sparse_compact<<<(int)ceil_div(T, 8), 256, 0, stream>>>((int)T, pw);
  return cudaGetLastError();
}

cudaError_t launch_decompose_pack(const float* W, int N, int K, int P, const sq_packed_weight& pw,
                                  int32_t* status, cudaStream_t stream) {
  if (P > 0) {
    k_threshold<<<N, 256, 0, stream>>>(W, N, K, P, pw.alpha);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int G = pw.group_size;
  const bool asym = pw.layout == SQ_LAYOUT_TILES_ASYM;
  const bool tiled = pw.layout == SQ_LAYOUT_TILES || asym;
  const size_t smem = (size_t)kPackRows * (G + 1) * sizeof(float);
  const void* fn = asym ? (const void*)k_pack<true, true>
                        : tiled ? (const void*)k_pack<true, false> : (const void*)k_pack<false, false>;
  cudaError_t e = ensure_smem_attr(fn, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t rows = tiled ? tiles_rows(N) : N;
  const int blocks = (int)ceil_div(rows, kPackRows);
  if (asym)
    k_pack<true, true><<<blocks, kPackRows, smem, stream>>>(W, N, K, P, G, pw, status);
  else if (tiled)
    k_pack<true, false><<<blocks, kPackRows, smem, stream>>>(W, N, K, P, G, pw, status);
  else
    k_pack<false, false><<<blocks, kPackRows, smem, stream>>>(W, N, K, P, G, pw, status);
  return cudaGetLastError();
}

}  // namespace sq
