// sq_probe.cu -- the peaks the kernels are measured against, taken on the
// device itself.
// Tensor cores: every SM issues back-to-back tcgen05.mma of one kind on
// operands resident in its shared memory, accumulating in tensor memory,
// with nothing else running.
// HBM reads: a read-only sweep of a caller's buffer larger than L2 (the
// decode kernels only read weights; a copy also writes).
//   kind 0: kind::i8 (s8 x s8 -> s32), M = 128, N = 256, K = 32
//   kind 1: kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scales of 16), M = 128,
//           N = 256, K = 64
// Operands are a fixed pseudo-random byte pattern (every E2M1 code is finite)
// and every scale is 1.0, so the MMAs do real work.  One thread per CTA
// issues; the CTA waits (bounded) for their completion before it frees its
// tensor memory.
#include <stdint.h>

#include "sq_internal.h"
#include "sq_tcgen05.cuh"

namespace sq {
namespace {

constexpr int PM = 128, PN = 256;
constexpr int kProbeThreads = 128;
constexpr uint32_t kProbeCols = 512;  // D [0,256), scales (mxf4nvf4): A at 256, B at 264
constexpr int kBytesA = PM * 128, kBytesB = PN * 128;  // one 128-byte row each, 128-byte swizzle
// more than half of an SM's shared memory, so that no two probe CTAs share an SM
constexpr int kProbeSmem = 120 * 1024;
static_assert(kBytesA + kBytesB + 1024 + 64 <= kProbeSmem, "probe operands past the allocation");

constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PN >> 3) << 17) |
                              ((uint32_t)(PM >> 4) << 24);
constexpr uint32_t kIdescF4 = (1u << 7) | (1u << 10) | ((uint32_t)(PN >> 3) << 17) |
                              ((uint32_t)(PM >> 4) << 24);

template <int KIND>
__global__ void __launch_bounds__(kProbeThreads, 1) k_mma_peak(int iters, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + kBytesA + kBytesB);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // operands: a fixed pattern (a multiplicative hash of the byte index)
  for (int i = threadIdx.x; i < (kBytesA + kBytesB) / 4; i += kProbeThreads)
    reinterpret_cast<uint32_t*>(smem)[i] = (uint32_t)i * 2654435761u;
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_barrier_init();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) tc05::tmem_alloc(tbase, kProbeCols);
  tc05::fence_before();
  __syncthreads();
  tc05::fence_after();
  const uint32_t tmem = *tbase;
  if (KIND == 1) {
    // every scale 1.0 (UE4M3 0x38): columns 256-271 of every lane (A's 4
    // words at 256, B's 8 at 264)
    const uint32_t one = 0x38383838u;
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(
            tmem + ((uint32_t)(32 * warp) << 16) + 256),
        "r"(one)
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
  tc05::fence_before();
  __syncthreads();
  tc05::fence_after();
  if (threadIdx.x == 0) {
    const uint32_t sa = smem_u32(smem), sb = sa + kBytesA;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = tc05::sw128_desc(sa + 32 * kk), db = tc05::sw128_desc(sb + 32 * kk);
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        if (KIND == 0) {
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
              "l"(da), "l"(db), "r"(kIdescI8), "r"(acc));
        } else {
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
              "[%6], p;\n\t}" ::"r"(tmem),
              "l"(da), "l"(db), "r"(kIdescF4), "r"(acc), "r"(tmem + 256), "r"(tmem + 264));
        }
      }
    }
    tc05::mma_commit(done);
    if (!mbar_wait(done, 0u, 2000000000ull)) set_status(status, SQ_ERR_TIMEOUT);
  }
  (void)lane;
  tc05::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc05::fence_after();
    tc05::tmem_dealloc(tmem, kProbeCols);
  }
}

// ---- pure-read sweep --------------------------------------------------------------
constexpr int kReadThreads = 512, kReadUnroll = 8;
__device__ int g_read_sink;

// Every thread reads 16-byte words `stride` apart (consecutive threads,
// consecutive words: one warp load covers 512 contiguous bytes), eight loads
// in flight; the words are folded into one value so that no load is dead.
__global__ void __launch_bounds__(kReadThreads) k_read_peak(const int4* __restrict__ p, size_t n4) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  int acc = 0;
  for (; i + (kReadUnroll - 1) * stride < n4; i += kReadUnroll * stride) {
    int4 v[kReadUnroll];
#pragma unroll
    for (int u = 0; u < kReadUnroll; ++u) v[u] = ldg_nc_v4(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kReadUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n4; i += stride) {
    const int4 v = ldg_nc_v4(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (acc == 0x5EED1234) g_read_sink = acc;  // (practically never taken)
}

}  // namespace

// Bytes per second read by `iters` back-to-back sweeps of [buf, buf + bytes)
// (bytes a multiple of 16), after one warm-up sweep.
cudaError_t run_read_peak(const void* buf, size_t bytes, int iters, double* bytes_per_s,
                          cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = 4 * sms;  // four 512-thread CTAs per SM
  const int4* p = static_cast<const int4*>(buf);
  const size_t n4 = bytes / 16;
  cudaEvent_t a, b;
  if ((e = cudaEventCreate(&a)) != cudaSuccess) return e;
  if ((e = cudaEventCreate(&b)) != cudaSuccess) {
    cudaEventDestroy(a);
    return e;
  }
  k_read_peak<<<grid, kReadThreads, 0, stream>>>(p, n4);  // warm-up
  cudaEventRecord(a, stream);
  for (int it = 0; it < iters; ++it) k_read_peak<<<grid, kReadThreads, 0, stream>>>(p, n4);
  cudaEventRecord(b, stream);
  e = cudaEventSynchronize(b);
  float ms = 0.0f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (e != cudaSuccess) return e;
  *bytes_per_s = ms > 0.0f ? (double)bytes * iters / (ms * 1e-3) : 0.0;
  return cudaGetLastError();
}

// Multiply-adds x 2 per second of one probe launch (iters x 4 MMAs per SM).
cudaError_t run_mma_peak(int kind, int iters, double* ops_per_s, int32_t* status,
                         cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  auto* fn = kind == 0 ? k_mma_peak<0> : k_mma_peak<1>;
  if ((e = ensure_smem_attr((const void*)fn, kProbeSmem)) != cudaSuccess) return e;
  cudaEvent_t a, b;
  if ((e = cudaEventCreate(&a)) != cudaSuccess) return e;
  if ((e = cudaEventCreate(&b)) != cudaSuccess) {
    cudaEventDestroy(a);
    return e;
  }
  fn<<<sms, kProbeThreads, kProbeSmem, stream>>>(iters / 8 + 1, status);  // warm-up
  cudaEventRecord(a, stream);
  fn<<<sms, kProbeThreads, kProbeSmem, stream>>>(iters, status);
  cudaEventRecord(b, stream);
  e = cudaEventSynchronize(b);
  float ms = 0.0f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (e != cudaSuccess) return e;
  const double k = kind == 0 ? 32.0 : 64.0;
  const double macs = (double)sms * iters * 4.0 * PM * PN * k;
  *ops_per_s = ms > 0.0f ? 2.0 * macs / (ms * 1e-3) : 0.0;
  return cudaGetLastError();
}

}  // namespace sq
