// sq_probe.cu -- the dense tensor-core peak the prefill kernels are measured
// against, taken on the device itself: every SM issues back-to-back
// tcgen05.mma of one kind on operands resident in its shared memory,
// accumulating in tensor memory, with nothing else running.
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

}  // namespace

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
