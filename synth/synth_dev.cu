// synth_dev.cu -- device generator for the seeded synthetic inputs.
//
// Same definition as synth/__init__.py (SplitMix64 counter stream, Laplace by
// inverse CDF, Box-Muller normals, series log and cosine), written here with
// explicitly rounded binary64 intrinsics (__dadd_rn, __dmul_rn, __ddiv_rn,
// __dsqrt_rn) so that no multiply-add is ever contracted and every step rounds
// exactly as the host's numpy sequence does.  Holds none of the method's
// arithmetic: it only produces W and x.
//
// Build: nvcc -gencode arch=compute_100a,code=sm_100a -fmad=false -shared
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kMix1 = 0xBF58476D1CE4E5B9ull;
constexpr uint64_t kMix2 = 0x94D049BB133111EBull;
constexpr int kAtanhTerms = 12;
constexpr int kCosTerms = 12;

__constant__ double c_atanh[kAtanhTerms];   // 1/(2i+1)
__constant__ double c_cos[kCosTerms];       // (-1)^k/(2k)!

__device__ __forceinline__ uint64_t mix(uint64_t z) {
  z = (z ^ (z >> 30)) * kMix1;
  z = (z ^ (z >> 27)) * kMix2;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double uniform(uint64_t key, uint64_t ctr) {
  uint64_t w = mix(key + (ctr + 1ull) * kGamma);
  return __dmul_rn(__dadd_rn((double)(w >> 11), 0.5), 0x1p-53);
}

__device__ double series_ln(double y) {
  const double kLn2 = 0x1.62e42fefa39efp-1;
  const double kSqrtHalf = 0x1.6a09e667f3bcdp-1;
  int e;
  double m = frexp(y, &e);
  if (m < kSqrtHalf) {
    m = __dmul_rn(m, 2.0);
    e -= 1;
  }
  double z = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
  double z2 = __dmul_rn(z, z);
  double p = c_atanh[kAtanhTerms - 1];
  for (int i = kAtanhTerms - 2; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, z2), c_atanh[i]);
  return __dadd_rn(__dmul_rn((double)e, kLn2), __dmul_rn(__dadd_rn(z, z), p));
}

__device__ double cos_turn(double u) {
  const double kTwoPi = 0x1.921fb54442d18p+2;
  double v = u >= 0.5 ? __dadd_rn(u, -1.0) : u;
  double a = fabs(v);
  bool flip = a > 0.25;
  if (flip) a = __dadd_rn(0.5, -a);
  double th = __dmul_rn(a, kTwoPi);
  double t2 = __dmul_rn(th, th);
  double p = c_cos[kCosTerms - 1];
  for (int i = kCosTerms - 2; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, t2), c_cos[i]);
  return flip ? -p : p;
}

__device__ __forceinline__ double laplace(uint64_t key, uint64_t ctr, double b) {
  double u = uniform(key, ctr);
  double v = __dadd_rn(u, -0.5);
  double a = fabs(v);
  double mag = -series_ln(__dadd_rn(1.0, -__dadd_rn(a, a)));
  double t = __dmul_rn(b, mag);
  return v >= 0.0 ? t : -t;
}

__device__ __forceinline__ double gauss(uint64_t key, uint64_t ctr) {
  double u1 = uniform(key, 2ull * ctr);
  double u2 = uniform(key, 2ull * ctr + 1ull);
  double r = __dsqrt_rn(__dmul_rn(-2.0, series_ln(u1)));
  return __dmul_rn(r, cos_turn(u2));
}

__global__ void k_laplace(float* out, int64_t n, uint64_t ctr0, uint64_t key, double b) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __double2float_rn(laplace(key, ctr0 + (uint64_t)i, b));
}

__global__ void k_gauss(float* out, int64_t n, int64_t K, uint64_t ctr0, uint64_t key,
                        double sigma, uint64_t heavy_key, double heavy_frac, double heavy_mul,
                        const float* col_factor) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t c = ctr0 + (uint64_t)i;
    double g = gauss(key, c);
    double t = sigma == 1.0 ? g : __dmul_rn(sigma, g);
    if (heavy_frac > 0.0 && uniform(heavy_key, c) < heavy_frac) t = __dmul_rn(t, heavy_mul);
    if (col_factor) {
      float f = col_factor[i % K];
      if (f != 1.0f) t = __dmul_rn(t, (double)f);
    }
    out[i] = __double2float_rn(t);
  }
}

bool g_init = false;

int ensure_tables() {
  if (g_init) return 0;
  double a[kAtanhTerms], c[kCosTerms];
  for (int i = 0; i < kAtanhTerms; ++i) a[i] = 1.0 / (double)(2 * i + 1);
  c[0] = 1.0;
  for (int k = 1; k < kCosTerms; ++k) c[k] = c[k - 1] / (double)(-(2 * k - 1) * (2 * k));
  if (cudaMemcpyToSymbol(c_atanh, a, sizeof(a)) != cudaSuccess) return 1;
  if (cudaMemcpyToSymbol(c_cos, c, sizeof(c)) != cudaSuccess) return 1;
  g_init = true;
  return 0;
}

int grid_for(int64_t n) {
  int64_t b = (n + 255) / 256;
  return (int)(b < 148 * 32 ? (b > 0 ? b : 1) : 148 * 32);
}

}  // namespace

extern "C" {

// out[i] = float(Laplace(0, b)) of counter ctr0 + i, i in [0, n).  Device pointer,
// caller's stream.  Returns 0, or the CUDA error code.
int synth_fill_laplace(float* out, int64_t n, uint64_t ctr0, uint64_t key, double b,
                       void* stream) {
  if (ensure_tables()) return 1;
  if (n <= 0) return 0;
  k_laplace<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, ctr0, key, b);
  return (int)cudaGetLastError();
}

// out[i] = float(sigma * N(0,1) [* heavy_mul if heavy] [* col_factor[i % K]]) of
// counter ctr0 + i.  col_factor is a device pointer or NULL.
int synth_fill_gauss(float* out, int64_t n, int64_t K, uint64_t ctr0, uint64_t key,
                     double sigma, uint64_t heavy_key, double heavy_frac, double heavy_mul,
                     const float* col_factor, void* stream) {
  if (ensure_tables()) return 1;
  if (n <= 0) return 0;
  k_gauss<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, K, ctr0, key, sigma,
                                                          heavy_key, heavy_frac, heavy_mul,
                                                          col_factor);
  return (int)cudaGetLastError();
}

}  // extern "C"
