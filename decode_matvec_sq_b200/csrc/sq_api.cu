// sq_api.cu -- the extern "C" entry points declared in include/sq.h:
// host-side validation, device checks and launch orchestration.  No device
// memory is allocated here.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "sq_internal.h"
#include "sq_layout.h"

namespace sq {

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

struct AttrEntry {
  const void* fn;
  int device;
  int bytes;
};
AttrEntry g_attr[256];
int g_attr_n = 0;
}  // namespace

bool current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.device != dev) {
    DeviceInfo n;
    n.device = dev;
    if (cudaDeviceGetAttribute(&n.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return false;
    d = n;
  }
  *out = d;
  return true;
}

cudaError_t ensure_smem_attr(const void* func, int bytes) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].fn == func && g_attr[i].device == dev) {
      if (g_attr[i].bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) g_attr[i].bytes = bytes;
      return e;
    }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && g_attr_n < 256) g_attr[g_attr_n++] = AttrEntry{func, dev, bytes};
  return e;
}

}  // namespace sq

using namespace sq;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_group(int g) { return g == 32 || g == 64 || g == 128; }

// Shapes the library supports (int32 indexing of rows and channels).
bool valid_shape(int64_t N, int64_t K) {
  return N >= 1 && K >= 1 && N <= (1 << 28) && K <= (1 << 24) && N * round_up(K, 16) < (1ll << 40);
}

sq_status check_device(DeviceInfo* d) {
  if (!current_device(d)) return SQ_ERR_CUDA;
  if (d->major != 10 || d->minor != 0) return SQ_ERR_UNSUPPORTED_DEVICE;
  return SQ_OK;
}

sq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

// Largest K of the tiled layout (the decode kernel keeps a bitmap of the
// outlier channels of a whole row in shared memory).
constexpr int32_t kMaxTiledK = 131072;

bool known_layout(int32_t layout) {
  return layout == SQ_LAYOUT_ROWS || layout == SQ_LAYOUT_TILES || layout == SQ_LAYOUT_TILES_SPARSE ||
         layout == SQ_LAYOUT_TILES_ASYM;
}
bool tiled(int32_t layout) {
  return layout == SQ_LAYOUT_TILES || layout == SQ_LAYOUT_TILES_SPARSE || layout == SQ_LAYOUT_TILES_ASYM;
}

bool valid_layout(int32_t layout, int32_t G, int32_t K) {
  if (layout == SQ_LAYOUT_ROWS) return true;
  return tiled(layout) && G == kTileK && K <= kMaxTiledK;
}

int32_t sign_stride_of(int32_t K, int32_t layout) {
  return tiled(layout) ? (int32_t)(tiles_cols(K) / 32) : (int32_t)round_up(ceil_div(K, 32), 4);
}
int32_t res_stride_of(int32_t K, int32_t layout) {
  return tiled(layout) ? (int32_t)tiles_cols(K) : (int32_t)round_up(K, 16);
}
int32_t scale_stride_of(int32_t K, int32_t G, int32_t layout) {
  return tiled(layout) ? (int32_t)(tiles_cols(K) / kTileK) : (int32_t)round_up(ceil_div(K, G), 4);
}
// Rows of every array (the tiled layouts pad N to a multiple of 16).
int64_t rows_of(int32_t N, int32_t layout) {
  return tiled(layout) ? tiles_rows(N) : (int64_t)N;
}
// Tiles of a tiled layout.
int64_t tiles_of(int32_t N, int32_t K) { return tiles_rows(N) / kTileRows * (tiles_cols(K) / kTileK); }

sq_status check_weight(const sq_packed_weight* w) {
  if (!w || !w->sign_bits || !w->alpha || !w->res_q || !w->res_scale) return SQ_ERR_INVALID_ARG;
  if (!valid_group(w->group_size) || !valid_shape(w->N, w->K)) return SQ_ERR_SHAPE;
  if (!known_layout(w->layout)) return SQ_ERR_INVALID_ARG;
  if (!valid_layout(w->layout, w->group_size, w->K)) return SQ_ERR_SHAPE;
  if (w->layout == SQ_LAYOUT_TILES_SPARSE) {
    if (!w->keep_bits || !w->res_bytes) return SQ_ERR_INVALID_ARG;
    if (!aligned16(w->keep_bits) || !aligned16(w->res_bytes)) return SQ_ERR_ALIGN;
  }
  if (w->layout == SQ_LAYOUT_TILES_ASYM) {
    if (!w->res_zero) return SQ_ERR_INVALID_ARG;
    if (!aligned16(w->res_zero)) return SQ_ERR_ALIGN;
  }
  if (w->sign_stride != sign_stride_of(w->K, w->layout) ||
      w->res_stride != res_stride_of(w->K, w->layout) ||
      w->scale_stride != scale_stride_of(w->K, w->group_size, w->layout))
    return SQ_ERR_SHAPE;
  if (!aligned16(w->sign_bits) || !aligned16(w->alpha) || !aligned16(w->res_q) ||
      !aligned16(w->res_scale) || (w->mask_bits && !aligned16(w->mask_bits)))
    return SQ_ERR_ALIGN;
  return SQ_OK;
}

// Offsets of the five arrays inside one allocation, each 256-byte aligned.
// alpha holds roundup(N, 8) (rows) or N16 (tiles) floats.
struct Carve {
  size_t sign, mask, alpha, res, scale, keep, count, zero, total;
};

Carve carve(int32_t N, int32_t K, int32_t G, int32_t with_mask, int32_t layout) {
  Carve c;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = (size_t)round_up((int64_t)(off + bytes), 256);
    return at;
  };
  const int64_t rows = rows_of(N, layout);
  c.sign = take((size_t)rows * sign_stride_of(K, layout) * 4);
  c.mask = with_mask ? take((size_t)rows * sign_stride_of(K, layout) * 4) : 0;
  c.alpha = take((size_t)round_up(rows, 8) * 4);
  c.res = take((size_t)rows * res_stride_of(K, layout));
  c.scale = take((size_t)rows * scale_stride_of(K, G, layout) * 4);
  c.keep = c.count = c.zero = 0;
  if (layout == SQ_LAYOUT_TILES_SPARSE) {
    c.keep = take((size_t)rows * sign_stride_of(K, layout) * 4);
    c.count = take((size_t)tiles_of(N, K) * 4);
  }
  if (layout == SQ_LAYOUT_TILES_ASYM) c.zero = take((size_t)rows * scale_stride_of(K, G, layout) * 4);
  c.total = off;
  return c;
}

}  // namespace

extern "C" {

const char* sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "ok";
    case SQ_ERR_INVALID_ARG: return "invalid argument";
    case SQ_ERR_SHAPE: return "unsupported shape";
    case SQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SQ_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100 (B200)";
    case SQ_ERR_CUDA: return "CUDA runtime error";
    case SQ_ERR_NONFINITE: return "non-finite input";
    case SQ_ERR_TIMEOUT: return "bounded wait ran out";
    case SQ_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

sq_status sq_device_check(void) {
  DeviceInfo d;
  return check_device(&d);
}

size_t sq_packed_bytes(int32_t N, int32_t K, int32_t group_size, int32_t with_mask,
                       int32_t layout) {
  if (!valid_shape(N, K) || !valid_group(group_size)) return 0;
  if (!known_layout(layout)) return 0;
  if (!valid_layout(layout, group_size, K)) return 0;
  return carve(N, K, group_size, with_mask, layout).total;
}

sq_status sq_packed_view(void* base, int32_t N, int32_t K, int32_t group_size, int32_t with_mask,
                         int32_t layout, sq_packed_weight* out) {
  if (!base || !out) return SQ_ERR_INVALID_ARG;
  if (!known_layout(layout)) return SQ_ERR_INVALID_ARG;
  if (!valid_shape(N, K) || !valid_group(group_size)) return SQ_ERR_SHAPE;
  if (!valid_layout(layout, group_size, K)) return SQ_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(base) & 255u) != 0) return SQ_ERR_ALIGN;
  const Carve c = carve(N, K, group_size, with_mask, layout);
  uint8_t* b = static_cast<uint8_t*>(base);
  out->N = N;
  out->K = K;
  out->group_size = group_size;
  out->layout = layout;
  out->sign_stride = sign_stride_of(K, layout);
  out->res_stride = res_stride_of(K, layout);
  out->scale_stride = scale_stride_of(K, group_size, layout);
  out->sign_bits = reinterpret_cast<uint32_t*>(b + c.sign);
  out->mask_bits = with_mask ? reinterpret_cast<uint32_t*>(b + c.mask) : nullptr;
  out->alpha = reinterpret_cast<float*>(b + c.alpha);
  out->res_q = reinterpret_cast<int8_t*>(b + c.res);
  out->res_scale = reinterpret_cast<float*>(b + c.scale);
  const bool sparse = layout == SQ_LAYOUT_TILES_SPARSE;
  out->keep_bits = sparse ? reinterpret_cast<uint32_t*>(b + c.keep) : nullptr;
  out->res_bytes = sparse ? reinterpret_cast<int32_t*>(b + c.count) : nullptr;
  out->res_zero = layout == SQ_LAYOUT_TILES_ASYM ? reinterpret_cast<int32_t*>(b + c.zero) : nullptr;
  return SQ_OK;
}

sq_status sq_decompose_pack(const float* W, int32_t N, int32_t K, int32_t trunk_percent,
                            const sq_packed_weight* out, int32_t* dev_status, void* stream) {
  if (!W || !out) return SQ_ERR_INVALID_ARG;
  sq_status st = check_weight(out);
  if (st != SQ_OK) return st;
  if (out->N != N || out->K != K) return SQ_ERR_SHAPE;
  if (out->layout == SQ_LAYOUT_TILES_SPARSE) return SQ_ERR_INVALID_ARG;  // sq_decompose_pack_sparse
  if (trunk_percent == 0 || trunk_percent > 100) return SQ_ERR_INVALID_ARG;
  if (trunk_percent > 0 && !out->mask_bits) return SQ_ERR_INVALID_ARG;
  if (!aligned16(W) || (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)))
    return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  // full trunk with a mask array present: the mask is written all ones
  sq_packed_weight pw = *out;
  return from_cuda(launch_decompose_pack(W, N, K, trunk_percent, pw, dev_status,
                                         static_cast<cudaStream_t>(stream)));
}

sq_status sq_decompose_pack_sparse(const float* W, int32_t N, int32_t K, int32_t trunk_percent,
                                   int32_t residual_percent, const sq_packed_weight* out,
                                   int32_t* dev_status, void* stream) {
  if (!W || !out) return SQ_ERR_INVALID_ARG;
  sq_status st = check_weight(out);
  if (st != SQ_OK) return st;
  if (out->layout != SQ_LAYOUT_TILES_SPARSE) return SQ_ERR_INVALID_ARG;
  if (out->N != N || out->K != K) return SQ_ERR_SHAPE;
  if (trunk_percent == 0 || trunk_percent > 100) return SQ_ERR_INVALID_ARG;
  if (trunk_percent > 0 && !out->mask_bits) return SQ_ERR_INVALID_ARG;
  if (residual_percent < 1 || residual_percent > 99) return SQ_ERR_INVALID_ARG;
  if (!aligned16(W) || (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)))
    return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the dense tiled decomposition first (trunk, alpha, codes), then the
  // sparse residual over it
  sq_packed_weight dense = *out;
  dense.layout = SQ_LAYOUT_TILES;
  cudaError_t e = launch_decompose_pack(W, N, K, trunk_percent, dense, dev_status, s);
  if (e != cudaSuccess) return SQ_ERR_CUDA;
  return from_cuda(launch_sparsify_residual(W, N, K, residual_percent, *out, s));
}

size_t sq_residual_errors_scratch_bytes(int32_t N) {
  return N < 1 ? 0 : (size_t)round_up(16 * (int64_t)N, 256);
}

sq_status sq_residual_errors(const float* W, const sq_packed_weight* w, double* err, void* scratch,
                             size_t scratch_bytes, int32_t* dev_status, void* stream) {
  if (!W || !err || !scratch) return SQ_ERR_INVALID_ARG;
  sq_status st = check_weight(w);
  if (st != SQ_OK) return st;
  if (w->layout == SQ_LAYOUT_TILES_SPARSE) return SQ_ERR_INVALID_ARG;
  if (scratch_bytes < sq_residual_errors_scratch_bytes(w->N)) return SQ_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(err) || !aligned16(scratch)) return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  return from_cuda(launch_residual_errors(W, *w, err, static_cast<double*>(scratch), dev_status,
                                          static_cast<cudaStream_t>(stream)));
}

sq_status sq_decompose_pack_auto(const float* W, int32_t N, int32_t K, int32_t trunk_percent,
                                 sq_packed_weight* out, void* scratch, size_t scratch_bytes,
                                 int32_t* fell_back, double* err_host, int32_t* dev_status,
                                 void* stream) {
  if (!W || !out || !scratch) return SQ_ERR_INVALID_ARG;
  if (!out->mask_bits) return SQ_ERR_INVALID_ARG;  // the fallback needs an (empty) mask
  sq_status st = check_weight(out);
  if (st != SQ_OK) return st;
  if (out->layout == SQ_LAYOUT_TILES_SPARSE) return SQ_ERR_INVALID_ARG;
  if (scratch_bytes < sq_residual_errors_scratch_bytes(N) + 256) return SQ_ERR_WORKSPACE;
  if (!aligned16(scratch)) return SQ_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = sq_decompose_pack(W, N, K, trunk_percent, out, dev_status, stream)) != SQ_OK) return st;
  double* err = static_cast<double*>(scratch);
  void* rest = static_cast<uint8_t*>(scratch) + 256;
  if ((st = sq_residual_errors(W, out, err, rest, scratch_bytes - 256, dev_status, stream)) != SQ_OK)
    return st;
  double e[2];
  if (cudaMemcpyAsync(e, err, sizeof(e), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SQ_ERR_CUDA;
  if (err_host) {
    err_host[0] = e[0];
    err_host[1] = e[1];
  }
  const bool fall = e[1] <= e[0];
  if (fell_back) *fell_back = fall ? 1 : 0;
  if (fall) return sq_decompose_pack(W, N, K, 100, out, dev_status, stream);
  if (trunk_percent < 0) out->mask_bits = nullptr;
  return SQ_OK;
}

sq_status sq_calibrate_outliers(const float* X, int32_t T, int32_t K, int32_t k, int32_t* idx_out,
                                int32_t* dev_status, void* stream) {
  if (!X || !idx_out) return SQ_ERR_INVALID_ARG;
  if (T < 1 || K < 1 || K > 40960 || k < 1 || k > K) return SQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(idx_out)) return SQ_ERR_ALIGN;
  DeviceInfo d;
  sq_status st = check_device(&d);
  if (st != SQ_OK) return st;
  return from_cuda(launch_calibrate(X, T, K, k, idx_out, dev_status, static_cast<cudaStream_t>(stream)));
}

sq_status sq_quantize_act(const float* x, int32_t M, int32_t K, const int32_t* idx, int32_t n_out,
                          int8_t* xq, float* sx, float* x_out, int32_t* dev_status, uint32_t flags,
                          void* stream) {
  if (!x || !xq || !sx) return SQ_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || K > (1 << 24) || M > (1 << 24)) return SQ_ERR_SHAPE;
  if (n_out < 0 || n_out > kMaxOutliers || n_out > K) return SQ_ERR_SHAPE;
  if (n_out > 0 && (!idx || !x_out)) return SQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(sx) || (n_out > 0 && (!aligned16(idx) || !aligned16(x_out))))
    return SQ_ERR_ALIGN;
  if (flags & ~SQ_LAUNCH_PDL) return SQ_ERR_INVALID_ARG;
  DeviceInfo d;
  sq_status st = check_device(&d);
  if (st != SQ_OK) return st;
  return from_cuda(launch_quantize_act(x, M, K, idx, n_out, xq, sx, x_out, dev_status,
                                       (flags & SQ_LAUNCH_PDL) != 0, static_cast<cudaStream_t>(stream)));
}

size_t sq_linear_workspace_bytes(const sq_packed_weight* w, int32_t M) {
  if (!w || check_weight(w) != SQ_OK || M < 1) return 0;
  DeviceInfo d;
  if (!current_device(&d)) return 0;
  return linear_workspace_bytes(*w, M, d.sm_count);
}

static sq_status linear_common(const sq_packed_weight* w, const int8_t* xq, const float* sx,
                               const float* x_out, const int32_t* idx, int32_t n_out, int32_t M,
                               float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                               size_t ws_bytes, int32_t* dev_status, uint32_t flags, void* stream) {
  sq_status st = check_weight(w);
  if (st != SQ_OK) return st;
  if (!xq || !sx || !y) return SQ_ERR_INVALID_ARG;
  if (M < 1 || M > (1 << 20)) return SQ_ERR_SHAPE;
  if (n_out < 0 || n_out > kMaxOutliers || n_out > w->K) return SQ_ERR_SHAPE;
  if (n_out > 0 && (!idx || !x_out)) return SQ_ERR_INVALID_ARG;
  if (flags & ~(SQ_LAUNCH_PDL | SQ_TRUNK_ONLY)) return SQ_ERR_INVALID_ARG;
  const bool trunk_only = (flags & SQ_TRUNK_ONLY) != 0;
  if (trunk_only && (!tiled(w->layout) || T_out || R_out)) return SQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(y) ||
      (n_out > 0 && (!aligned16(idx) || !aligned16(x_out))) || (workspace && !aligned16(workspace)))
    return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  const size_t need = linear_workspace_bytes(*w, M, d.sm_count);
  if (!workspace || ws_bytes < need) return SQ_ERR_WORKSPACE;
  const size_t part = linear_part_bytes(d.sm_count);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T_out) {
    cudaError_t e = cudaMemsetAsync(T_out, 0, (size_t)M * w->N * sizeof(int32_t), s);
    if (e != cudaSuccess) return SQ_ERR_CUDA;
  }
  const int ng = (int)ceil_div(w->K, w->group_size);
  if (w->layout == SQ_LAYOUT_ROWS && M >= kPrefillMinTokens && prefill_supported(*w)) {
    // many tokens: one tcgen05 GEMM-shaped launch over all of them
    const cudaError_t e = launch_prefill(*w, M, xq, sx, x_out, idx, n_out, y, T_out, R_out,
                                         dev_status, s);
    return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
  }
  const bool tc = tiled(w->layout);
  const int per_pass = tc ? linear_tc_pass_tokens(*w, trunk_only) : kMaxTokensPerPass;
  const int64_t xs = xq_stride_of(w->K);
  for (int t0 = 0; t0 < M; t0 += per_pass) {
    const int m = std::min(per_pass, M - t0);
    const int8_t* xq_t = xq + (int64_t)t0 * xs;
    const float* xo_t = n_out ? x_out + (int64_t)t0 * n_out : nullptr;
    float* y_t = y + (int64_t)t0 * w->N;
    int32_t* T_t = T_out ? T_out + (int64_t)t0 * w->N : nullptr;
    int32_t* R_t = R_out ? R_out + (int64_t)t0 * w->N * ng : nullptr;
    cudaError_t e;
    if (tc) {
      e = launch_linear_tc(*w, m, xq_t, sx + t0, xo_t, nullptr, idx, n_out, y_t, T_t, R_t,
                           workspace, part, d.sm_count, dev_status, (flags & SQ_LAUNCH_PDL) != 0,
                           trunk_only, s);
    } else {
      LinearPlan plan;
      if (!plan_linear(*w, m, n_out, d.sm_count, &plan)) return SQ_ERR_SHAPE;
      if (plan.smem_bytes > d.smem_optin) return SQ_ERR_SHAPE;
      e = launch_linear(*w, plan, xq_t, sx + t0, xo_t, idx, n_out, y_t, T_t, R_t, workspace, part,
                        dev_status, (flags & SQ_LAUNCH_PDL) != 0, s);
    }
    if (e != cudaSuccess) return SQ_ERR_CUDA;
  }
  return SQ_OK;
}

sq_status sq_linear(const sq_packed_weight* w, const int8_t* xq, const float* sx,
                    const float* x_out, const int32_t* idx, int32_t n_out, int32_t M, float* y,
                    void* workspace, size_t ws_bytes, int32_t* dev_status, uint32_t flags,
                    void* stream) {
  return linear_common(w, xq, sx, x_out, idx, n_out, M, y, nullptr, nullptr, workspace, ws_bytes,
                       dev_status, flags, stream);
}

sq_status sq_linear_accumulators(const sq_packed_weight* w, const int8_t* xq, const float* sx,
                                 const float* x_out, const int32_t* idx, int32_t n_out, int32_t M,
                                 float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                                 size_t ws_bytes, int32_t* dev_status, uint32_t flags,
                                 void* stream) {
  if (!T_out || !R_out) return SQ_ERR_INVALID_ARG;
  if (!aligned16(T_out) || !aligned16(R_out)) return SQ_ERR_ALIGN;
  if (flags & (SQ_LAUNCH_PDL | SQ_TRUNK_ONLY)) return SQ_ERR_INVALID_ARG;
  return linear_common(w, xq, sx, x_out, idx, n_out, M, y, T_out, R_out, workspace, ws_bytes,
                       dev_status, flags, stream);
}

// The staged route of sq_quantize_linear: the activation split once
// (k_quantize_act into the workspace), then the decode kernel on its codes.
// Measured on B200 (70B-shaped MLP, 8192 <-> 28672): every CTA of the fused
// kernel quantizes all M tokens of x, which costs more than a separate split
// once M > 1 and M * roundup(K, 128) > 16 KiB (8192 -> 28672 at M = 4: 62.3
// against 60.0 us); and where the codes of M tokens do not fit one pass of
// the fused kernel, it reads the weights once per pass (28672 -> 8192 at
// M = 8: 215.8 against 69.9 us).
constexpr int64_t kFusedMaxCodeBytes = 16 << 10;

static size_t stage_bytes(const sq_packed_weight& w, int M, int n_out) {
  return (size_t)round_up((int64_t)M * xq_stride_of(w.K), 256) + (size_t)round_up(4 * (int64_t)M, 256) +
         (size_t)round_up(4 * (int64_t)M * n_out, 256);
}

size_t sq_quantize_linear_workspace_bytes(const sq_packed_weight* w, int32_t M, int32_t n_out) {
  if (!w || check_weight(w) != SQ_OK || M < 1 || n_out < 0 || n_out > kMaxOutliers) return 0;
  DeviceInfo d;
  if (!current_device(&d)) return 0;
  const size_t need = linear_workspace_bytes(*w, M, d.sm_count);
  if (need == 0) return 0;
  return (size_t)round_up((int64_t)need, 256) + stage_bytes(*w, M, n_out);
}

int32_t sq_linear_tokens_per_pass(const sq_packed_weight* w, uint32_t flags) {
  if (!w || check_weight(w) != SQ_OK || (flags & ~SQ_TRUNK_ONLY)) return 0;
  const bool trunk_only = (flags & SQ_TRUNK_ONLY) != 0;
  if (!tiled(w->layout)) return trunk_only ? 0 : kMaxTokensPerPass;
  return linear_tc_pass_tokens(*w, trunk_only);
}

int32_t sq_quantize_linear_tokens_per_pass(const sq_packed_weight* w, int32_t n_out) {
  if (!w || check_weight(w) != SQ_OK || !tiled(w->layout)) return 0;
  if (n_out < 0 || n_out > kMaxOutliers || n_out > w->K) return 0;
  return linear_tc_fused_tokens(*w, n_out);
}

sq_status sq_quantize_linear(const sq_packed_weight* w, const float* x, int32_t M,
                             const int32_t* idx, int32_t n_out, float* y, void* workspace,
                             size_t ws_bytes, int32_t* dev_status, uint32_t flags, void* stream) {
  sq_status st = check_weight(w);
  if (st != SQ_OK) return st;
  if (!x || !y) return SQ_ERR_INVALID_ARG;
  if (!tiled(w->layout)) return SQ_ERR_SHAPE;
  if (M < 1 || M > (1 << 20)) return SQ_ERR_SHAPE;
  if (n_out < 0 || n_out > kMaxOutliers || n_out > w->K) return SQ_ERR_SHAPE;
  if (n_out > 0 && !idx) return SQ_ERR_INVALID_ARG;
  if (flags & ~(SQ_LAUNCH_PDL | SQ_TRUNK_ONLY)) return SQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || (n_out > 0 && !aligned16(idx)) ||
      (workspace && !aligned16(workspace)))
    return SQ_ERR_ALIGN;
  const int per_pass = linear_tc_fused_tokens(*w, n_out);
  if (per_pass < 1) return SQ_ERR_SHAPE;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  const size_t need = linear_workspace_bytes(*w, M, d.sm_count);
  if (!workspace || ws_bytes < need) return SQ_ERR_WORKSPACE;
  const size_t part = linear_part_bytes(d.sm_count);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool staged_faster = M > 1 && ((int64_t)M * xq_stride_of(w->K) > kFusedMaxCodeBytes ||
                                       ceil_div(M, per_pass) >
                                           ceil_div(M, linear_tc_pass_tokens(*w, (flags & SQ_TRUNK_ONLY) != 0)));
  const size_t base = (size_t)round_up((int64_t)need, 256);
  if (staged_faster && ws_bytes >= base + stage_bytes(*w, M, n_out)) {
    int8_t* xq = static_cast<int8_t*>(workspace) + base;
    float* sx = reinterpret_cast<float*>(xq + round_up((int64_t)M * xq_stride_of(w->K), 256));
    float* xo = n_out > 0 ? sx + round_up(4 * (int64_t)M, 256) / 4 : nullptr;
    const cudaError_t e = launch_quantize_act(x, M, w->K, idx, n_out, xq, sx, xo, dev_status,
                                              (flags & SQ_LAUNCH_PDL) != 0, s);
    if (e != cudaSuccess) return SQ_ERR_CUDA;
    return linear_common(w, xq, sx, xo, idx, n_out, M, y, nullptr, nullptr, workspace, need,
                         dev_status, flags, stream);
  }
  for (int t0 = 0; t0 < M; t0 += per_pass) {
    const int m = std::min(per_pass, M - t0);
    cudaError_t e = launch_linear_tc(*w, m, nullptr, nullptr, nullptr, x + (int64_t)t0 * w->K, idx,
                                     n_out, y + (int64_t)t0 * w->N, nullptr, nullptr, workspace,
                                     part, d.sm_count, dev_status, (flags & SQ_LAUNCH_PDL) != 0,
                                     (flags & SQ_TRUNK_ONLY) != 0, s);
    if (e != cudaSuccess) return SQ_ERR_CUDA;
  }
  return SQ_OK;
}

// ---- NVFP4 prefill ------------------------------------------------------------

static bool nvfp4_shape(int32_t rows, int32_t K) {
  return rows >= 1 && K >= 1 && rows <= (1 << 24) && K <= (1 << 20);
}

struct Nvfp4Carve {
  size_t codes, scales, g, total;
  int32_t rows_pad, code_stride, sf_chunks;
};

static Nvfp4Carve nvfp4_carve(int32_t rows, int32_t K, int32_t per_row) {
  Nvfp4Carve c;
  c.rows_pad = (int32_t)round_up(rows, 128);
  const int64_t k256 = round_up(K, 256);
  c.code_stride = (int32_t)(k256 / 2);
  c.sf_chunks = (int32_t)(k256 / 64);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = (size_t)round_up((int64_t)(off + bytes), 256);
    return at;
  };
  c.codes = take((size_t)c.rows_pad * c.code_stride);
  c.scales = take((size_t)(c.rows_pad / 128) * c.sf_chunks * 512);
  c.g = take(per_row ? (size_t)c.rows_pad * 4 : 8);
  c.total = off;
  return c;
}

static sq_status check_nvfp4(const sq_nvfp4_matrix* m) {
  if (!m || !m->codes || !m->scales || !m->g) return SQ_ERR_INVALID_ARG;
  if (m->per_row != 0 && m->per_row != 1) return SQ_ERR_INVALID_ARG;
  if (!nvfp4_shape(m->rows, m->K)) return SQ_ERR_SHAPE;
  const Nvfp4Carve c = nvfp4_carve(m->rows, m->K, m->per_row);
  if (m->rows_pad != c.rows_pad || m->code_stride != c.code_stride || m->sf_chunks != c.sf_chunks)
    return SQ_ERR_SHAPE;
  if (!aligned16(m->codes) || !aligned16(m->scales) || !aligned16(m->g)) return SQ_ERR_ALIGN;
  return SQ_OK;
}

size_t sq_nvfp4_bytes(int32_t rows, int32_t K, int32_t per_row) {
  if (!nvfp4_shape(rows, K) || (per_row != 0 && per_row != 1)) return 0;
  return nvfp4_carve(rows, K, per_row).total;
}

sq_status sq_nvfp4_view(void* base, int32_t rows, int32_t K, int32_t per_row,
                        sq_nvfp4_matrix* out) {
  if (!base || !out || (per_row != 0 && per_row != 1)) return SQ_ERR_INVALID_ARG;
  if (!nvfp4_shape(rows, K)) return SQ_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(base) & 255u) != 0) return SQ_ERR_ALIGN;
  const Nvfp4Carve c = nvfp4_carve(rows, K, per_row);
  uint8_t* b = static_cast<uint8_t*>(base);
  out->rows = rows;
  out->K = K;
  out->per_row = per_row;
  out->rows_pad = c.rows_pad;
  out->code_stride = c.code_stride;
  out->sf_chunks = c.sf_chunks;
  out->codes = b + c.codes;
  out->scales = b + c.scales;
  out->g = reinterpret_cast<float*>(b + c.g);
  return SQ_OK;
}

sq_status sq_nvfp4_quantize(const float* X, const sq_nvfp4_matrix* out, int32_t* dev_status,
                            void* stream) {
  sq_status st = check_nvfp4(out);
  if (st != SQ_OK) return st;
  if (!X) return SQ_ERR_INVALID_ARG;
  if (!aligned16(X)) return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  return from_cuda(launch_nvfp4_quantize(X, *out, dev_status, static_cast<cudaStream_t>(stream)));
}

sq_status sq_nvfp4_linear(const sq_nvfp4_matrix* w, const sq_nvfp4_matrix* x, float* y,
                          int32_t* dev_status, void* stream) {
  sq_status st = check_nvfp4(w);
  if (st != SQ_OK) return st;
  if ((st = check_nvfp4(x)) != SQ_OK) return st;
  if (!y) return SQ_ERR_INVALID_ARG;
  if (w->per_row != 0 || x->per_row != 1) return SQ_ERR_INVALID_ARG;
  if (w->K != x->K) return SQ_ERR_SHAPE;
  if (!aligned16(y)) return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  return from_cuda(launch_nvfp4_gemm(*w, *x, y, dev_status, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ---- failure injection for the tests (include/sq_testing.h) -----------------------
#include "../../include/sq_testing.h"

extern "C" sq_status sq_testing_prefill_stalled(const sq_packed_weight* w, const int8_t* xq,
                                                const float* sx, const float* x_out,
                                                const int32_t* idx, int32_t n_out, int32_t M,
                                                float* y, int32_t skip_group, uint64_t wait_ns,
                                                int32_t* dev_status, void* stream) {
  sq_status st = check_weight(w);
  if (st != SQ_OK) return st;
  if (!xq || !sx || !y) return SQ_ERR_INVALID_ARG;
  if (w->layout != SQ_LAYOUT_ROWS || w->group_size != kTileK || M < kPrefillMinTokens ||
      M > (1 << 20))
    return SQ_ERR_SHAPE;
  if (n_out < 0 || n_out > kMaxOutliers || n_out > w->K) return SQ_ERR_SHAPE;
  if (n_out > 0 && (!idx || !x_out)) return SQ_ERR_INVALID_ARG;
  if (skip_group < -1 || skip_group >= (int32_t)ceil_div(w->K, kTileK)) return SQ_ERR_INVALID_ARG;
  if (wait_ns < 1 || wait_ns > 1000000000ull) return SQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(y) ||
      (n_out > 0 && (!aligned16(idx) || !aligned16(x_out))))
    return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  if (!prefill_supported(*w)) return SQ_ERR_UNSUPPORTED_DEVICE;
  return from_cuda(launch_prefill(*w, M, xq, sx, x_out, idx, n_out, y, nullptr, nullptr, dev_status,
                                  static_cast<cudaStream_t>(stream), wait_ns, skip_group));
}

extern "C" sq_status sq_testing_nvfp4_stalled(const sq_nvfp4_matrix* w, const sq_nvfp4_matrix* x,
                                              float* y, int32_t skip_stage, uint64_t wait_ns,
                                              int32_t* dev_status, void* stream) {
  sq_status st = check_nvfp4(w);
  if (st != SQ_OK) return st;
  if ((st = check_nvfp4(x)) != SQ_OK) return st;
  if (!y) return SQ_ERR_INVALID_ARG;
  if (w->per_row != 0 || x->per_row != 1) return SQ_ERR_INVALID_ARG;
  if (w->K != x->K) return SQ_ERR_SHAPE;
  if (skip_stage < -1 || skip_stage >= w->code_stride / 128) return SQ_ERR_INVALID_ARG;
  if (wait_ns < 1 || wait_ns > 1000000000ull) return SQ_ERR_INVALID_ARG;
  if (!aligned16(y)) return SQ_ERR_ALIGN;
  DeviceInfo d;
  if ((st = check_device(&d)) != SQ_OK) return st;
  return from_cuda(launch_nvfp4_gemm(*w, *x, y, dev_status, static_cast<cudaStream_t>(stream),
                                     wait_ns, skip_stage));
}

extern "C" sq_status sq_testing_mma_peak(int32_t kind, int32_t iters, double* ops_per_s,
                                         int32_t* dev_status, void* stream) {
  if (!ops_per_s || (kind != 0 && kind != 1)) return SQ_ERR_INVALID_ARG;
  if (iters < 1 || iters > 100000) return SQ_ERR_SHAPE;
  DeviceInfo d;
  sq_status st = check_device(&d);
  if (st != SQ_OK) return st;
  return from_cuda(run_mma_peak(kind, iters, ops_per_s, dev_status, static_cast<cudaStream_t>(stream)));
}

namespace sq {
// sq_probe.cu
cudaError_t run_read_peak(const void* buf, size_t bytes, int iters, double* bytes_per_s,
                          cudaStream_t stream);
}  // namespace sq

extern "C" sq_status sq_testing_read_peak(const void* buf, uint64_t bytes, int32_t iters,
                                          double* bytes_per_s, void* stream) {
  if (!buf || !bytes_per_s) return SQ_ERR_INVALID_ARG;
  if (!aligned16(buf)) return SQ_ERR_ALIGN;
  if (bytes < 16 || bytes % 16 != 0 || iters < 1 || iters > 1000) return SQ_ERR_SHAPE;
  DeviceInfo d;
  sq_status st = check_device(&d);
  if (st != SQ_OK) return st;
  return from_cuda(run_read_peak(buf, (size_t)bytes, iters, bytes_per_s, static_cast<cudaStream_t>(stream)));
}
