// sq_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sq.h"

namespace sq {

struct DeviceInfo {
  int device = -1;
  int major = 0, minor = 0;
  int sm_count = 0;
  int smem_optin = 0;  // max dynamic shared memory per block (opt-in)
};

// Properties of the current device (cached per device).  false on CUDA error.
bool current_device(DeviceInfo* out);

// Sets the kernel's max dynamic shared memory once per device.
cudaError_t ensure_smem_attr(const void* func, int bytes);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Row stride of the activation codes xq: roundup(K, 128) bytes, zero padded,
// so that the decode kernels read whole 128-channel groups.
inline int64_t xq_stride_of(int64_t K) { return round_up(K, 128); }

// ---- launchers ---------------------------------------------------------------
cudaError_t launch_decompose_pack(const float* W, int N, int K, int P, const sq_packed_weight& pw,
                                  int32_t* status, cudaStream_t stream);

// The sparse residual over a tiled decomposition already in pw's arrays:
// per-row threshold, re-quantized groups, keep bits, packed codes, byte counts.
cudaError_t launch_sparsify_residual(const float* W, int N, int K, int Ps, const sq_packed_weight& pw,
                                     cudaStream_t stream);

// Per-row squared reconstruction errors of w and of plain INT8 groups of W
// into scratch[2N], then their sums in row order into err[2] (binary64).
cudaError_t launch_residual_errors(const float* W, const sq_packed_weight& w, double* err,
                                   double* scratch, int32_t* status, cudaStream_t stream);

cudaError_t launch_calibrate(const float* X, int T, int K, int k, int32_t* idx_out,
                             int32_t* status, cudaStream_t stream);

cudaError_t launch_quantize_act(const float* x, int M, int K, const int32_t* idx, int n_out,
                                int8_t* xq, float* sx, float* x_out, int32_t* status, bool pdl,
                                cudaStream_t stream);

// Launch plan of the CUDA-core decode kernel (SQ_LAYOUT_ROWS).
struct LinearPlan {
  int M = 1;           // tokens in this pass (1..kMaxTokensPerPass)
  int Kc = 0;          // channels per piece
  int n_c = 0;         // pieces per row
  int U = 0;           // work units = N * n_c
  int grid = 0;        // CTAs
  int smem_bytes = 0;
  size_t ws_cnt_bytes = 0;
  size_t ws_part_bytes = 0;
};

constexpr int kMaxTokensPerPass = 4;     // CUDA-core decode kernel
constexpr int kMaxOutliers = 4096;

// Plans a decode launch for M tokens (M <= kMaxTokensPerPass) on the current device.
bool plan_linear(const sq_packed_weight& w, int M, int n_out, int sm_count, LinearPlan* plan);

// Workspace: [partial sums of rows shared by warps: linear_part_bytes()]
// [one int32 arrival counter per row].  The first area depends only on the
// device, so one workspace can serve weights of any N and both kernels.
size_t linear_part_bytes(int sm_count);
size_t linear_workspace_bytes(const sq_packed_weight& w, int M, int sm_count);

cudaError_t launch_linear(const sq_packed_weight& w, const LinearPlan& plan, const int8_t* xq,
                          const float* sx, const float* x_out, const int32_t* idx, int n_out,
                          float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                          size_t part_bytes, int32_t* status, bool pdl, cudaStream_t stream);

// Tensor-core decode kernel (tiled layouts), up to linear_tc_pass_tokens()
// tokens (16 where their partial sums fit in shared memory, else 8): the
// weights are read once per pass.  With x != NULL (fused mode) it performs the
// activation split of x itself (xq, sx, x_out unused) for at most
// linear_tc_fused_tokens() tokens.
size_t linear_tc_part_bytes(int sm_count);
int linear_tc_pass_tokens(const sq_packed_weight& w, bool trunk_only);
int linear_tc_fused_tokens(const sq_packed_weight& w, int n_out);
cudaError_t launch_linear_tc(const sq_packed_weight& w, int M, const int8_t* xq, const float* sx,
                             const float* x_out, const float* x, const int32_t* idx, int n_out,
                             float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                             size_t part_bytes, int sm_count, int32_t* status, bool pdl,
                             bool trunk_only, cudaStream_t stream);

// Prefill kernel (SQ_LAYOUT_ROWS, group size 128, many tokens): tcgen05 int8
// MMAs with TMEM accumulators.  T_out / R_out optional (both or neither).
constexpr int kPrefillMinTokens = 64;
bool prefill_supported(const sq_packed_weight& w);
// wait_ns bounds every wait of the kernel; skip_group >= 0 (tests only) never
// requests that channel group's operands, so the kernel's waits run out.
// NVFP4 prefill (sq_nvfp4.cu): the quantizer (per tensor: amax reduction,
// then the quantizer; per row: one kernel) and the block-scaled tcgen05 GEMM.
cudaError_t launch_nvfp4_quantize(const float* X, const sq_nvfp4_matrix& out, int32_t* status,
                                  cudaStream_t stream);
cudaError_t launch_nvfp4_gemm(const sq_nvfp4_matrix& w, const sq_nvfp4_matrix& x, float* y,
                              int32_t* status, cudaStream_t stream,
                              uint64_t wait_ns = 1000000000ull, int skip_stage = -1);

// Tensor-core peak probe (sq_probe.cu; include/sq_testing.h).
cudaError_t run_mma_peak(int kind, int iters, double* ops_per_s, int32_t* status,
                         cudaStream_t stream);

cudaError_t launch_prefill(const sq_packed_weight& w, int M, const int8_t* xq, const float* sx,
                           const float* x_out, const int32_t* idx, int n_out, float* y,
                           int32_t* T_out, int32_t* R_out, int32_t* status, cudaStream_t stream,
                           uint64_t wait_ns = 1000000000ull, int skip_group = -1);

}  // namespace sq
