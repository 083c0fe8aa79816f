/*
 * sq_oracle.h -- plain, slow, single-threaded CPU oracle for the
 * "separated quantization" decode linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include,
 * link or call this code: only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg use it.  It shares no source with the
 * CUDA library and the CUDA library shares none with it.
 *
 * Sources (Chinese-language web pages on the method):
 *   [P1] "1-bit量化不是玄学..." (m.lqnn.cn/news/241359):
 *        s2.1 weight split  W ~ alpha*sign(W) + W_res,  W_res = W - alpha*sign(W),
 *             residual re-quantized to 8 bit, optional |W| > threshold trunk;
 *        s2.2 activation outlier channels kept at high precision, the rest
 *             INT8, outlier index detected once and cached;
 *        s2.3 trunk product by bit operations, residual by integer product,
 *             the two results summed;
 *        s5.2 threshold by a percentile of |W|;  s5.3 sep_linear pseudocode;
 *        s6.2 per-row (per output channel) scale and threshold.
 *   [P2] "visual guide to LLM quantization" (puppylpg.github.io):
 *        "对称量化以零为中心" absmax quantizer, range [-127,127];
 *        BitNet "权重量化": sign maps non-negative to +1, scale = mean |W|;
 *        "动态量化": per-token runtime scale;  Q4_K section: per-block scales.
 *   [P3] 2048ai.net quantization explainer, s3.1 "核心步骤": s = alpha/127,
 *        q = round(x/s), x = q*s, worked example alpha = 10.8.
 *
 * Arithmetic: IEEE binary64, round-to-nearest-even, no FMA contraction
 * (built with -ffp-contract=off), integer sums in int64.  The readings of
 * what the pages leave open are listed beside each function.
 *
 * Parity pins: every function here is pinned by the CPU tests against a
 * worked example from the pages, a closed form, an exact brute force or an
 * independent second route (see tests/test_oracle_pins.py).  The per-row
 * scale alpha is pinned only by closed-form rows whose mean |W| is exact.
 *
 * Unpacked conventions used by every function below (the oracle never packs
 * bits or pads rows; it works on one value per element):
 *   W      [N][K] float, row-major (N output rows, K input channels)
 *   sign   [N][K] uint8, 1 <=> W >= 0  (so +0.0 and -0.0 give 1)
 *   mask   [N][K] uint8, 1 <=> element belongs to the 1-bit trunk
 *   alpha  [N]    float
 *   res    [N][K] double, residual before rounding (may be NULL)
 *   q      [N][K] int8 residual codes
 *   s      [N][ng] float group scales, ng = ceil(K/G)
 *   idx    [n_out] int32 outlier channels, strictly ascending
 *   xq     [M][K] int8 activation codes (0 on outlier channels)
 *   sx     [M]    float per-token activation scale
 *   xout   [M][n_out] float outlier activations
 * Return value of the int functions: 0 = ok, 1 = invalid argument,
 * 2 = non-finite input.
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symmetric quantizer Q(v, s) ([P2] absmax, [P3] s3.1 divide convention):
 * s == 0 -> 0; otherwise clip(round(v / s), -127, 127) with the quotient in
 * binary64 and round() = half away from zero. */
int sqo_quantize(double v, float s);

/* Scale from an absolute maximum a: (float)(a / 127.0) ([P3] s3.1 step 2). */
float sqo_scale_from_absmax(double a);

/* Group-wise symmetric INT8 quantization of one residual row r[K]: groups of
 * G consecutive channels (the last one may be partial) each get their own
 * absmax scale ([P2] Q4_K block section; [P3] s2.3 per-group granularity). */
int sqo_quantize_groups(const double *r, int64_t K, int G, int8_t *q, float *s);

/* Per-row trunk threshold ([P1] s5.2 percentile, s6.2 per row): the
 * nearest-rank P-th percentile of |w|, i.e. the ceil(P*K/100)-th smallest
 * |w|.  1 <= P <= 100. */
int sqo_trunk_threshold(const float *w, int64_t K, int P, float *tau);

/* Offline decomposition ([P1] s2.1, s5.3, s6.2).  P < 0: every element is in
 * the trunk (mask all ones).  1 <= P <= 100: mask = |W| > tau_r (strict).
 * alpha_r = mean of |W| over the trunk members (ascending-channel binary64
 * sum, then one division, then rounding to float; 0 if the trunk is empty).
 * Residual r = W - mask*alpha*(2*sign-1) in binary64, quantized per group. */
int sqo_decompose(const float *W, int64_t N, int64_t K, int G, int P,
                  uint8_t *sign, uint8_t *mask, float *alpha, double *res,
                  int8_t *q, float *s);

/* Outlier calibration ([P1] s2.2): magnitude_j = max over T tokens |X_tj|;
 * the k channels of largest magnitude (ties: lower channel first), returned
 * in ascending channel order. */
int sqo_calibrate(const float *X, int64_t T, int64_t K, int k, int32_t *idx);

/* Per-token activation split ([P1] s2.2, [P2] "动态量化"): outlier channels
 * copied to xout; the absmax over the remaining channels gives sx; those
 * channels are quantized with Q; outlier slots of xq are 0. */
int sqo_quantize_act(const float *x, int64_t M, int64_t K, const int32_t *idx,
                     int n_out, int8_t *xq, float *sx, float *xout);

/* Exact integer accumulators ([P1] s2.3):
 *   T[t][r]     = sum_j mask*(2*sign-1)*xq_tj   (direct +-1 sum)
 *   R[t][r][g]  = sum_{j in group g} q_rj*xq_tj
 * T is [M][N], R is [M][N][ng]. */
int sqo_accumulate(int64_t M, int64_t N, int64_t K, int G,
                   const uint8_t *sign, const uint8_t *mask, const int8_t *q,
                   const int8_t *xq, int64_t *T, int64_t *R);

/* Second, independent route to T: sign and mask bits packed 32 per word,
 * xq split into its 8 two's-complement bit planes, and
 *   T = 2*sum_p c_p*popc(m & b & plane_p) - sum_p c_p*popc(m & plane_p)
 * with c_p = 2^p (p < 7) and c_7 = -128.  Result [M][N]. */
int sqo_trunk_popcount(int64_t M, int64_t N, int64_t K, const uint8_t *sign,
                       const uint8_t *mask, const int8_t *xq, int64_t *T);

/* Factored output ([P1] s2.3 two paths summed, s3.3 fused; [P2] BitNet
 * output rescale):
 *   y_tr = sx_t*(alpha_r*T_tr + sum_g s_rg*R_trg) + sum_i What_{r,idx_i}*xout_ti
 * What_rj = mask*alpha*(2*sign-1) + s_{r,g(j)}*q_rj.  All binary64. */
int sqo_linear(int64_t M, int64_t N, int64_t K, int G, const uint8_t *sign,
               const uint8_t *mask, const float *alpha, const int8_t *q,
               const float *s, const int8_t *xq, const float *sx,
               const float *xout, const int32_t *idx, int n_out, double *y);

/* Sparse residual (m.lqnn.cn news 241359, section 3.3, second point: a small
 * threshold zeroes the residual entries near zero, typically 50-70 % of
 * them, which are then stored in a sparse form).  For one residual row r[K]
 * (binary64): theta = the ceil(Ps*K/100)-th smallest |r_j| (nearest rank,
 * 1 <= Ps <= 99; Ps = 0 keeps every entry); keep[j] = (|r_j| > theta)
 * (strict: ties at theta are dropped); then the kept entries (the dropped
 * ones as 0) are quantized by groups of G exactly as sqo_quantize_groups. */
int sqo_sparsify_residual(const double *r, int64_t K, int G, int Ps, uint8_t *keep,
                          int8_t *q, float *s);

/* Asymmetric residual groups ([P1] section 2 pitfalls: the residual gets its
 * own min/max, scale and zero-point; [P3] asymmetric quantization, divide
 * form; INT8 range [-128, 127]).  Per group of G entries of r (binary64),
 * beta = min, alpha = max:
 *   s = (float)((alpha - beta) / 255)
 *   z = round(-beta / s - 128)            (half away from zero; any int)
 *   q = clip(round(r / s + z), -128, 127),  dequantized (q - z) * s;
 * alpha == beta (a constant group) gives s = 0, z = 0, q = 0. */
int sqo_quantize_groups_asym(const double *r, int64_t K, int G, int8_t *q, float *s,
                             int32_t *z);

/* Output with asymmetric residual groups:
 *   y_tr = sx_t*(alpha_r*T_tr + sum_g s_rg*(R_trg - z_rg*S_tg)) + sum_i What_{r,idx_i}*xout_ti
 * S_tg = sum_{j in g} xq_tj (exact), What_rj = trunk + s_{r,g(j)}*(q_rj - z_{r,g(j)}). */
int sqo_linear_asym(int64_t M, int64_t N, int64_t K, int G, const uint8_t *sign,
                    const uint8_t *mask, const float *alpha, const int8_t *q, const float *s,
                    const int32_t *z, const int8_t *xq, const float *sx, const float *xout,
                    const int32_t *idx, int n_out, double *y);

/* Trunk-only output (m.lqnn.cn news 241359, section 3.3: the 1-bit trunk is
 * computed first and the residual added on demand; a request may skip the
 * residual path).  The residual arrays are not read:
 *   y_tr = sx_t*alpha_r*T_tr + sum_i Wt_{r,idx_i}*xout_ti,
 *   Wt_rj = mask*alpha*(2*sign-1).  All binary64. */
int sqo_linear_trunk(int64_t M, int64_t N, int64_t K, const uint8_t *sign,
                     const uint8_t *mask, const float *alpha, const int8_t *xq,
                     const float *sx, const float *xout, const int32_t *idx, int n_out,
                     double *y);

/* Naive second route: y_tr = sum_j What_rj * xhat_tj with
 * xhat = xq*sx off the outlier set and x itself on it. */
int sqo_linear_naive(int64_t M, int64_t N, int64_t K, int G, const uint8_t *sign,
                     const uint8_t *mask, const float *alpha, const int8_t *q,
                     const float *s, const int8_t *xq, const float *sx,
                     const float *xout, const int32_t *idx, int n_out, double *y);

/* Reconstruction error of a decomposition over a layer (m.lqnn.cn news
 * 241359, section 2.3, last paragraph: a layer that gains nothing from the
 * split falls back to plain 8-bit; this is the measure compared):
 *   E = sum_r e_r,  e_r = sum_j (W_rj - What_rj)^2 in ascending j,
 *   What = mask*(sign ? alpha : -alpha) + s_g*(q - z_g)
 * with z = NULL for a symmetric residual (z_g = 0).  Binary64, rows in
 * order. */
int sqo_layer_sq_error(int64_t N, int64_t K, int G, const float *W, const uint8_t *sign,
                       const uint8_t *mask, const float *alpha, const int8_t *q,
                       const float *s, const int32_t *z, double *err);

/* The same error for plain symmetric INT8 groups of W itself (no trunk):
 * What = s_g*Q(W, s_g), s_g = float(absmax_g |W| / 127). */
int sqo_plain_sq_error(int64_t N, int64_t K, int G, const float *W, double *err);

/* Tolerance scale sum_j |W_rj * x_tj| from the original fp32 W and x, [M][N]. */
int sqo_abs_dot(int64_t M, int64_t N, int64_t K, const float *W,
                const float *x, double *out);

/* ---- NVFP4 prefill format ([P4], the ISTA-DASLab page on separated
 * quantization, paragraphs 2-4: prefill in the hardware's native NVFP4,
 * decode in its own weight-only format).  The page does not define the
 * format; the reading taken (the format the Blackwell tensor cores read):
 *   E2M1 elements (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; bit 3 = sign; a
 *   value rounding to 0 is +0), blocks of 16 along K with a UE4M3 scale
 *   (bias 7, 3 mantissa bits, largest 448), and a binary32 second-level
 *   scale g = amax / (6 * 448): per tensor for weights, per token (row) for
 *   activations.  s_b = RNE_ue4m3(amax_b / (6 g)); q = RNE_e2m1(x / (s_b g))
 *   saturating at 6; ties to the even code; g = 0 or s_b = 0 -> codes 0.
 *   Codes one per byte, [R][K]; scales [R][ceil(K/16)]. */
double sqo_e2m1_value(int code);
int sqo_e2m1_round(double v);
double sqo_ue4m3_value(int code);
int sqo_ue4m3_round(double v);  /* v >= 0 */
int sqo_nvfp4_quantize(const float *X, int64_t R, int64_t K, int per_row, uint8_t *codes,
                       uint8_t *scales, float *g);
/* y_tr = sum_j What_rj * xhat_tj (binary64, ascending j) with
 * What = e2m1(wc) * ue4m3(ws) * gw and xhat = e2m1(xc) * ue4m3(xs) * gx[t]. */
int sqo_nvfp4_linear(int64_t M, int64_t N, int64_t K, const uint8_t *wc, const uint8_t *ws,
                     float gw, const uint8_t *xc, const uint8_t *xs, const float *gx, double *y);

#ifdef __cplusplus
}
#endif
#endif /* SQ_ORACLE_H */
