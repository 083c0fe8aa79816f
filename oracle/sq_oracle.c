/*
 * sq_oracle.c -- plain single-threaded CPU oracle (test infrastructure only;
 * see sq_oracle.h for the sources, the conventions and what pins each part).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * Everything is written as the plain definition: loops in channel order,
 * binary64 arithmetic, int64 sums.  No blocking, no reordering.
 */
#include "sq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define SQO_OK 0
#define SQO_BAD_ARG 1
#define SQO_NONFINITE 2

static int64_t n_groups(int64_t K, int G) { return (K + G - 1) / G; }

static int valid_group(int G) { return G == 32 || G == 64 || G == 128; }

/* ---- quantizer ([P2] absmax section, [P3] s3.1) ------------------------ */

int sqo_quantize(double v, float s)
{
    if (s == 0.0f)
        return 0;
    double t = v / (double)s;     /* binary64 quotient */
    double r = round(t);          /* C round(): half away from zero */
    if (r > 127.0)
        r = 127.0;
    if (r < -127.0)
        r = -127.0;
    return (int)r;
}

float sqo_scale_from_absmax(double a)
{
    return (float)(a / 127.0);
}

int sqo_quantize_groups(const double *r, int64_t K, int G, int8_t *q, float *s)
{
    if (!r || !q || !s || K < 1 || G < 1)
        return SQO_BAD_ARG;
    for (int64_t g = 0; g * G < K; ++g) {
        int64_t j0 = g * G;
        int64_t j1 = j0 + G < K ? j0 + G : K;
        double a = 0.0;
        for (int64_t j = j0; j < j1; ++j)
            if (fabs(r[j]) > a)
                a = fabs(r[j]);
        s[g] = sqo_scale_from_absmax(a);
        for (int64_t j = j0; j < j1; ++j)
            q[j] = (int8_t)sqo_quantize(r[j], s[g]);
    }
    return SQO_OK;
}

/* ---- threshold ([P1] s5.2, s6.2) -------------------------------------- */

static int cmp_float(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

int sqo_trunk_threshold(const float *w, int64_t K, int P, float *tau)
{
    if (!w || !tau || K < 1 || P < 1 || P > 100)
        return SQO_BAD_ARG;
    float *a = (float *)malloc((size_t)K * sizeof(float));
    if (!a)
        return SQO_BAD_ARG;
    for (int64_t j = 0; j < K; ++j)
        a[j] = fabsf(w[j]);
    qsort(a, (size_t)K, sizeof(float), cmp_float);
    int64_t rank = ((int64_t)P * K + 99) / 100; /* ceil(P*K/100), >= 1 */
    *tau = a[rank - 1];
    free(a);
    return SQO_OK;
}

/* ---- decomposition ([P1] s2.1, s5.3, s6.2; [P2] BitNet weight sign) ---- */

int sqo_decompose(const float *W, int64_t N, int64_t K, int G, int P,
                  uint8_t *sign, uint8_t *mask, float *alpha, double *res,
                  int8_t *q, float *s)
{
    if (!W || !sign || !mask || !alpha || !q || !s || N < 1 || K < 1 ||
        !valid_group(G) || P == 0 || P > 100)
        return SQO_BAD_ARG;
    int64_t ng = n_groups(K, G);
    double *r = (double *)malloc((size_t)K * sizeof(double));
    if (!r)
        return SQO_BAD_ARG;
    int status = SQO_OK;
    for (int64_t row = 0; row < N; ++row) {
        const float *w = W + row * K;
        for (int64_t j = 0; j < K; ++j)
            if (!isfinite(w[j]))
                status = SQO_NONFINITE;

        /* trunk membership */
        float tau = -1.0f;
        if (P > 0)
            sqo_trunk_threshold(w, K, P, &tau);
        for (int64_t j = 0; j < K; ++j) {
            mask[row * K + j] = (uint8_t)(P < 0 ? 1 : (fabsf(w[j]) > tau));
            sign[row * K + j] = (uint8_t)(w[j] >= 0.0f);
        }

        /* alpha_r = mean |W| over the trunk, ascending-channel sum */
        double sum = 0.0;
        int64_t cnt = 0;
        for (int64_t j = 0; j < K; ++j)
            if (mask[row * K + j]) {
                sum += fabs((double)w[j]);
                cnt += 1;
            }
        float a = cnt ? (float)(sum / (double)cnt) : 0.0f;
        alpha[row] = a;

        /* residual W - trunk, then group-wise INT8 */
        for (int64_t j = 0; j < K; ++j) {
            double t = 0.0;
            if (mask[row * K + j])
                t = sign[row * K + j] ? (double)a : -(double)a;
            r[j] = (double)w[j] - t;
            if (res)
                res[row * K + j] = r[j];
        }
        sqo_quantize_groups(r, K, G, q + row * K, s + row * ng);
    }
    free(r);
    return status;
}

/* ---- outlier calibration ([P1] s2.2) ----------------------------------- */

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

int sqo_calibrate(const float *X, int64_t T, int64_t K, int k, int32_t *idx)
{
    if (!X || !idx || T < 1 || K < 1 || k < 1 || k > K)
        return SQO_BAD_ARG;
    int status = SQO_OK;
    float *mag = (float *)malloc((size_t)K * sizeof(float));
    uint8_t *taken = (uint8_t *)calloc((size_t)K, 1);
    if (!mag || !taken) {
        free(mag);
        free(taken);
        return SQO_BAD_ARG;
    }
    for (int64_t j = 0; j < K; ++j) {
        float m = 0.0f;
        for (int64_t t = 0; t < T; ++t) {
            float v = X[t * K + j];
            if (!isfinite(v))
                status = SQO_NONFINITE;
            else if (fabsf(v) > m)
                m = fabsf(v);
        }
        mag[j] = m;
    }
    /* selection: the largest remaining magnitude, lower channel on ties */
    for (int i = 0; i < k; ++i) {
        int64_t best = -1;
        for (int64_t j = 0; j < K; ++j)
            if (!taken[j] && (best < 0 || mag[j] > mag[best]))
                best = j;
        taken[best] = 1;
        idx[i] = (int32_t)best;
    }
    qsort(idx, (size_t)k, sizeof(int32_t), cmp_i32);
    free(mag);
    free(taken);
    return status;
}

/* ---- per-token activation split ([P1] s2.2, [P2] dynamic quantization) -- */

static int check_idx(const int32_t *idx, int n_out, int64_t K)
{
    if (n_out < 0 || (n_out > 0 && !idx))
        return 0;
    for (int i = 0; i < n_out; ++i) {
        if (idx[i] < 0 || idx[i] >= K)
            return 0;
        if (i > 0 && idx[i] <= idx[i - 1])
            return 0;
    }
    return 1;
}

int sqo_quantize_act(const float *x, int64_t M, int64_t K, const int32_t *idx,
                     int n_out, int8_t *xq, float *sx, float *xout)
{
    if (!x || !xq || !sx || M < 1 || K < 1 || !check_idx(idx, n_out, K) ||
        (n_out > 0 && !xout))
        return SQO_BAD_ARG;
    int status = SQO_OK;
    uint8_t *is_out = (uint8_t *)calloc((size_t)K, 1);
    if (!is_out)
        return SQO_BAD_ARG;
    for (int i = 0; i < n_out; ++i)
        is_out[idx[i]] = 1;
    for (int64_t t = 0; t < M; ++t) {
        const float *v = x + t * K;
        for (int i = 0; i < n_out; ++i)
            xout[t * n_out + i] = v[idx[i]];
        double a = 0.0;
        for (int64_t j = 0; j < K; ++j) {
            if (!isfinite(v[j]))
                status = SQO_NONFINITE;
            if (!is_out[j] && fabs((double)v[j]) > a)
                a = fabs((double)v[j]);
        }
        float s = sqo_scale_from_absmax(a);
        sx[t] = s;
        for (int64_t j = 0; j < K; ++j)
            xq[t * K + j] = is_out[j] ? 0 : (int8_t)sqo_quantize((double)v[j], s);
    }
    free(is_out);
    return status;
}

/* ---- integer accumulators ([P1] s2.3) ---------------------------------- */

int sqo_accumulate(int64_t M, int64_t N, int64_t K, int G,
                   const uint8_t *sign, const uint8_t *mask, const int8_t *q,
                   const int8_t *xq, int64_t *T, int64_t *R)
{
    if (M < 1 || N < 1 || K < 1 || !valid_group(G) || !sign || !mask || !q ||
        !xq || !T || !R)
        return SQO_BAD_ARG;
    int64_t ng = n_groups(K, G);
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            int64_t tr = 0;
            for (int64_t j = 0; j < K; ++j) {
                int64_t pm = 0; /* the +-1 / 0 trunk weight */
                if (mask[r * K + j])
                    pm = sign[r * K + j] ? 1 : -1;
                tr += pm * (int64_t)xq[t * K + j];
            }
            T[t * N + r] = tr;
            for (int64_t g = 0; g < ng; ++g) {
                int64_t acc = 0;
                for (int64_t j = g * G; j < (g + 1) * G && j < K; ++j)
                    acc += (int64_t)q[r * K + j] * (int64_t)xq[t * K + j];
                R[(t * N + r) * ng + g] = acc;
            }
        }
    return SQO_OK;
}

static int popcount32(uint32_t v)
{
    int c = 0;
    while (v) {
        c += (int)(v & 1u);
        v >>= 1;
    }
    return c;
}

int sqo_trunk_popcount(int64_t M, int64_t N, int64_t K, const uint8_t *sign,
                       const uint8_t *mask, const int8_t *xq, int64_t *T)
{
    if (M < 1 || N < 1 || K < 1 || !sign || !mask || !xq || !T)
        return SQO_BAD_ARG;
    int64_t nw = (K + 31) / 32;
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            int64_t total = 0;
            for (int64_t w = 0; w < nw; ++w) {
                uint32_t b = 0, m = 0, plane[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                for (int bit = 0; bit < 32; ++bit) {
                    int64_t j = w * 32 + bit;
                    if (j >= K)
                        break;
                    if (sign[r * K + j])
                        b |= 1u << bit;
                    if (mask[r * K + j])
                        m |= 1u << bit;
                    uint8_t byte = (uint8_t)xq[t * K + j]; /* two's complement */
                    for (int p = 0; p < 8; ++p)
                        if ((byte >> p) & 1u)
                            plane[p] |= 1u << bit;
                }
                for (int p = 0; p < 8; ++p) {
                    int64_t c = p < 7 ? ((int64_t)1 << p) : -128;
                    total += 2 * c * popcount32(m & b & plane[p]);
                    total -= c * popcount32(m & plane[p]);
                }
            }
            T[t * N + r] = total;
        }
    return SQO_OK;
}

/* ---- output ([P1] s2.3, s3.3; [P2] BitNet output rescale) -------------- */

static double dequant_weight(const uint8_t *sign, const uint8_t *mask,
                             const float *alpha, const int8_t *q, const float *s,
                             int64_t K, int64_t ng, int G, int64_t r, int64_t j)
{
    double t = 0.0;
    if (mask[r * K + j])
        t = sign[r * K + j] ? (double)alpha[r] : -(double)alpha[r];
    return t + (double)s[r * ng + j / G] * (double)q[r * K + j];
}

int sqo_linear(int64_t M, int64_t N, int64_t K, int G, const uint8_t *sign,
               const uint8_t *mask, const float *alpha, const int8_t *q,
               const float *s, const int8_t *xq, const float *sx,
               const float *xout, const int32_t *idx, int n_out, double *y)
{
    if (M < 1 || N < 1 || K < 1 || !valid_group(G) || !sign || !mask ||
        !alpha || !q || !s || !xq || !sx || !y || !check_idx(idx, n_out, K) ||
        (n_out > 0 && !xout))
        return SQO_BAD_ARG;
    int64_t ng = n_groups(K, G);
    int64_t *T = (int64_t *)malloc((size_t)(M * N) * sizeof(int64_t));
    int64_t *R = (int64_t *)malloc((size_t)(M * N * ng) * sizeof(int64_t));
    if (!T || !R) {
        free(T);
        free(R);
        return SQO_BAD_ARG;
    }
    sqo_accumulate(M, N, K, G, sign, mask, q, xq, T, R);
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            double inner = (double)alpha[r] * (double)T[t * N + r];
            for (int64_t g = 0; g < ng; ++g)
                inner += (double)s[r * ng + g] * (double)R[(t * N + r) * ng + g];
            double out = (double)sx[t] * inner;
            for (int i = 0; i < n_out; ++i)
                out += dequant_weight(sign, mask, alpha, q, s, K, ng, G, r, idx[i]) *
                       (double)xout[t * n_out + i];
            y[t * N + r] = out;
        }
    free(T);
    free(R);
    return SQO_OK;
}

int sqo_quantize_groups_asym(const double *r, int64_t K, int G, int8_t *q, float *s,
                             int32_t *z)
{
    if (!r || !q || !s || !z || K < 1 || !valid_group(G))
        return SQO_BAD_ARG;
    for (int64_t g = 0; g * G < K; ++g) {
        int64_t j0 = g * G;
        int64_t j1 = K < j0 + G ? K : j0 + G;
        double lo = r[j0], hi = r[j0];
        for (int64_t j = j0; j < j1; ++j) {
            if (r[j] < lo)
                lo = r[j];
            if (r[j] > hi)
                hi = r[j];
        }
        s[g] = (float)((hi - lo) / 255.0);
        if (s[g] == 0.0f) {
            z[g] = 0;
            for (int64_t j = j0; j < j1; ++j)
                q[j] = 0;
            continue;
        }
        double sd = (double)s[g];
        z[g] = (int32_t)round(-lo / sd - 128.0);
        for (int64_t j = j0; j < j1; ++j) {
            double v = round(r[j] / sd + (double)z[g]);
            if (v > 127.0)
                v = 127.0;
            if (v < -128.0)
                v = -128.0;
            q[j] = (int8_t)v;
        }
    }
    return SQO_OK;
}

int sqo_linear_asym(int64_t M, int64_t N, int64_t K, int G, const uint8_t *sign,
                    const uint8_t *mask, const float *alpha, const int8_t *q, const float *s,
                    const int32_t *z, const int8_t *xq, const float *sx, const float *xout,
                    const int32_t *idx, int n_out, double *y)
{
    if (M < 1 || N < 1 || K < 1 || !valid_group(G) || !sign || !mask || !alpha || !q || !s ||
        !z || !xq || !sx || !y || !check_idx(idx, n_out, K) || (n_out > 0 && !xout))
        return SQO_BAD_ARG;
    int64_t ng = n_groups(K, G);
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            int64_t T = 0;
            double inner = 0.0;
            for (int64_t g = 0; g < ng; ++g) {
                int64_t j0 = g * G, j1 = j0 + G < K ? j0 + G : K;
                int64_t R = 0, S = 0;
                for (int64_t j = j0; j < j1; ++j) {
                    int64_t x = xq[t * K + j];
                    if (mask[r * K + j])
                        T += sign[r * K + j] ? x : -x;
                    R += (int64_t)q[r * K + j] * x;
                    S += x;
                }
                inner += (double)s[r * ng + g] * (double)(R - (int64_t)z[r * ng + g] * S);
            }
            double out = (double)sx[t] * ((double)alpha[r] * (double)T + inner);
            for (int i = 0; i < n_out; ++i) {
                int64_t j = idx[i], g = j / G;
                double w = mask[r * K + j] ? (sign[r * K + j] ? (double)alpha[r] : -(double)alpha[r]) : 0.0;
                w += (double)s[r * ng + g] * (double)((int64_t)q[r * K + j] - z[r * ng + g]);
                out += w * (double)xout[t * n_out + i];
            }
            y[t * N + r] = out;
        }
    return SQO_OK;
}

static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

int sqo_sparsify_residual(const double *r, int64_t K, int G, int Ps, uint8_t *keep,
                          int8_t *q, float *s)
{
    if (!r || !keep || !q || !s || K < 1 || !valid_group(G) || Ps < 0 || Ps > 99)
        return SQO_BAD_ARG;
    double *a = (double *)malloc((size_t)K * sizeof(double));
    double *kept = (double *)malloc((size_t)K * sizeof(double));
    if (!a || !kept) {
        free(a);
        free(kept);
        return SQO_BAD_ARG;
    }
    for (int64_t j = 0; j < K; ++j)
        a[j] = fabs(r[j]);
    double theta = -1.0; /* Ps = 0: nothing dropped */
    if (Ps > 0) {
        qsort(a, (size_t)K, sizeof(double), cmp_double);
        int64_t rank = ((int64_t)Ps * K + 99) / 100; /* ceil(Ps*K/100), >= 1 */
        theta = a[rank - 1];
    }
    for (int64_t j = 0; j < K; ++j) {
        keep[j] = (uint8_t)(fabs(r[j]) > theta);
        kept[j] = keep[j] ? r[j] : 0.0;
    }
    int rc = sqo_quantize_groups(kept, K, G, q, s);
    free(a);
    free(kept);
    return rc;
}

int sqo_linear_trunk(int64_t M, int64_t N, int64_t K, const uint8_t *sign,
                     const uint8_t *mask, const float *alpha, const int8_t *xq,
                     const float *sx, const float *xout, const int32_t *idx, int n_out,
                     double *y)
{
    if (M < 1 || N < 1 || K < 1 || !sign || !mask || !alpha || !xq || !sx || !y ||
        !check_idx(idx, n_out, K) || (n_out > 0 && !xout))
        return SQO_BAD_ARG;
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            int64_t T = 0;  /* the direct +-1 sum over the trunk */
            for (int64_t j = 0; j < K; ++j)
                if (mask[r * K + j])
                    T += (sign[r * K + j] ? 1 : -1) * (int64_t)xq[t * K + j];
            double out = (double)sx[t] * ((double)alpha[r] * (double)T);
            for (int i = 0; i < n_out; ++i) {
                int64_t j = idx[i];
                double wt = mask[r * K + j] ? (sign[r * K + j] ? (double)alpha[r] : -(double)alpha[r]) : 0.0;
                out += wt * (double)xout[t * n_out + i];
            }
            y[t * N + r] = out;
        }
    return SQO_OK;
}

int sqo_linear_naive(int64_t M, int64_t N, int64_t K, int G, const uint8_t *sign,
                     const uint8_t *mask, const float *alpha, const int8_t *q,
                     const float *s, const int8_t *xq, const float *sx,
                     const float *xout, const int32_t *idx, int n_out, double *y)
{
    if (M < 1 || N < 1 || K < 1 || !valid_group(G) || !sign || !mask ||
        !alpha || !q || !s || !xq || !sx || !y || !check_idx(idx, n_out, K) ||
        (n_out > 0 && !xout))
        return SQO_BAD_ARG;
    int64_t ng = n_groups(K, G);
    double *xhat = (double *)malloc((size_t)K * sizeof(double));
    if (!xhat)
        return SQO_BAD_ARG;
    for (int64_t t = 0; t < M; ++t) {
        for (int64_t j = 0; j < K; ++j)
            xhat[j] = (double)xq[t * K + j] * (double)sx[t];
        for (int i = 0; i < n_out; ++i)
            xhat[idx[i]] = (double)xout[t * n_out + i];
        for (int64_t r = 0; r < N; ++r) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j)
                acc += dequant_weight(sign, mask, alpha, q, s, K, ng, G, r, j) * xhat[j];
            y[t * N + r] = acc;
        }
    }
    free(xhat);
    return SQO_OK;
}

int sqo_abs_dot(int64_t M, int64_t N, int64_t K, const float *W,
                const float *x, double *out)
{
    if (M < 1 || N < 1 || K < 1 || !W || !x || !out)
        return SQO_BAD_ARG;
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j)
                acc += fabs((double)W[r * K + j] * (double)x[t * K + j]);
            out[t * N + r] = acc;
        }
    return SQO_OK;
}

/* ---- per-layer fallback measure ([P1] s2.3, last paragraph) ------------- */

int sqo_layer_sq_error(int64_t N, int64_t K, int G, const float *W, const uint8_t *sign,
                       const uint8_t *mask, const float *alpha, const int8_t *q,
                       const float *s, const int32_t *z, double *err)
{
    if (N < 1 || K < 1 || !valid_group(G) || !W || !sign || !mask || !alpha || !q || !s || !err)
        return SQO_BAD_ARG;
    int64_t ng = n_groups(K, G);
    double total = 0.0;
    for (int64_t r = 0; r < N; ++r) {
        double e = 0.0;
        for (int64_t j = 0; j < K; ++j) {
            int64_t g = j / G;
            double t = mask[r * K + j] ? (sign[r * K + j] ? (double)alpha[r] : -(double)alpha[r]) : 0.0;
            int64_t zz = z ? (int64_t)z[r * ng + g] : 0;
            double what = t + (double)s[r * ng + g] * (double)((int64_t)q[r * K + j] - zz);
            double d = (double)W[r * K + j] - what;
            e += d * d;
        }
        total += e;
    }
    *err = total;
    return SQO_OK;
}

int sqo_plain_sq_error(int64_t N, int64_t K, int G, const float *W, double *err)
{
    if (N < 1 || K < 1 || !valid_group(G) || !W || !err)
        return SQO_BAD_ARG;
    double total = 0.0;
    for (int64_t r = 0; r < N; ++r) {
        double e = 0.0;
        for (int64_t j0 = 0; j0 < K; j0 += G) {
            const int64_t jend = (j0 + G < K) ? (j0 + G) : K;
            double a = 0.0;
            for (int64_t j = j0; j < jend; ++j)
                if (fabs((double)W[r * K + j]) > a)
                    a = fabs((double)W[r * K + j]);
            float sg = sqo_scale_from_absmax(a);
            for (int64_t j = j0; j < jend; ++j) {
                double w = (double)W[r * K + j];
                double d = w - (double)sg * (double)sqo_quantize(w, sg);
                e += d * d;
            }
        }
        total += e;
    }
    *err = total;
    return SQO_OK;
}

/* ---- NVFP4: the prefill format of format separation ---------------------
 * [P4] (the ISTA-DASLab page on separated quantization, paragraphs 2-4):
 * prefill runs in the hardware's native quantized format, NVFP4, while
 * decode keeps its own low-bit weight-only format.  The page names the
 * format without defining it; the reading taken is the format as the
 * Blackwell tensor cores consume it:
 *   element  E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; the
 *            magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 in code order 0..7, the
 *            sign in bit 3; a value that rounds to 0 is stored as +0;
 *   block    16 consecutive elements along K share one UE4M3 scale (no
 *            sign, 4 exponent bits with bias 7, 3 mantissa bits; largest
 *            finite 448, code 127 is NaN and never produced);
 *   second   a binary32 scale g = amax / (6 * 448) per weight tensor, and
 *   level    per token for activations.
 * Quantization of x in block b: s_b = RNE_ue4m3(amax_b / (6 g)), then
 * q = RNE_e2m1(x / (s_b g)), saturating at 6; ties go to the even code.  A
 * zero g or s_b gives all-zero codes.  The dequantized value is
 * e2m1(q) * s_b * g. */

static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double sqo_e2m1_value(int code)
{
    double m = kE2M1Mag[code & 7];
    return (code & 8) ? -m : m;
}

int sqo_e2m1_round(double v)
{
    double a = fabs(v);
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        double dc = fabs(a - kE2M1Mag[c]), db = fabs(a - kE2M1Mag[best]);
        if (dc < db || (dc == db && (c & 1) == 0))
            best = c;
    }
    if (best == 0)
        return 0;
    return v < 0.0 ? (best | 8) : best;
}

double sqo_ue4m3_value(int code)
{
    int e = (code >> 3) & 15, m = code & 7;
    if (e == 0)
        return ldexp((double)m, -9);
    return ldexp(1.0 + (double)m / 8.0, e - 7);
}

int sqo_ue4m3_round(double v)
{
    int best = 0;
    for (int c = 1; c < 127; ++c) {
        double dc = fabs(v - sqo_ue4m3_value(c)), db = fabs(v - sqo_ue4m3_value(best));
        if (dc < db || (dc == db && c % 2 == 0))
            best = c;
    }
    return best;
}

int sqo_nvfp4_quantize(const float *X, int64_t R, int64_t K, int per_row, uint8_t *codes,
                       uint8_t *scales, float *g)
{
    if (!X || !codes || !scales || !g || R < 1 || K < 1)
        return SQO_BAD_ARG;
    const int64_t nb = (K + 15) / 16;
    for (int64_t i = 0; i < R * K; ++i)
        if (!isfinite(X[i]))
            return SQO_NONFINITE;
    double amax_all = 0.0;
    if (!per_row)
        for (int64_t i = 0; i < R * K; ++i)
            if (fabs((double)X[i]) > amax_all)
                amax_all = fabs((double)X[i]);
    if (!per_row)
        g[0] = (float)(amax_all / 2688.0);
    for (int64_t r = 0; r < R; ++r) {
        const float *x = X + r * K;
        if (per_row) {
            double a = 0.0;
            for (int64_t j = 0; j < K; ++j)
                if (fabs((double)x[j]) > a)
                    a = fabs((double)x[j]);
            g[r] = (float)(a / 2688.0);
        }
        const double gr = (double)(per_row ? g[r] : g[0]);
        for (int64_t b = 0; b < nb; ++b) {
            int64_t j0 = 16 * b, j1 = j0 + 16 < K ? j0 + 16 : K;
            double ab = 0.0;
            for (int64_t j = j0; j < j1; ++j)
                if (fabs((double)x[j]) > ab)
                    ab = fabs((double)x[j]);
            int sc = gr == 0.0 ? 0 : sqo_ue4m3_round(ab / (6.0 * gr));
            scales[r * nb + b] = (uint8_t)sc;
            double step = sqo_ue4m3_value(sc) * gr;
            for (int64_t j = j0; j < j1; ++j)
                codes[r * K + j] = (uint8_t)(step == 0.0 ? 0 : sqo_e2m1_round((double)x[j] / step));
        }
    }
    return SQO_OK;
}

int sqo_nvfp4_linear(int64_t M, int64_t N, int64_t K, const uint8_t *wc, const uint8_t *ws,
                     float gw, const uint8_t *xc, const uint8_t *xs, const float *gx, double *y)
{
    if (!wc || !ws || !xc || !xs || !gx || !y || M < 1 || N < 1 || K < 1)
        return SQO_BAD_ARG;
    const int64_t nb = (K + 15) / 16;
    for (int64_t t = 0; t < M; ++t)
        for (int64_t r = 0; r < N; ++r) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j) {
                double w = sqo_e2m1_value(wc[r * K + j]) * sqo_ue4m3_value(ws[r * nb + j / 16]) *
                           (double)gw;
                double x = sqo_e2m1_value(xc[t * K + j]) * sqo_ue4m3_value(xs[t * nb + j / 16]) *
                           (double)gx[t];
                acc += w * x;
            }
            y[t * N + r] = acc;
        }
    return SQO_OK;
}
