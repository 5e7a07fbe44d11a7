/*
 * CPU oracle for the FP4 dense-attention path -- TEST INFRASTRUCTURE ONLY.
 * See oracle.h for what each function computes and which passage it follows.
 *
 * Build flags matter: this file must be compiled without -ffast-math and with
 * -ffp-contract=off so every fp32 operation is a single IEEE round-to-nearest
 * operation in the order written.
 */
#include "oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* Codecs.  Both are "round to the nearest representable value, ties to the  */
/* even code, saturate to the largest finite value": written as a search of  */
/* the ascending table of non-negative values.                               */
/* ------------------------------------------------------------------------ */

/* E2M1 magnitudes by code 0..7: exponent field e (2 bits, bias 1), mantissa m
 * (1 bit): e == 0 -> m * 0.5 ; else (1 + m/2) * 2^(e-1). */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* a >= 0 and a <= vals[n-1]: index of the nearest value, ties to even index. */
static int nearest_even(double a, const double* vals, int n) {
    int lo = 0, hi = n - 1; /* largest i with vals[i] <= a */
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (vals[mid] <= a) lo = mid; else hi = mid - 1;
    }
    if (lo == n - 1) return lo;
    double dlo = a - vals[lo], dhi = vals[lo + 1] - a; /* exact: dyadic values */
    if (dlo < dhi) return lo;
    if (dhi < dlo) return lo + 1;
    return (lo % 2 == 0) ? lo : lo + 1;
}

uint8_t oracle_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (isnan(x)) return sign | 0x7;
    if (a >= 6.0) return sign | 0x7; /* satfinite */
    return (uint8_t)(sign | nearest_even(a, kE2M1, 8));
}

float oracle_e2m1_decode(uint8_t code) {
    float v = (float)kE2M1[code & 0x7];
    return (code & 0x8) ? -v : v;
}

/* UE4M3 values by code 0..126 (127 = 0x7F is NaN in E4M3 and never used). */
static double kUE4M3[127];
static int kUE4M3_ready = 0;

float oracle_ue4m3_decode(uint8_t code) {
    int c = code & 0x7F;
    int e = c >> 3, m = c & 7;
    if (e == 0) return ldexpf((float)m, -9);           /* m/8 * 2^(1-7)   */
    return ldexpf((float)(8 + m), e - 10);             /* (1+m/8) * 2^(e-7) */
}

static void ue4m3_table(void) {
    if (kUE4M3_ready) return;
    for (int c = 0; c < 127; ++c) kUE4M3[c] = (double)oracle_ue4m3_decode((uint8_t)c);
    kUE4M3_ready = 1;
}

uint8_t oracle_ue4m3_encode(float x) {
    ue4m3_table();
    if (!(x > 0.0f)) return 0; /* zero, negative, NaN */
    double a = (double)x;
    if (a >= 448.0) return 0x7E; /* satfinite */
    return (uint8_t)nearest_even(a, kUE4M3, 127);
}

void oracle_e2m1_encode_array(const float* x, int64_t n, uint8_t* codes) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e2m1_encode(x[i]);
}

void oracle_ue4m3_encode_array(const float* x, int64_t n, uint8_t* codes) {
    ue4m3_table();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) codes[i] = oracle_ue4m3_encode(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Smooth K (page section "FP4 attention": subtract each head's mean key).   */
/* Reading: the mean is an exact fixed-point sum at 2^-24 resolution, so its */
/* bits do not depend on summation order.                                    */
/* ------------------------------------------------------------------------ */

int oracle_ksum(const uint16_t* k, int64_t BH, int64_t N, int64_t* S) {
    int err = ORACLE_OK;
    for (int64_t bh = 0; bh < BH; ++bh) {
        int64_t acc[128];
        for (int c = 0; c < 128; ++c) acc[c] = 0;
        for (int64_t n = 0; n < N; ++n) {
            for (int c = 0; c < 128; ++c) {
                float v = oracle_bf16_to_f32(k[(bh * N + n) * 128 + c]);
                if (!isfinite(v) || fabsf(v) >= 1048576.0f) { err = ORACLE_ERR_RANGE; continue; }
                double scaled = (double)v * 16777216.0;  /* exact */
                acc[c] += (int64_t)llrint(scaled);        /* ties to even */
            }
        }
        for (int c = 0; c < 128; ++c) S[bh * 128 + c] = acc[c];
    }
    return err;
}

void oracle_kmean(const int64_t* S, int64_t BH, int64_t N, float* mean) {
    for (int64_t i = 0; i < BH * 128; ++i) {
        double num = (double)S[i];
        double den = (double)N * 16777216.0;
        mean[i] = (float)(num / den);
    }
}

/* ------------------------------------------------------------------------ */
/* Hadamard rotation (page section "FP4 attention": the same orthonormal     */
/* Hadamard applied to Q and K).  Reading: Sylvester order, no sign flips,   */
/* butterflies with ascending stride, then one multiply by fp32 1/sqrt(128). */
/* ------------------------------------------------------------------------ */

void oracle_fwht128(float* x) {
    for (int h = 1; h < 128; h *= 2) {
        for (int i = 0; i < 128; ++i) {
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
        }
    }
}

float oracle_hadamard_scale(void) { return (float)(1.0 / sqrt(128.0)); }

static void transform_row(const uint16_t* row_bf16, const float* mean, uint32_t flags, float* y) {
    const float c = oracle_hadamard_scale();
    float x[128];
    for (int i = 0; i < 128; ++i) {
        float v = oracle_bf16_to_f32(row_bf16[i]);
        x[i] = mean ? (v - mean[i]) : v;
    }
    if (!(flags & ORACLE_NO_HADAMARD)) {
        oracle_fwht128(x);
        for (int i = 0; i < 128; ++i) x[i] = x[i] * c;
    }
    memcpy(y, x, sizeof x);
}

void oracle_transform_rows(const uint16_t* rows_bf16, int64_t rows, const float* mean,
                           uint32_t flags, float* y) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) transform_row(rows_bf16 + r * 128, mean, flags, y + r * 128);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 pack (page section "FP4 attention": E2M1 values, one E4M3 scale per */
/* 16 channels, a per-tensor global scale; block scale = amax / 6).          */
/* ------------------------------------------------------------------------ */

static void quantize_row(const float* y, float g, uint8_t* codes, uint8_t* scales) {
    for (int blk = 0; blk < 8; ++blk) {
        const float* yb = y + 16 * blk;
        float a = 0.0f;
        for (int i = 0; i < 16; ++i) {
            float m = fabsf(yb[i]);
            if (m > a) a = m;
        }
        float t = a / 6.0f;
        t = t / g;
        uint8_t s = oracle_ue4m3_encode(t);
        float sd = oracle_ue4m3_decode(s);
        float inv = 0.0f;
        if (sd != 0.0f) {
            float gs = g * sd;
            inv = 1.0f / gs;
        }
        scales[blk] = s;
        for (int i = 0; i < 16; i += 2) {
            float r0 = yb[i] * inv;
            float r1 = yb[i + 1] * inv;
            uint8_t c0 = oracle_e2m1_encode(r0);
            uint8_t c1 = oracle_e2m1_encode(r1);
            codes[8 * blk + i / 2] = (uint8_t)(c0 | (c1 << 4));
        }
    }
}

void oracle_quantize_rows(const float* y, int64_t rows, float g, uint8_t* codes, uint8_t* scales) {
    ue4m3_table();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) quantize_row(y + r * 128, g, codes + r * 64, scales + r * 8);
}

static int row_has_nonfinite(const uint16_t* row) {
    for (int i = 0; i < 128; ++i)
        if (!isfinite(oracle_bf16_to_f32(row[i]))) return 1;
    return 0;
}

int oracle_quantize_qk(const uint16_t* q, const uint16_t* k, int64_t B, int64_t H, int64_t N,
                       float gq, float gk, uint32_t flags,
                       uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales,
                       float* k_mean) {
    ue4m3_table();
    const int64_t BH = B * H;
    int err = ORACLE_OK;
    int64_t* S = (int64_t*)calloc((size_t)(BH * 128), sizeof(int64_t));
    float* mean = (float*)calloc((size_t)(BH * 128), sizeof(float));
    if (!(flags & ORACLE_NO_SMOOTH_K) && N > 0) {
        /* heads are independent: one thread per head */
        int herr = ORACLE_OK;
#pragma omp parallel for schedule(dynamic) reduction(max : herr)
        for (int64_t bh = 0; bh < BH; ++bh) {
            int e = oracle_ksum(k + bh * N * 128, 1, N, S + bh * 128);
            if (e > herr) herr = e;
        }
        if (herr) err = herr;
        oracle_kmean(S, BH, N, mean);
    }
    if (k_mean) memcpy(k_mean, mean, sizeof(float) * (size_t)(BH * 128));

    int qerr = ORACLE_OK;
#pragma omp parallel for schedule(static) reduction(max : qerr)
    for (int64_t row = 0; row < BH * N; ++row) {
        const int64_t bh = row / (N > 0 ? N : 1);
        float y[128];
        if (row_has_nonfinite(q + row * 128)) qerr = ORACLE_ERR_RANGE;
        transform_row(q + row * 128, NULL, flags, y);
        quantize_row(y, gq, q_codes + row * 64, q_scales + row * 8);
        if (row_has_nonfinite(k + row * 128)) qerr = ORACLE_ERR_RANGE;
        transform_row(k + row * 128, (flags & ORACLE_NO_SMOOTH_K) ? NULL : mean + bh * 128, flags, y);
        quantize_row(y, gk, k_codes + row * 64, k_scales + row * 8);
    }
    if (qerr) err = qerr;
    free(S);
    free(mean);
    return err;
}

/* ------------------------------------------------------------------------ */
/* Dynamic per-tensor scale.  The page's NVFP4 section ("NVFP4 QAD") names   */
/* scaling to the largest value as the plain alternative to calibrated       */
/* static scales; its attention uses a unit scale.  Reading: g maps the      */
/* largest magnitude of the transformed tensor (all heads, after smoothing   */
/* and rotation) to the top of the two-level range, 6 (E2M1) x 448 (E4M3):   */
/* g = fl32(amax / 2688), raised to 2^-64 when smaller (an all-zero tensor   */
/* included) so that g * scale and 1 / (g * scale) stay finite and normal.   */
/* ------------------------------------------------------------------------ */

static float tensor_gscale(float amax) {
    float g = amax / 2688.0f;
    const float g_min = 5.42101086242752217e-20f; /* 2^-64 */
    return g < g_min ? g_min : g;
}

int oracle_dynamic_gscale(const uint16_t* q, const uint16_t* k, int64_t B, int64_t H, int64_t N,
                          uint32_t flags, float* gq, float* gk) {
    const int64_t BH = B * H;
    int err = ORACLE_OK;
    float* mean = (float*)calloc((size_t)(BH * 128) + 1, sizeof(float));
    if (!(flags & ORACLE_NO_SMOOTH_K) && N > 0) {
        int64_t* S = (int64_t*)calloc((size_t)(BH * 128) + 1, sizeof(int64_t));
        int herr = ORACLE_OK;
#pragma omp parallel for schedule(dynamic) reduction(max : herr)
        for (int64_t bh = 0; bh < BH; ++bh) {
            int e = oracle_ksum(k + bh * N * 128, 1, N, S + bh * 128);
            if (e > herr) herr = e;
        }
        if (herr) err = herr;
        oracle_kmean(S, BH, N, mean);
        free(S);
    }
    float aq = 0.0f, ak = 0.0f;
    int rerr = ORACLE_OK;
#pragma omp parallel for schedule(static) reduction(max : aq, ak, rerr)
    for (int64_t row = 0; row < BH * N; ++row) {
        const int64_t bh = row / N;
        float y[128];
        if (row_has_nonfinite(q + row * 128) || row_has_nonfinite(k + row * 128)) rerr = ORACLE_ERR_RANGE;
        transform_row(q + row * 128, NULL, flags, y);
        for (int i = 0; i < 128; ++i)
            if (fabsf(y[i]) > aq) aq = fabsf(y[i]);
        transform_row(k + row * 128, (flags & ORACLE_NO_SMOOTH_K) ? NULL : mean + bh * 128, flags, y);
        for (int i = 0; i < 128; ++i)
            if (fabsf(y[i]) > ak) ak = fabsf(y[i]);
    }
    if (rerr) err = rerr;
    free(mean);
    *gq = tensor_gscale(aq);
    *gk = tensor_gscale(ak);
    return err;
}

void oracle_dequant(const uint8_t* codes, const uint8_t* scales, float g, int64_t rows, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int blk = 0; blk < 8; ++blk) {
            float gs = g * oracle_ue4m3_decode(scales[r * 8 + blk]);
            for (int i = 0; i < 16; ++i) {
                int e = 16 * blk + i;
                uint8_t byte = codes[r * 64 + e / 2];
                uint8_t code = (e % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                out[r * 128 + e] = gs * oracle_e2m1_decode(code);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Attention: softmax(Q K^T * scale) V in fp64 over the dequantised Q and K  */
/* (the exact result the tiled GPU kernel reaches with online softmax).      */
/* ------------------------------------------------------------------------ */

void oracle_attention_head(const float* qhat, const float* khat, const uint16_t* v,
                           int64_t N, double scale, const int64_t* rows, int64_t nrows,
                           double* O, double* lse) {
    if (rows == NULL) nrows = N;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < nrows; ++t) {
            const int64_t r = rows ? rows[t] : t;
            const float* q = qhat + r * 128;
            double mx = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                const float* kk = khat + j * 128;
                double dot = 0.0;
                for (int c = 0; c < 128; ++c) dot += (double)q[c] * (double)kk[c];
                s[j] = dot * scale;
                if (s[j] > mx) mx = s[j];
            }
            double l = 0.0;
            double o[128];
            for (int c = 0; c < 128; ++c) o[c] = 0.0;
            for (int64_t j = 0; j < N; ++j) {
                double p = exp(s[j] - mx);
                l += p;
                const uint16_t* vv = v + j * 128;
                for (int c = 0; c < 128; ++c) o[c] += p * (double)oracle_bf16_to_f32(vv[c]);
            }
            for (int c = 0; c < 128; ++c) O[t * 128 + c] = o[c] / l;
            lse[t] = mx + log(l);
        }
        free(s);
    }
}

/* ------------------------------------------------------------------------ */
/* Training-time backward (page section "NVFP4 QAD": 4-bit math on from the  */
/* first step of distillation; the summary list: the training-time FP4       */
/* attention matches the inference kernel).  Reading: fake quantisation with */
/* a straight-through estimator -- the attention gradients are taken at the  */
/* dequantised Q and K, and the quantiser passes them through unchanged, so  */
/* only the exact transforms (rotation, key centring) are differentiated.    */
/* ------------------------------------------------------------------------ */

/* Scores of query row i against all keys (fp64), and the row's lse. */
static double score_row(const float* q, const float* khat, int64_t N, double scale, double* s) {
    double mx = -INFINITY;
    for (int64_t j = 0; j < N; ++j) {
        const float* kk = khat + j * 128;
        double dot = 0.0;
        for (int c = 0; c < 128; ++c) dot += (double)q[c] * (double)kk[c];
        s[j] = dot * scale;
        if (s[j] > mx) mx = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < N; ++j) l += exp(s[j] - mx);
    return mx + log(l);
}

void oracle_attention_backward_head(const float* qhat, const float* khat, const uint16_t* v, const double* dO,
                                    const double* O_in, int64_t N, double scale, double* dqhat, double* dkhat,
                                    double* dv) {
    double* lse = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double* D = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    /* pass over queries: lse_i, D_i = sum_j P_ij dP_ij, dQhat_i = scale sum_j dS_ij khat_j */
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < N; ++i) {
            const double li = score_row(qhat + i * 128, khat, N, scale, s);
            const double* g = dO + i * 128;
            double Di = 0.0;
            if (O_in) { /* D from the given forward output: sum_c dO_ic O_ic */
                for (int c = 0; c < 128; ++c) Di += g[c] * O_in[i * 128 + c];
            } else {    /* the definition: sum_j P_ij dP_ij */
                for (int64_t j = 0; j < N; ++j) {
                    const uint16_t* vv = v + j * 128;
                    double dp = 0.0;
                    for (int c = 0; c < 128; ++c) dp += g[c] * (double)oracle_bf16_to_f32(vv[c]);
                    Di += exp(s[j] - li) * dp;
                }
            }
            lse[i] = li;
            D[i] = Di;
            /* second sweep for dS_ij = P_ij (dP_ij - D_i) */
            score_row(qhat + i * 128, khat, N, scale, s);
            double acc[128];
            for (int c = 0; c < 128; ++c) acc[c] = 0.0;
            for (int64_t j = 0; j < N; ++j) {
                const uint16_t* vv = v + j * 128;
                double dp = 0.0;
                for (int c = 0; c < 128; ++c) dp += g[c] * (double)oracle_bf16_to_f32(vv[c]);
                const double ds = exp(s[j] - li) * (dp - Di);
                const float* kk = khat + j * 128;
                for (int c = 0; c < 128; ++c) acc[c] += ds * (double)kk[c];
            }
            for (int c = 0; c < 128; ++c) dqhat[i * 128 + c] = scale * acc[c];
        }
        free(s);
    }
    /* pass over keys: dKhat_j = scale sum_i dS_ij qhat_i, dV_j = sum_i P_ij dO_i */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t j = 0; j < N; ++j) {
        const float* kk = khat + j * 128;
        const uint16_t* vv = v + j * 128;
        double ak[128], av[128];
        for (int c = 0; c < 128; ++c) ak[c] = av[c] = 0.0;
        for (int64_t i = 0; i < N; ++i) {
            const float* q = qhat + i * 128;
            const double* g = dO + i * 128;
            double dot = 0.0, dp = 0.0;
            for (int c = 0; c < 128; ++c) {
                dot += (double)q[c] * (double)kk[c];
                dp += g[c] * (double)oracle_bf16_to_f32(vv[c]);
            }
            const double p = exp(dot * scale - lse[i]);
            const double ds = p * (dp - D[i]);
            for (int c = 0; c < 128; ++c) {
                ak[c] += ds * (double)q[c];
                av[c] += p * g[c];
            }
        }
        for (int c = 0; c < 128; ++c) {
            dkhat[j * 128 + c] = scale * ak[c];
            dv[j * 128 + c] = av[c];
        }
    }
    free(lse);
    free(D);
}

/* fp64 Walsh-Hadamard transform of 128 values, the same Sylvester order as
 * the forward (the matrix is symmetric, so it is its own transpose). */
static void fwht128_f64(double* x) {
    for (int h = 1; h < 128; h *= 2)
        for (int i = 0; i < 128; ++i)
            if ((i & h) == 0) {
                const double a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
}

void oracle_ste_grads(const double* dqhat, const double* dkhat, int64_t N, uint32_t flags, double* dq, double* dk) {
    const double c = 1.0 / sqrt(128.0);
    double mean[128];
    for (int ch = 0; ch < 128; ++ch) mean[ch] = 0.0;
    if (!(flags & ORACLE_NO_SMOOTH_K) && N > 0) {
        for (int64_t n = 0; n < N; ++n)
            for (int ch = 0; ch < 128; ++ch) mean[ch] += dkhat[n * 128 + ch];
        for (int ch = 0; ch < 128; ++ch) mean[ch] /= (double)N;
    }
    for (int64_t n = 0; n < N; ++n) {
        double xq[128], xk[128];
        for (int ch = 0; ch < 128; ++ch) {
            xq[ch] = dqhat[n * 128 + ch];
            xk[ch] = dkhat[n * 128 + ch] - mean[ch];
        }
        if (!(flags & ORACLE_NO_HADAMARD)) {
            fwht128_f64(xq);
            fwht128_f64(xk);
            for (int ch = 0; ch < 128; ++ch) {
                xq[ch] *= c;
                xk[ch] *= c;
            }
        }
        memcpy(dq + n * 128, xq, sizeof xq);
        memcpy(dk + n * 128, xk, sizeof xk);
    }
}
