/*
 * CPU oracle for the FP4 dense-attention path -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code with the CUDA library: it is a plain,
 * slow, scalar restatement of what the path computes, used to decide whether
 * the GPU results are right.
 *
 * Sources (FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention"):
 *   - smooth K: subtract each head's mean key before quantising; exact because
 *     softmax ignores a shift shared by every key;
 *   - rotate Q and K with the same orthonormal Hadamard matrix; exact because
 *     (qH)(kH)^T = q k^T;
 *   - NVFP4: E2M1 values with one E4M3 scale per 16 channels under a per-tensor
 *     (unit by default) global scale; P and V stay in BF16;
 *   - the block-scale figure caption on the yuxiaoba.github.io review page
 *     ("Quantization must account for both modalities"): sixteen values share a
 *     scale and a small one rounds to zero.
 * Details the pages leave open (rounding, scale rule amax/6, the fp32 order of
 * the Hadamard butterflies, how the mean is summed) follow the readings listed
 * in the repository's design notes; each function below names its reading.
 *
 * Parity pins: every function here is checked by the CPU test-suite against
 * something other than itself (format definitions, brute force, exact integer
 * arithmetic, scipy's Hadamard matrix, torch's fp64 SDPA, invariants).
 */
#ifndef FP4ATTN_ORACLE_H
#define FP4ATTN_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_OK = 0, ORACLE_ERR_RANGE = 4 };
enum { ORACLE_NO_SMOOTH_K = 1u, ORACLE_NO_HADAMARD = 2u };

/* bf16 bit pattern -> fp32 (exact). */
float oracle_bf16_to_f32(uint16_t b);

/* E2M1 (1 sign, 2 exponent, 1 mantissa bit; magnitudes 0,.5,1,1.5,2,3,4,6).
 * Encode: round to nearest, ties to the even code, saturate to +-6; the sign
 * bit (bit 3) follows the sign of x, zero included. */
uint8_t oracle_e2m1_encode(float x);
float oracle_e2m1_decode(uint8_t code);

/* Unsigned E4M3 scale (4 exponent bits, bias 7, 3 mantissa bits; finite max
 * 448, smallest subnormal 2^-9).  Encode: x >= 0, round to nearest, ties to
 * even, saturate to 448; x <= 0 or NaN gives 0. */
uint8_t oracle_ue4m3_encode(float x);
float oracle_ue4m3_decode(uint8_t code);

void oracle_e2m1_encode_array(const float* x, int64_t n, uint8_t* codes);
void oracle_ue4m3_encode_array(const float* x, int64_t n, uint8_t* codes);

/* Smooth-K step 1: exact fixed-point column sums of one or more heads.
 * S[bh][c] = sum_n round_half_even(k[bh][n][c] * 2^24) as int64.
 * Returns ORACLE_ERR_RANGE if any |k| >= 2^20 or k is not finite. */
int oracle_ksum(const uint16_t* k_bf16, int64_t BH, int64_t N, int64_t* S);

/* Smooth-K step 2: m = (float)((double)S / ((double)N * 2^24)). */
void oracle_kmean(const int64_t* S, int64_t BH, int64_t N, float* mean);

/* Unnormalised Sylvester Walsh-Hadamard transform of 128 fp32 values in the
 * pinned butterfly order: strides 1, 2, 4, ..., 64, each butterfly
 * (a, b) -> (a + b, a - b) in fp32 round-to-nearest. */
void oracle_fwht128(float* x);

/* The fp32 constant 1/sqrt(128) the transform is normalised with. */
float oracle_hadamard_scale(void);

/* Pre-quantisation transform of rows of 128: x = row - mean (fp32, K only;
 * mean may be NULL), then y = fl(fl(FWHT(x)) * (1/sqrt(128))) unless
 * ORACLE_NO_HADAMARD is set. */
void oracle_transform_rows(const uint16_t* rows_bf16, int64_t rows, const float* mean,
                           uint32_t flags, float* y);

/* NVFP4 pack of rows of 128 fp32 values with per-tensor scale g:
 * for each block of 16: a = max|y|, t = fl(fl(a/6)/g), s = UE4M3(t),
 * inv = (dec(s) == 0) ? 0 : fl(1/fl(g*dec(s))), code_i = E2M1(fl(y_i*inv)).
 * codes: 64 bytes per row, element 2i in the low nibble of byte i.
 * scales: 8 bytes per row. */
void oracle_quantize_rows(const float* y, int64_t rows, float g, uint8_t* codes, uint8_t* scales);

/* The whole prologue on [B,H,N,128] bf16 Q and K. k_mean may be NULL.
 * Returns ORACLE_OK or ORACLE_ERR_RANGE (non-finite input, |k| >= 2^20). */
int oracle_quantize_qk(const uint16_t* q, const uint16_t* k, int64_t B, int64_t H, int64_t N,
                       float gq, float gk, uint32_t flags,
                       uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales,
                       float* k_mean);

/* Dynamic per-tensor global scales of Q and K for oracle_quantize_qk: the
 * largest magnitude of each transformed tensor (smoothing and rotation as
 * selected by flags, over all B*H heads) mapped to 6 * 448, that is
 * g = fl32(amax / 2688), raised to 2^-64 when smaller.  Returns ORACLE_OK, or
 * ORACLE_ERR_RANGE for a non-finite input or |k| >= 2^20 (g then unspecified). */
int oracle_dynamic_gscale(const uint16_t* q, const uint16_t* k, int64_t B, int64_t H, int64_t N,
                          uint32_t flags, float* gq, float* gk);

/* Dequantise rows: out = fl(fl(g * dec(scale)) * e2m1(code)). */
void oracle_dequant(const uint8_t* codes, const uint8_t* scales, float g, int64_t rows, float* out);

/* Exact (fp64) attention of one head over dequantised Q and K and bf16 V:
 * for each requested query row r:
 *   s_j = scale * sum_c qhat[r][c] * khat[j][c]   (fp64)
 *   O[r] = sum_j exp(s_j - max) v_j / sum_j exp(s_j - max),
 *   lse[r] = max + ln(sum_j exp(s_j - max)).
 * rows == NULL means all N rows in order. */
void oracle_attention_head(const float* qhat, const float* khat, const uint16_t* v_bf16,
                           int64_t N, double scale, const int64_t* rows, int64_t nrows,
                           double* O, double* lse);

/* Number of OpenMP threads the oracle uses. */
int oracle_num_threads(void);

/* Backward of oracle_attention_head for one head (fp64 throughout), the
 * training-time gradient at the dequantised Q and K:
 *   P = softmax(scale * qhat khat^T), O = P V, dP = dO V^T,
 *   D_i = sum_j P_ij dP_ij, dS = P * (dP - D),
 *   dqhat = scale * dS khat, dkhat = scale * dS^T qhat, dv = P^T dO.
 * qhat, khat: fp32 [N,128]; v: bf16 bits [N,128]; dO: fp64 [N,128];
 * outputs fp64 [N,128].  O_in: NULL, or a forward output [N,128] from which
 * D is taken instead (D_i = sum_c dO_ic O_in_ic, equal to the definition when
 * O_in is the exact O): the backward's contract when the caller supplies the
 * forward's stored output. */
void oracle_attention_backward_head(const float* qhat, const float* khat, const uint16_t* v_bf16,
                                    const double* dO, const double* O_in, int64_t N, double scale,
                                    double* dqhat, double* dkhat, double* dv);

/* Straight-through estimator of the prologue for one head: the quantiser
 * passes gradients unchanged, the exact transforms are differentiated.
 *   dq_n = c * H dqhat_n,  dk_n = c * H (dkhat_n - mean_n' dkhat_n'),
 * with c = 1/sqrt(128) and H the Sylvester Hadamard matrix (symmetric); the
 * centring is the Jacobian of the key mean (skipped with ORACLE_NO_SMOOTH_K),
 * the rotation skipped with ORACLE_NO_HADAMARD.  fp64 in and out, [N,128]. */
void oracle_ste_grads(const double* dqhat, const double* dkhat, int64_t N, uint32_t flags, double* dq,
                      double* dk);

#ifdef __cplusplus
}
#endif
#endif
