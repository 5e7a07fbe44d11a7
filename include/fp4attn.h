/*
 * fp4attn -- FP4 dense attention for long non-causal sequences on NVIDIA B200.
 *
 * C ABI of the CUDA library (nvfp4_precision_b200/libfp4attn.so).  Plain
 * pointers and sizes only; every call is stream-ordered and asynchronous
 * unless stated otherwise.  The library allocates no memory and keeps no
 * state between calls: the caller owns every buffer, including the small
 * workspace that holds the device-side status word and the key-mean sums.
 *
 * The method (FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention"):
 *   1. smooth K: subtract each head's mean key (exact for softmax, since
 *      q.(k_j - kbar) = q.k_j - q.kbar is a shift shared by every key);
 *   2. rotate Q and K by the same orthonormal 128x128 Hadamard matrix (exact,
 *      since (qH).(kH) = q.k; spreads outlier channels across scale blocks);
 *   3. quantise Q and K to NVFP4: E2M1 values with one E4M3 scale per 16
 *      channels under an fp32 per-tensor scale (unit by default);
 *   4. softmax(Q K^T * scale) V with Q K^T from the FP4 operands and P, V in
 *      BF16, non-causal, dense.
 * Also here: the same attention with BF16 Q and K (the layers kept in BF16),
 * an optional dynamic per-tensor scale (section "NVFP4 QAD": scaling to the
 * largest value), and the training-time straight-through backward.
 * Details the pages leave open are fixed as follows: block scale amax/6,
 * round-to-nearest-even with saturation for both formats, Sylvester-ordered
 * Hadamard applied as seven fp32 butterfly stages of ascending stride followed
 * by one multiply by fp32(1/sqrt(128)), and an exact int64 fixed-point key sum
 * (2^-24 resolution) so the mean does not depend on summation order.
 *
 * Layouts (row-major, head dim D = 128; contiguous for the plain entry points,
 * any strides for the bf16 tensors of the *_ex entry points, see
 * fp4attn_strides):
 *   Q, K, V      bf16  [B, H, N, 128]
 *   codes        uint8 [B, H, N, 64]   element 2i in the low nibble of byte i;
 *                                      sign in bit 3 of each nibble
 *   scales       uint8 [B, H, N, 8]    UE4M3 scale of channels 16j..16j+15
 *   k_mean       fp32  [B, H, 128]
 *   O            bf16  [B, H, N, 128]
 *   lse          fp32  [B, H, N]       natural-log sum of exp of the scaled logits
 * Heads of D = 64 channels (the page's toy heads: section "FP4 attention",
 * 64 channels in four 16-value blocks) are taken by fp4attn_quantize_qk,
 * fp4attn_quantize_qk_ex (static global scales), fp4attn_forward,
 * fp4attn_forward_ex and the dequantisers: Q, K, V and O are [B, H, N, 64],
 * codes [B, H, N, 32], scales [B, H, N, 4], k_mean [B, H, 64]; the rotation
 * is the 64-point transform (six butterfly stages) times fp32(1/sqrt(64)),
 * and softmax_scale <= 0 selects 1/sqrt(64).  The other entry points take
 * D = 128 only.
 * Every pointer must be 16-byte aligned.  Pointers named *_dev are device
 * pointers (cudaMalloc / torch CUDA tensors); none may alias another output.
 *
 * Error behaviour: argument errors are returned synchronously and nothing is
 * launched.  A failed launch returns FP4ATTN_ERR_CUDA (the CUDA error is
 * cleared).  Errors found on the device (non-finite or out-of-range input,
 * a bounded wait that ran out) are written to the workspace status word and
 * read with fp4attn_read_status.  No call exits the process or traps.
 */
#ifndef FP4ATTN_H
#define FP4ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4ATTN_OK = 0,
    FP4ATTN_ERR_INVALID_ARG = 1,  /* bad shape, NULL or misaligned pointer      */
    FP4ATTN_ERR_UNSUPPORTED = 2,  /* valid but not supported (e.g. D = 96)      */
    FP4ATTN_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed          */
    FP4ATTN_ERR_RANGE = 4,        /* device: non-finite input, |k| >= 2^20, g<=0 */
    FP4ATTN_ERR_TIMEOUT = 5,      /* device: a bounded wait ran out             */
    FP4ATTN_ERR_WORKSPACE = 6     /* workspace missing or too small             */
} fp4attn_status;

/* Flags of fp4attn_quantize_qk (0 = the full method).  Both exist for
 * ablation and for checking the quantiser on its own. */
enum {
    FP4ATTN_NO_SMOOTH_K = 1u,  /* do not subtract the key mean (k_mean reports 0) */
    FP4ATTN_NO_HADAMARD = 2u,  /* do not rotate Q and K                           */
    /* fp4attn_quantize_qk_ex only: compute each tensor's global scale from its
     * largest transformed magnitude instead of taking it from the caller. */
    FP4ATTN_DYNAMIC_GSCALE = 4u
};

typedef struct {
    int32_t B, H, N, D;  /* D = 128 (or 64 where stated); B, H, N >= 0; N <= 262144 */
} fp4attn_shape;

/* Element strides of a bf16 tensor indexed [b][h][n][c] (c, the D channels,
 * always contiguous).  Each stride must be a positive multiple of 8 elements
 * (16 bytes) below 2^39; the stride of a dimension of size 1 is ignored.  The
 * contiguous [B,H,N,128] layout is {H*N*128, N*128, 128}; a [B,N,H,128]
 * tensor (the layout a QKV projection produces) is {N*H*128, 128, H*128}. */
typedef struct {
    int64_t b, h, n;
} fp4attn_strides;

/* Bytes of workspace that fp4attn_quantize_qk and fp4attn_forward need for
 * this shape (status word, per-head int64 key sums).  Never 0. */
size_t fp4attn_workspace_bytes(fp4attn_shape s);

/* Smooth K + Hadamard + NVFP4 pack of Q and K (method steps 1-3).
 *   q_bf16_dev, k_bf16_dev : [B,H,N,128] bf16 inputs.
 *   q_gscale_dev, k_gscale_dev : device fp32 scalars g (finite, > 0), or NULL
 *     for 1.0.  Block scale s = UE4M3(amax / 6 / g); the value of a code is
 *     g * s * e2m1.
 *   flags : FP4ATTN_NO_SMOOTH_K | FP4ATTN_NO_HADAMARD, or 0 (a dynamic
 *     global scale needs fp4attn_quantize_qk_ex).
 *   q_codes_dev, k_codes_dev : [B,H,N,64] out.  q_scales_dev, k_scales_dev :
 *     [B,H,N,8] out.  k_mean_dev : [B,H,128] fp32 out, or NULL.
 *   workspace_dev : fp4attn_workspace_bytes(s) bytes; cleared by this call.
 * Device errors: FP4ATTN_ERR_RANGE for a non-finite Q or K value, |k| >= 2^20
 * (the key sum would leave its exact range) or g not finite and > 0; the
 * affected outputs are unspecified. */
int fp4attn_quantize_qk(const void* q_bf16_dev, const void* k_bf16_dev, fp4attn_shape s,
                        const float* q_gscale_dev, const float* k_gscale_dev, uint32_t flags,
                        uint8_t* q_codes_dev, uint8_t* q_scales_dev,
                        uint8_t* k_codes_dev, uint8_t* k_scales_dev, float* k_mean_dev,
                        void* workspace_dev, size_t workspace_bytes, cudaStream_t stream);

/* fp4attn_quantize_qk for Q and K of any strides (fp4attn_strides), with an
 * optional dynamic global scale.  The codes, scales and k_mean outputs keep the
 * layouts of fp4attn_quantize_qk.
 *   flags : as for fp4attn_quantize_qk, plus FP4ATTN_DYNAMIC_GSCALE (D = 128
 *     only; FP4ATTN_ERR_UNSUPPORTED for D = 64).
 *   q_gscale_dev, k_gscale_dev : without FP4ATTN_DYNAMIC_GSCALE, inputs as for
 *     fp4attn_quantize_qk (NULL for 1.0).  With it, both must be non-NULL and
 *     receive g = fl32(amax / (6 * 448)), raised to 2^-64 when smaller, where
 *     amax is the largest magnitude of the whole transformed tensor (after
 *     smoothing and rotation, over all B*H heads); the block holding that
 *     value gets scale 448 and code 6.  Pass the same pointers to
 *     fp4attn_forward.  This reads Q and K twice (two kernel launches).
 *     Source: FastVideo "Pika H3 Flex in FastVideo", section "NVFP4 QAD"
 *     (scaling to the largest value, the plain alternative to calibrated
 *     static scales) and section "FP4 attention" (the per-tensor scale).
 * Errors as for fp4attn_quantize_qk; FP4ATTN_ERR_INVALID_ARG for a bad stride
 * or a NULL scale pointer with FP4ATTN_DYNAMIC_GSCALE. */
int fp4attn_quantize_qk_ex(const void* q_bf16_dev, fp4attn_strides q_strides,
                           const void* k_bf16_dev, fp4attn_strides k_strides, fp4attn_shape s,
                           float* q_gscale_dev, float* k_gscale_dev, uint32_t flags,
                           uint8_t* q_codes_dev, uint8_t* q_scales_dev,
                           uint8_t* k_codes_dev, uint8_t* k_scales_dev, float* k_mean_dev,
                           void* workspace_dev, size_t workspace_bytes, cudaStream_t stream);

/* Non-causal attention over NVFP4 Q and K and bf16 V (method step 4):
 *   O = softmax(scale * gQ * gK * (Qc K c^T)) V,  Qc, Kc the block-scaled E2M1
 *   values; Q K^T on the FP4 tensor cores with fp32 accumulation, P rounded to
 *   bf16 for P.V, fp32 accumulation, online softmax.
 *   softmax_scale : <= 0 selects 1/sqrt(D).
 *   o_bf16_dev : [B,H,N,128] out.  lse_dev : [B,H,N] out or NULL.
 *   workspace_dev : as for fp4attn_quantize_qk (status word only; not cleared).
 * Device errors: FP4ATTN_ERR_RANGE for a bad g; FP4ATTN_ERR_TIMEOUT if an
 * internal wait ran out (the output is then incomplete). */
int fp4attn_forward(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev,
                    const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                    const float* q_gscale_dev, const float* k_gscale_dev,
                    const void* v_bf16_dev, fp4attn_shape s, float softmax_scale,
                    void* o_bf16_dev, float* lse_dev,
                    void* workspace_dev, size_t workspace_bytes, cudaStream_t stream);

/* fp4attn_forward with V and O of any strides (fp4attn_strides); lse stays
 * [B,H,N].  O's rows must not overlap one another or any input.  Errors as
 * for fp4attn_forward; FP4ATTN_ERR_INVALID_ARG for a bad stride. */
int fp4attn_forward_ex(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev,
                       const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                       const float* q_gscale_dev, const float* k_gscale_dev,
                       const void* v_bf16_dev, fp4attn_strides v_strides, fp4attn_shape s,
                       float softmax_scale, void* o_bf16_dev, fp4attn_strides o_strides, float* lse_dev,
                       void* workspace_dev, size_t workspace_bytes, cudaStream_t stream);

/* The same non-causal attention with Q and K in BF16 instead of NVFP4: the
 * baseline the FP4 kernel is measured against, and the path for layers kept in
 * BF16 (FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention": two of
 * the model's attention blocks stay in BF16).  S = Q K^T runs on the BF16
 * tensor cores with fp32 accumulation; softmax, P (bf16) and P V are as in
 * fp4attn_forward.  No smoothing, rotation or quantisation is applied.
 *   q_bf16_dev, k_bf16_dev, v_bf16_dev : [B,H,N,128] bf16.
 *   softmax_scale : <= 0 selects 1/sqrt(D).
 *   o_bf16_dev : [B,H,N,128] out.  lse_dev : [B,H,N] out or NULL.
 *   workspace_dev : as for fp4attn_forward (status word only; not cleared).
 * Device errors: FP4ATTN_ERR_TIMEOUT if an internal wait ran out. */
int fp4attn_forward_bf16qk(const void* q_bf16_dev, const void* k_bf16_dev, const void* v_bf16_dev,
                           fp4attn_shape s, float softmax_scale, void* o_bf16_dev, float* lse_dev,
                           void* workspace_dev, size_t workspace_bytes, cudaStream_t stream);

/* fp4attn_forward_bf16qk with Q, K, V and O of any strides (fp4attn_strides);
 * lse stays [B,H,N].  O's rows must not overlap one another or any input. */
int fp4attn_forward_bf16qk_ex(const void* q_bf16_dev, fp4attn_strides q_strides,
                              const void* k_bf16_dev, fp4attn_strides k_strides,
                              const void* v_bf16_dev, fp4attn_strides v_strides, fp4attn_shape s,
                              float softmax_scale, void* o_bf16_dev, fp4attn_strides o_strides,
                              float* lse_dev, void* workspace_dev, size_t workspace_bytes,
                              cudaStream_t stream);

/* fp4attn_quantize_qk without a workspace argument.  The pages have no
 * counterpart to this entry point: it exists for callers that cannot allocate
 * device memory for the workspace -- cudaMalloc/cudaFree may synchronise the
 * whole device, which a latency-bound caller sharing the GPU cannot afford,
 * and some callers run where another allocator owns all device memory and
 * raw allocations are not allowed.  It allocates nothing: its scratch (status
 * word, ticket, key sums) is a fixed array of about 1 MB in the library's
 * device memory, held by every GPU that loads the library until the process
 * exits.  The caller still passes every input and output, as for
 * fp4attn_quantize_qk, whose arguments and results this call shares.
 *   status_dev : device int32 that receives the device status word of this
 *     call (FP4ATTN_OK or the first device error), or NULL.
 * Limits and behaviour:
 *   - B*H at most 1024; larger shapes return FP4ATTN_ERR_UNSUPPORTED and
 *     launch nothing;
 *   - the first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process: after cudaDeviceReset (or anything else that tears down the
 *     device's primary context) it is stale, so do not call this entry point
 *     on that device again;
 *   - every call shares the one array and clears what must start at zero on
 *     its stream; calls that overlap on the GPU (other streams, other host
 *     threads) race on it and must be serialised by the caller. */
int fp4attn_quantize_qk_noalloc(const void* q_bf16_dev, const void* k_bf16_dev, fp4attn_shape s,
                                const float* q_gscale_dev, const float* k_gscale_dev, uint32_t flags,
                                uint8_t* q_codes_dev, uint8_t* q_scales_dev,
                                uint8_t* k_codes_dev, uint8_t* k_scales_dev, float* k_mean_dev,
                                int* status_dev, cudaStream_t stream);

/* Training-time attention (FastVideo "Pika H3 Flex in FastVideo", section
 * "NVFP4 QAD": the 4-bit student trains with 4-bit math on from the first
 * step; the summary list: the training-time FP4 attention matches the
 * inference kernel).  The forward is the inference path (fp4attn_quantize_qk,
 * fp4attn_forward with lse); the backward below is a straight-through
 * estimator: attention gradients at the dequantised Q^ = gQ Q~ and
 * K^ = gK K~ (Q~, K~ the unit-scale values of the NVFP4 codes), passed
 * unchanged through the quantiser, then the exact transforms differentiated:
 *   P = exp(scale Q^K^T - lse), dP = dO V^T, D = rowsum(dO * O),
 *   dS = P * (dP - D), dV = P^T dO, dQ^ = scale dS K^, dK^ = scale dS^T Q^,
 *   dq = c H dQ^, dk = c H (dK^ - mean_n dK^)   (c = 1/sqrt(128)).
 * Both kernels compute their scores (S, and S^T on the key side) from the
 * codes with the forward's block-scaled FP4 MMA (the scores the forward's lse
 * was taken over); the products dQ^ += dS K~ and dK^ += dS^T Q~ take Q~, K~
 * in bf16 (exact), which this call dequantises into the workspace.  P and dS
 * are rounded to bf16 for the BF16 tensor-core products, which accumulate in
 * fp32; dq, dk, dv are bf16.  The global
 * scales are applied as scalars (in the softmax scale and the dQ^ / dK^
 * factors), never by rounding gQ * Q~ to bf16.
 *   q_codes_dev, q_scales_dev, k_codes_dev, k_scales_dev : the forward's
 *     NVFP4 Q and K from fp4attn_quantize_qk ([B,H,N,64] / [B,H,N,8]).
 *   q_gscale_dev, k_gscale_dev : the forward's global scales (device fp32
 *     scalars, finite and > 0), or NULL for 1.0.
 *   v_dev, o_dev, do_dev : [B,H,N,128] bf16: V, the forward's O and dL/dO.
 *   lse_dev : [B,H,N] fp32 from the forward.
 *   softmax_scale : that of the forward (<= 0 selects 1/sqrt(128)).
 *   flags : the forward's FP4ATTN_NO_SMOOTH_K / FP4ATTN_NO_HADAMARD.
 *   dq_dev, dk_dev, dv_dev : [B,H,N,128] bf16 out: gradients of the bf16 Q,
 *     K (the prologue's inputs) and V.
 *   workspace_dev : fp4attn_backward_workspace_bytes(s) bytes (status word
 *     first, so fp4attn_read_status works on it; about 1 KB per row).
 * All tensors contiguous.  Device errors: FP4ATTN_ERR_RANGE for a bad global
 * scale; FP4ATTN_ERR_TIMEOUT if an internal wait ran out. */
size_t fp4attn_backward_workspace_bytes(fp4attn_shape s);
int fp4attn_backward(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev, const uint8_t* k_codes_dev,
                     const uint8_t* k_scales_dev, const float* q_gscale_dev, const float* k_gscale_dev,
                     const void* v_dev, const void* o_dev, const void* do_dev, const float* lse_dev,
                     fp4attn_shape s, float softmax_scale, uint32_t flags, void* dq_dev, void* dk_dev,
                     void* dv_dev, void* workspace_dev, size_t workspace_bytes, cudaStream_t stream);

/* fp4attn_backward with V, O, dO and the outputs dq, dk, dv in one layout of
 * any element strides (fp4attn_strides; e.g. [B,N,H,128] as a QKV projection
 * writes them); the codes, scales and lse keep their layouts (the library's
 * own outputs).  The outputs' rows must not overlap one another or any
 * input.  Errors as for fp4attn_backward; FP4ATTN_ERR_INVALID_ARG for a bad
 * stride. */
int fp4attn_backward_ex(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev, const uint8_t* k_codes_dev,
                        const uint8_t* k_scales_dev, const float* q_gscale_dev, const float* k_gscale_dev,
                        const void* v_dev, const void* o_dev, const void* do_dev, fp4attn_strides io_strides,
                        const float* lse_dev, fp4attn_shape s, float softmax_scale, uint32_t flags,
                        void* dq_dev, void* dk_dev, void* dv_dev, void* workspace_dev, size_t workspace_bytes,
                        cudaStream_t stream);

/* Decode NVFP4 rows to bf16: out = bf16(fl(fl(g * s) * e2m1)), exact when
 * g = 1.  codes_dev [rows,64], scales_dev [rows,8], gscale_dev scalar or
 * NULL, out_dev bf16 [rows,128], rows = B*H*N of s. */
int fp4attn_dequant_bf16(const uint8_t* codes_dev, const uint8_t* scales_dev, const float* gscale_dev,
                         fp4attn_shape s, void* out_dev, cudaStream_t stream);

/* Testing: decode NVFP4 rows back to fp32, out = fl(fl(g * s) * e2m1).
 *   codes_dev [rows,64], scales_dev [rows,8], gscale_dev scalar or NULL,
 *   out_dev fp32 [rows,128], rows = B*H*N of s. */
int fp4attn_dequant(const uint8_t* codes_dev, const uint8_t* scales_dev, const float* gscale_dev,
                    fp4attn_shape s, float* out_dev, cudaStream_t stream);

/* Read (synchronously: waits for the stream) and return in *device_status the
 * workspace status word: FP4ATTN_OK or the first device error. */
int fp4attn_read_status(const void* workspace_dev, cudaStream_t stream, int* device_status);

/* Reset the workspace status word to FP4ATTN_OK (stream-ordered). */
int fp4attn_reset_status(void* workspace_dev, cudaStream_t stream);

/* Static description of a status code. */
const char* fp4attn_status_string(int code);

/* ---- test hooks: the same device building blocks, exposed for unit tests ---- */

/* Element-wise fp32 -> E2M1 code (low nibble; sign in bit 3) and -> E4M3 byte
 * with the device conversions the quantiser uses (round to nearest even,
 * saturating).  n elements; either output may be NULL. */
int fp4attn_encode_f32(const float* x_dev, int64_t n, uint8_t* e2m1_dev, uint8_t* e4m3_dev,
                       cudaStream_t stream);

/* One 128x128 tile of raw FP4 scores S = Qc . Kc^T (fp32, no softmax scale,
 * no global scales) through the same tcgen05 block-scaled MMA, scale-factor
 * staging and descriptors as fp4attn_forward.  q_* and k_* point at the
 * first of 128 rows (codes [128,64], scales [128,8]); s_out_dev fp32 [128,128]. */
int fp4attn_probe_qk_tile(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev,
                          const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                          float* s_out_dev, cudaStream_t stream);

/* One 128x128 tile of O = P . V (fp32) through the same TMEM-resident P
 * (bf16) and tcgen05 BF16 MMA path as fp4attn_forward.  p_bf16_dev [128,128]
 * (rows = queries, columns = keys), v_bf16_dev [128,128] (rows = keys),
 * o_out_dev fp32 [128,128]. */
int fp4attn_probe_pv_tile(const void* p_bf16_dev, const void* v_bf16_dev, float* o_out_dev,
                          cudaStream_t stream);

/* Testing: the block-scale quotient amax / 6 is computed without a divide
 * (one multiply by fl(1/6) and an FMA refinement).  This checks it against the
 * IEEE quotient for every non-negative finite fp32 value (synchronous).
 *   result_dev : device uint32[2] out: [0] the number of mismatches, [1] the
 *     smallest mismatching bit pattern (0xFFFFFFFF if none). */
int fp4attn_probe_div6(uint32_t* result_dev, cudaStream_t stream);

/* Tensor-core rate probe (a measurement of the roofline's denominators, not a
 * step of the path): one CTA per SM issues `reps` groups of back-to-back
 * tcgen05 MMAs into one TMEM accumulator, every operand resident.
 *   mode 0: block-scaled FP4 (kind::mxf4nvf4, scale_vec::4X, E2M1 operands,
 *           UE4M3 factors per 16 values) M=128 N=256 K=64, two per group:
 *           2*2*128*256*64 FLOPs per group per SM;
 *   mode 1: BF16 (kind::f16, fp32 accumulate) M=128 N=256 K=16, eight per
 *           group: 8*2*128*256*16 FLOPs per group per SM.
 * *cycles_dev (device int64) receives CTA 0's clock64() count from its first
 * issue to the completion of its last MMA, or -1 if that completion was not
 * seen within 4 s (then FP4ATTN_ERR_TIMEOUT is in *status_dev, a device int32
 * the caller zeroes).  The caller times the launch with events on `stream`.
 * 1 <= reps <= 10^6; asynchronous. */
int fp4attn_probe_mma_rate(int mode, int reps, long long* cycles_dev, int* status_dev, cudaStream_t stream);

/* Runs the bounded mbarrier wait of the attention kernel on a barrier that
 * nothing arrives at, with the given limit; the kernel must give up and write
 * FP4ATTN_ERR_TIMEOUT into *status_dev (device int32, set to 0 first). */
int fp4attn_probe_wait_timeout(int* status_dev, uint64_t limit_ns, cudaStream_t stream);

/* Runs fp4attn_quantize_qk on contiguous Q and K with the key-sum tiles
 * withheld, so the first K tile of every head waits for column sums that no
 * tile computes.  That wait must give up after limit_ns (at most 10 s), write
 * FP4ATTN_ERR_TIMEOUT into the workspace status word and let every CTA wind
 * down (each waits for its own copies in flight) and return.  Arguments as
 * fp4attn_quantize_qk without the global scales, flags and key mean; the
 * workspace is cleared first.  Q codes and scales are written as usual; the
 * K outputs are unspecified. */
int fp4attn_probe_withheld_key_sums(const void* q_bf16_dev, const void* k_bf16_dev, fp4attn_shape s,
                                    uint8_t* q_codes_dev, uint8_t* q_scales_dev,
                                    uint8_t* k_codes_dev, uint8_t* k_scales_dev,
                                    void* workspace_dev, size_t workspace_bytes, uint64_t limit_ns,
                                    cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4ATTN_H */
