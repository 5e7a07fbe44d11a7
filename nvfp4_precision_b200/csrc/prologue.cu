// Quantisation prologue: smooth K + Hadamard + NVFP4 pack of Q and K.
//
// Method: FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention" --
// subtract each head's mean key, rotate Q and K by the same orthonormal
// Hadamard matrix, quantise both to NVFP4 (E2M1 values, one E4M3 scale per 16
// channels, fp32 per-tensor scale).  The fused transform there costs under
// 1 ms per attention call on GB200.
//
// Two kernels, stream-ordered:
//   ksum_kernel      exact int64 fixed-point column sums of K per head
//                    (sum of round_half_even(k * 2^24)); order-independent,
//                    so the atomics give the same bits as any serial order.
//   quantize_kernel  one thread per 128-channel row: bf16 -> fp32, K minus the
//                    head mean, 7 butterfly stages of ascending stride in
//                    registers (no shuffles), x fp32(1/sqrt(128)), per-16 amax,
//                    UE4M3 scale amax/6/g, E2M1 codes of y * (1/(g*scale)).
// Every fp32 step is an explicit round-to-nearest intrinsic so nothing is
// contracted into an FMA; the results are bit-identical to the plain CPU
// definition of the same steps.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr float kTwo24 = 16777216.0f;
constexpr float kKeyLimit = 1048576.0f;  // |k| < 2^20 keeps the int64 sum exact for N <= 2^18
constexpr int KSUM_THREADS = 256;
constexpr int KSUM_ROWS_PER_BLOCK = 2048;

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ----------------------------------------------------------- key sums -----

// grid (ceil(N / KSUM_ROWS_PER_BLOCK), BH); 16 threads per row (8 channels
// each, one 16-byte load), 16 rows in flight per block iteration.
__global__ void __launch_bounds__(KSUM_THREADS) ksum_kernel(const __nv_bfloat16* __restrict__ k,
                                                            int N, long long* __restrict__ ksum,
                                                            int* status) {
    const int bh = blockIdx.y;
    const int n0 = blockIdx.x * KSUM_ROWS_PER_BLOCK;
    const int n1 = min(N, n0 + KSUM_ROWS_PER_BLOCK);
    const int cg = threadIdx.x & 15;   // channel group: channels 8cg .. 8cg+7
    const int rg = threadIdx.x >> 4;   // row group 0..15
    long long acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0;
    bool bad = false;
    const uint4* base = reinterpret_cast<const uint4*>(k + ((size_t)bh * N) * D) + cg;
    for (int n = n0 + rg; n < n1; n += 16) {
        const uint4 raw = __ldg(base + (size_t)n * (D / 8));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float v = (e & 1) ? bf16hi(w[e >> 1]) : bf16lo(w[e >> 1]);
            if (fabsf(v) < kKeyLimit) {
                acc[e] += __float2ll_rn(__fmul_rn(v, kTwo24));  // exact product, ties-to-even
            } else {
                bad = true;  // also catches NaN
            }
        }
    }
    __shared__ long long part[16][D];
#pragma unroll
    for (int e = 0; e < 8; ++e) part[rg][cg * 8 + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < D) {
        long long t = 0;
#pragma unroll
        for (int r = 0; r < 16; ++r) t += part[r][threadIdx.x];
        atomicAdd(reinterpret_cast<unsigned long long*>(ksum + (size_t)bh * D + threadIdx.x),
                  static_cast<unsigned long long>(t));
    }
    if (bad) set_status(status, FP4ATTN_ERR_RANGE);
}

// ----------------------------------------------------------- transform -----

// Unnormalised Sylvester Walsh-Hadamard transform, butterflies of stride
// 1, 2, ..., 64 in that order.
__device__ __forceinline__ void fwht128(float (&x)[D]) {
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
        for (int i = 0; i < D; ++i) {
            if ((i & h) == 0) {
                const float a = x[i], b = x[i + h];
                x[i] = __fadd_rn(a, b);
                x[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

// NVFP4 pack of one 16-value block: two code words (element 0 in the low
// nibble of word0) and the UE4M3 scale byte.
__device__ __forceinline__ void pack_block(const float* y, float g, bool g_is_one, uint32_t& w0,
                                           uint32_t& w1, uint32_t& scale) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(y[i]));
    float t = __fdiv_rn(a, 6.0f);
    if (!g_is_one) t = __fdiv_rn(t, g);
    const uint32_t s = cvt_e4m3(t);  // t >= 0: the E4M3 byte is the UE4M3 byte
    const float sd = ue4m3_value(s);
    float inv = 0.0f;
    if (sd != 0.0f) inv = __frcp_rn(g_is_one ? sd : __fmul_rn(g, sd));
    float r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __fmul_rn(y[i], inv);
    w0 = cvt_e2m1x8(r[0], r[1], r[2], r[3], r[4], r[5], r[6], r[7]);
    w1 = cvt_e2m1x8(r[8], r[9], r[10], r[11], r[12], r[13], r[14], r[15]);
    scale = s;
}

struct QuantKernelArgs {
    const __nv_bfloat16* src[2];  // Q, K
    uint8_t* codes[2];
    uint8_t* scales[2];
    const float* g[2];
    const long long* ksum;
    float* k_mean;
    int N;
    uint32_t flags;
    int* status;
};

constexpr int QUANT_ROWS = 128;

// grid (ceil(N / 128), BH, 2): z = 0 quantises Q rows, z = 1 K rows.  One
// thread per row.
__global__ void __launch_bounds__(QUANT_ROWS) quantize_kernel(const QuantKernelArgs a) {
    const int which = blockIdx.z;
    const int bh = blockIdx.y;
    const int N = a.N;
    const int n = blockIdx.x * QUANT_ROWS + threadIdx.x;
    const bool smooth = (which == 1) && !(a.flags & FP4ATTN_NO_SMOOTH_K);
    const bool hadamard = !(a.flags & FP4ATTN_NO_HADAMARD);

    __shared__ float mean_s[D];
    if (smooth) {
        const int c = threadIdx.x;  // blockDim.x == D
        const double num = __ll2double_rn(a.ksum[(size_t)bh * D + c]);
        const double den = (double)N * 16777216.0;
        const float m = __double2float_rn(__ddiv_rn(num, den));
        mean_s[c] = m;
        if (a.k_mean && blockIdx.x == 0) a.k_mean[(size_t)bh * D + c] = m;
    } else if (which == 1 && a.k_mean && blockIdx.x == 0) {
        a.k_mean[(size_t)bh * D + threadIdx.x] = 0.0f;
    }
    __syncthreads();

    float g = 1.0f;
    if (a.g[which]) {
        g = *a.g[which];
        if (!(g > 0.0f && g < INFINITY)) set_status(a.status, FP4ATTN_ERR_RANGE);
    }
    const bool g_is_one = (g == 1.0f);
    if (n >= N) return;

    const size_t row = (size_t)bh * N + n;
    const uint4* src = reinterpret_cast<const uint4*>(a.src[which] + row * D);
    float x[D];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        const uint4 raw = __ldg(src + i);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) x[8 * i + e] = (e & 1) ? bf16hi(w[e >> 1]) : bf16lo(w[e >> 1]);
    }
    bool finite = true;
#pragma unroll
    for (int i = 0; i < D; ++i) finite &= (fabsf(x[i]) < INFINITY);
    if (!finite) set_status(a.status, FP4ATTN_ERR_RANGE);

    if (smooth) {
#pragma unroll
        for (int i = 0; i < D; ++i) x[i] = __fsub_rn(x[i], mean_s[i]);
    }
    if (hadamard) {
        fwht128(x);
        const float c = __uint_as_float(0x3DB504F3u);  // fp32(1/sqrt(128))
#pragma unroll
        for (int i = 0; i < D; ++i) x[i] = __fmul_rn(x[i], c);
    }

    uint32_t cw[16];
    uint32_t sb[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) pack_block(x + 16 * b, g, g_is_one, cw[2 * b], cw[2 * b + 1], sb[b]);

    uint4* dst = reinterpret_cast<uint4*>(a.codes[which] + row * 64);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(cw[4 * i], cw[4 * i + 1], cw[4 * i + 2], cw[4 * i + 3]);
    uint2 s2;
    s2.x = sb[0] | (sb[1] << 8) | (sb[2] << 16) | (sb[3] << 24);
    s2.y = sb[4] | (sb[5] << 8) | (sb[6] << 16) | (sb[7] << 24);
    *reinterpret_cast<uint2*>(a.scales[which] + row * 8) = s2;
}

}  // namespace

cudaError_t launch_quantize_qk(const QuantArgs& a, cudaStream_t stream) {
    if (a.BH == 0 || a.N == 0) return cudaSuccess;
    if (!(a.flags & FP4ATTN_NO_SMOOTH_K)) {
        dim3 grid((a.N + KSUM_ROWS_PER_BLOCK - 1) / KSUM_ROWS_PER_BLOCK, a.BH);
        ksum_kernel<<<grid, KSUM_THREADS, 0, stream>>>(a.k, a.N, a.ksum, a.status);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    QuantKernelArgs k{};
    k.src[0] = a.q;
    k.src[1] = a.k;
    k.codes[0] = a.q_codes;
    k.codes[1] = a.k_codes;
    k.scales[0] = a.q_scales;
    k.scales[1] = a.k_scales;
    k.g[0] = a.gq;
    k.g[1] = a.gk;
    k.ksum = a.ksum;
    k.k_mean = a.k_mean;
    k.N = a.N;
    k.flags = a.flags;
    k.status = a.status;
    dim3 grid((a.N + QUANT_ROWS - 1) / QUANT_ROWS, a.BH, 2);
    quantize_kernel<<<grid, QUANT_ROWS, 0, stream>>>(k);
    return cudaGetLastError();
}

}  // namespace fp4attn
