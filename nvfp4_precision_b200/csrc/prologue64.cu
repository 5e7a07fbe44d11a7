// Quantisation prologue for heads of 64 channels: smooth K + 64-point
// Hadamard + NVFP4 pack of Q and K.
//
// FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention": the page's
// toy heads have 64 channels (four 16-value blocks) and 32 keys, quantised
// like the FP4 attention kernel after subtracting each head's mean key and
// rotating Q and K by the same orthonormal Hadamard matrix.  Same method and
// the same pinned steps as the 128-channel prologue: the exact int64 key sum
// of round_half_even(k * 2^24), m = (float)((double)S / (N * 2^24)), the
// Sylvester-order butterflies with ascending strides 1..32 in fp32, then
// x fp32(1/sqrt(64)) = 1/8, and per 16-value block a UE4M3 scale amax/6/g
// and E2M1 codes of y * (1/(g * scale)).  A row has 32 code bytes (element
// 2i in the low nibble of byte i) and 4 scale bytes.
//
// Two plain launches, for the toy study and other narrow heads rather than
// for speed: the key sums (one CTA per 256 rows of a head, int64 atomics of
// the CTA's column sums), then the transform (two threads per row, the means
// computed by each CTA from the complete sums, which stream order makes
// available).
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr int D64 = 64;
constexpr float kTwo24f = 16777216.0f;
constexpr float kKeyLimit = 1048576.0f;  // |k| < 2^20 keeps the int64 sum exact for N <= 2^18

__device__ __forceinline__ void set_status64(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ const __nv_bfloat16* row_ptr(const __nv_bfloat16* base, Strides st, int H, int bh,
                                                        int n) {
    const int b = bh / H, h = bh - b * H;
    return base + (int64_t)b * st.b + (int64_t)h * st.h + (int64_t)n * st.n;
}

// Column sums of K: thread t sums channels 4(t%16)..+3 of rows t/16, t/16+16, ...
// of the CTA's 256 rows; the 16 partial sums of each channel meet in shared
// memory and one thread per channel adds them to the workspace.
__global__ void __launch_bounds__(256) ksum64_kernel(const __nv_bfloat16* k, Strides ks, int H, int N,
                                                     long long* ksum, int* status) {
    __shared__ long long part[16][D64];
    const int bh = blockIdx.y;
    const int t = threadIdx.x;
    const int cg = t & 15, r0 = t >> 4;
    long long acc[4] = {0, 0, 0, 0};
    float kmax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        const int n = blockIdx.x * 256 + r0 + 16 * i;
        if (n >= N) break;
        const uint2 w = *reinterpret_cast<const uint2*>(row_ptr(k, ks, H, bh, n) + 4 * cg);
        const float v[4] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            acc[c] += __float2ll_rn(__fmul_rn(v[c], kTwo24f));
            kmax = fmaxf(kmax, fabsf(v[c]));
        }
    }
    if (!(kmax < kKeyLimit)) set_status64(status, FP4ATTN_ERR_RANGE);
#pragma unroll
    for (int c = 0; c < 4; ++c) part[r0][4 * cg + c] = acc[c];
    __syncthreads();
    if (t < D64 && FP4ATTN_IN_BOUNDS(bh < (int)gridDim.y, status)) {
        long long tot = 0;
#pragma unroll
        for (int r = 0; r < 16; ++r) tot += part[r][t];
        atomicAdd(reinterpret_cast<unsigned long long*>(ksum + (size_t)bh * D + t), static_cast<unsigned long long>(tot));
    }
}

// Scale byte and 1/(g*scale) of one block with amax a (the 128-channel
// prologue's block_scale, without its table).
__device__ __forceinline__ void block_scale64(float a, float g, uint32_t& s, float& inv) {
    float t = div6_rn(a);
    if (g != 1.0f) t = __fdiv_rn(t, g);
    s = cvt_e4m3(t);
    const float sd = ue4m3_value(s);
    inv = (sd != 0.0f) ? __frcp_rn(__fmul_rn(g, sd)) : 0.0f;
}

__device__ __forceinline__ float amax16x(const float2* p, bool hi) {
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(hi ? p[k].y : p[k].x));
    return m;
}

// Two threads per row: lane h of a pair holds (x_i, x_{i+32}) for
// i in [16h, 16h+16).  Butterfly strides 1..8 inside the lane (packed fp32x2),
// stride 16 across the lane pair (lane 0 keeps the sum, lane 1 the difference,
// each fl(other + sign * own)), stride 32 inside each pair, then x 1/8.  Lane h
// then holds blocks h (.x) and h + 2 (.y).  blockIdx.z: 0 = Q, 1 = K.
__global__ void __launch_bounds__(128) transform64_kernel(Prologue64Args a) {
    __shared__ float2 neg_mean2[32];  // (-m_i, -m_{i+32})
    const int bh = blockIdx.y;
    const int which = blockIdx.z;
    const int N = a.N;
    const bool smooth = !(a.flags & FP4ATTN_NO_SMOOTH_K);
    const bool hadamard = !(a.flags & FP4ATTN_NO_HADAMARD);
    const int t = threadIdx.x;
    float g = 1.0f;
    const float* gp = which ? a.gk : a.gq;
    if (gp) g = *gp;
    if (t == 0 && blockIdx.x == 0 && bh == 0 && which == 0) {
        float gq = a.gq ? *a.gq : 1.0f, gk = a.gk ? *a.gk : 1.0f;
        if (!(gq > 0.0f && gq < INFINITY && gk > 0.0f && gk < INFINITY)) set_status64(a.status, FP4ATTN_ERR_RANGE);
    }
    if (which == 1 && t < D64) {
        float m = 0.0f;
        if (smooth) {
            const long long S = __ldcg(a.ksum + (size_t)bh * D + t);
            m = __double2float_rn(__ddiv_rn(__ll2double_rn(S), (double)N * 16777216.0));
        }
        if (t < 32) neg_mean2[t].x = -m; else neg_mean2[t - 32].y = -m;
        if (a.k_mean && blockIdx.x == 0) a.k_mean[(size_t)bh * D64 + t] = m;
    }
    __syncthreads();
    const int h = t & 1;
    const int n = blockIdx.x * 64 + (t >> 1);
    const bool valid = n < N;
    const __nv_bfloat16* src = row_ptr(which ? a.k : a.q, which ? a.ks : a.qs, a.H, bh, valid ? n : 0);
    // channels [16h, 16h+16) and [32+16h, 32+16h+16): two 16-byte loads each
    uint4 lo[2], hi[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        lo[j] = *reinterpret_cast<const uint4*>(src + 16 * h + 8 * j);
        hi[j] = *reinterpret_cast<const uint4*>(src + 32 + 16 * h + 8 * j);
    }
    float2 P[16];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t wl[4] = {lo[j].x, lo[j].y, lo[j].z, lo[j].w};
        const uint32_t wh[4] = {hi[j].x, hi[j].y, hi[j].z, hi[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            P[8 * j + 2 * e] = make_float2(bf16lo(wl[e]), bf16lo(wh[e]));
            P[8 * j + 2 * e + 1] = make_float2(bf16hi(wl[e]), bf16hi(wh[e]));
        }
    }
    if (which == 1 && smooth) {
#pragma unroll
        for (int k = 0; k < 16; ++k) P[k] = __fadd2_rn(P[k], neg_mean2[16 * h + k]);
    }
    bool finite = true;
    if (hadamard) {
#pragma unroll
        for (int st = 1; st < 16; st <<= 1) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                if ((k & st) == 0) {
                    const float2 x = P[k], y = P[k + st];
                    P[k] = __fadd2_rn(x, y);
                    P[k + st] = __ffma2_rn(y, make_float2(-1.0f, -1.0f), x);
                }
            }
        }
        const float sg = h ? -1.0f : 1.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float ox = __shfl_xor_sync(0xffffffffu, P[k].x, 1);
            const float oy = __shfl_xor_sync(0xffffffffu, P[k].y, 1);
            P[k] = __ffma2_rn(P[k], make_float2(sg, sg), make_float2(ox, oy));
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) P[k] = make_float2(__fadd_rn(P[k].x, P[k].y), __fsub_rn(P[k].x, P[k].y));
        const float c = 0.125f;  // fp32(1/sqrt(64)), exact
#pragma unroll
        for (int k = 0; k < 16; ++k) P[k] = __fmul2_rn(P[k], make_float2(c, c));
        finite = (h != 0) || (fabsf(P[0].x) < INFINITY);
    } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) finite &= (fabsf(P[k].x) < INFINITY) && (fabsf(P[k].y) < INFINITY);
    }
    if (!finite && valid) set_status64(a.status, FP4ATTN_ERR_RANGE);
    uint32_t sx, sy;
    float ix, iy;
    block_scale64(amax16x(P, false), g, sx, ix);
    block_scale64(amax16x(P, true), g, sy, iy);
    uint32_t wx[2], wy[2];
#pragma unroll
    for (int h8 = 0; h8 < 2; ++h8) {
        float2 R[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) R[k] = __fmul2_rn(P[8 * h8 + k], make_float2(ix, iy));
        wx[h8] = cvt_e2m1x8(R[0].x, R[1].x, R[2].x, R[3].x, R[4].x, R[5].x, R[6].x, R[7].x);
        wy[h8] = cvt_e2m1x8(R[0].y, R[1].y, R[2].y, R[3].y, R[4].y, R[5].y, R[6].y, R[7].y);
    }
    // scale bytes: lane 0 holds blocks 0 and 2, lane 1 blocks 1 and 3
    const uint32_t mine = sx | (sy << 8);
    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
    if (valid && FP4ATTN_IN_BOUNDS((size_t)bh * N + n < (size_t)gridDim.y * N, a.status)) {
        const size_t row = (size_t)bh * N + n;
        uint8_t* crow = (which ? a.k_codes : a.q_codes) + row * 32;
        *reinterpret_cast<uint2*>(crow + 8 * h) = make_uint2(wx[0], wx[1]);
        *reinterpret_cast<uint2*>(crow + 16 + 8 * h) = make_uint2(wy[0], wy[1]);
        if (h == 0) {
            uint32_t w;
            asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(w) : "r"(mine), "r"(other));
            *reinterpret_cast<uint32_t*>((which ? a.k_scales : a.q_scales) + row * 4) = w;
        }
    }
}

}  // namespace

cudaError_t launch_quantize_qk64(const Prologue64Args& a, cudaStream_t stream) {
    if (a.BH == 0 || a.N == 0) return cudaSuccess;
    if (!(a.flags & FP4ATTN_NO_SMOOTH_K)) {
        ksum64_kernel<<<dim3((a.N + 255) / 256, a.BH), 256, 0, stream>>>(a.k, a.ks, a.H, a.N, a.ksum, a.status);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    transform64_kernel<<<dim3((a.N + 63) / 64, a.BH, 2), 128, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace fp4attn
