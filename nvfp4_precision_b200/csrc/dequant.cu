// Test-side kernels: NVFP4 -> fp32 dequantisation and element-wise fp32 ->
// E2M1 / E4M3 conversion with the same device conversions the quantiser uses.
#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

// One thread per 16-value block: value = fl(fl(g * scale) * e2m1).
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                               const float* g_ptr, int64_t nblocks, float* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nblocks) return;
    const float g = g_ptr ? *g_ptr : 1.0f;
    const float gs = __fmul_rn(g, ue4m3_value(scales[i]));
    const uint2 c = *reinterpret_cast<const uint2*>(codes + i * 8);
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const uint32_t w = (e < 8) ? c.x : c.y;
        v[e] = __fmul_rn(gs, e2m1_value((w >> (4 * (e & 7))) & 0xF));
    }
    float4* dst = reinterpret_cast<float4*>(out + i * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// The same values rounded to bf16 (exact for a unit global scale: a 4-bit
// times a 2-bit significand): the dequantised Q and K of the training backward.
__global__ void dequant_bf16_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                    const float* g_ptr, int64_t nblocks, __nv_bfloat16* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nblocks) return;
    const float g = g_ptr ? *g_ptr : 1.0f;
    const float gs = __fmul_rn(g, ue4m3_value(scales[i]));
    const uint2 c = *reinterpret_cast<const uint2*>(codes + i * 8);
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint32_t word = (e < 4) ? c.x : c.y;
        const uint32_t lo = (word >> (8 * (e & 3))) & 0xF, hi = (word >> (8 * (e & 3) + 4)) & 0xF;
        w[e] = pack_bf16x2(__fmul_rn(gs, e2m1_value(lo)), __fmul_rn(gs, e2m1_value(hi)));
    }
    uint4* dst = reinterpret_cast<uint4*>(out + i * 16);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

__global__ void encode_kernel(const float* __restrict__ x, int64_t n, uint8_t* e2m1, uint8_t* e4m3) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = x[i];
        if (e2m1) e2m1[i] = (uint8_t)cvt_e2m1(v);
        if (e4m3) e4m3[i] = (uint8_t)cvt_e4m3(v);
    }
}

// Every non-negative finite fp32 bit pattern a: div6_rn(a) against the IEEE
// quotient, and the UE4M3 byte of the branch-free div6_refined(a) (the block
// scale at g = 1, sign bit cleared) against the byte of the IEEE quotient.
// res[0] counts the inputs where either differs, res[1] holds the smallest.
__global__ void div6_check_kernel(unsigned* res) {
    const uint32_t stride = gridDim.x * blockDim.x;
    unsigned count = 0;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < 0x7F800000u; i += stride) {
        const float a = __uint_as_float(i);
        const float q = __fdiv_rn(a, 6.0f);
        if (__float_as_uint(div6_rn(a)) != __float_as_uint(q) ||
            (cvt_e4m3(div6_refined(a)) & 0x7Fu) != cvt_e4m3(q)) {
            ++count;
            atomicMin(res + 1, i);
        }
    }
    if (count) atomicAdd(res, count);
}

}  // namespace

cudaError_t launch_div6_check(unsigned* res, cudaStream_t stream) {
    div6_check_kernel<<<148 * 8, 256, 0, stream>>>(res);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t nblocks,
                           float* out, cudaStream_t stream) {
    if (nblocks == 0) return cudaSuccess;
    const int threads = 256;
    dequant_kernel<<<(unsigned)((nblocks + threads - 1) / threads), threads, 0, stream>>>(
        codes, scales, g, nblocks, out);
    return cudaGetLastError();
}

cudaError_t launch_dequant_bf16(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t nblocks,
                                __nv_bfloat16* out, cudaStream_t stream) {
    if (nblocks == 0) return cudaSuccess;
    const int threads = 256;
    dequant_bf16_kernel<<<(unsigned)((nblocks + threads - 1) / threads), threads, 0, stream>>>(codes, scales, g,
                                                                                               nblocks, out);
    return cudaGetLastError();
}

cudaError_t launch_encode_f32(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                              cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t want = (n + threads - 1) / threads;
    const unsigned blocks = (unsigned)(want < 148 * 64 ? want : 148 * 64);
    encode_kernel<<<blocks, threads, 0, stream>>>(x, n, e2m1, e4m3);
    return cudaGetLastError();
}

}  // namespace fp4attn
