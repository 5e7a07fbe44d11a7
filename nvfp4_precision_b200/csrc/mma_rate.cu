// Tensor-core rate probe: the throughput of back-to-back tcgen05 MMAs with
// every operand resident (shared memory and TMEM), for the two products the
// attention kernel issues: the block-scaled FP4 score product
// (kind::mxf4nvf4, scale_vec::4X, M=128 N=256 K=64) and the BF16 product
// (kind::f16, M=128 N=256 K=16).  A measurement of the denominators of the
// roofline, not a step of the path.
//
// One CTA per SM; one thread fills the operand tiles with finite bit patterns,
// allocates the whole TMEM, stages the FP4 scale factors, then issues `reps`
// groups (two FP4 MMAs over K=128, or eight BF16 MMAs over K=128) into one
// accumulator, commits, and waits (bounded) for the last to complete.
#include <cstddef>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

struct __align__(1024) RateSmem {
    uint8_t a16[2][16384];  // bf16 A: 128 rows x 64 channels per 128B-swizzled panel, two panels (K = 128)
    uint8_t b16[4][16384];  // bf16 B: 256 rows, two 128-row panels per 64 channels
    uint8_t a4[8192];       // E2M1 A: 128 rows x 64 bytes (K = 128), 64B swizzle
    uint8_t b4[16384];      // E2M1 B: 256 rows x 64 bytes
    uint8_t sf[2][512];     // UE4M3 scale-factor atoms
    uint64_t bar;
    uint32_t tmem;
};

__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int mode, int reps, long long* cycles, int* status) {
    extern __shared__ uint8_t raw[];
    RateSmem& s = *reinterpret_cast<RateSmem*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    // finite operands: every byte <= 0x3F (bf16 halves of magnitude < 2, E2M1 codes, UE4M3 scales <= 0x3F)
    for (int i = threadIdx.x; i < (int)(offsetof(RateSmem, bar) / 4); i += blockDim.x) {
        uint32_t x = (uint32_t)i * 2654435761u ^ (uint32_t)blockIdx.x;
        x ^= x >> 13;
        x *= 0x85EBCA6Bu;
        x ^= x >> 16;
        reinterpret_cast<uint32_t*>(&s)[i] = x & 0x3F3F3F3Fu;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&s.bar), 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(smem_u32(&s.tmem), 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t = s.tmem;
    const uint32_t SFA = 384, SFB = 448;  // scale factors above the 256-column accumulator
    if (threadIdx.x == 0) {
        const uint32_t N = 256;
        long long c0 = 0;
        if (mode == 0) {
            tmem_cp_32x128b_x4(t + SFA, smem_desc(smem_u32(s.sf[0]), 0, 128, LAYOUT_NONE));
            tmem_cp_32x128b_x4(t + SFA + 4, smem_desc(smem_u32(s.sf[1]), 0, 128, LAYOUT_NONE));
            for (int c = 0; c < 4; ++c)
                tmem_cp_32x128b_x4(t + SFB + 4 * c, smem_desc(smem_u32(s.sf[c & 1]), 0, 128, LAYOUT_NONE));
            // D fp32, A and B E2M1, both K-major, N >> 3, M >> 4
            const uint32_t idesc = (1u << 7) | (1u << 10) | ((N >> 3) << 17) | (8u << 24);
            c0 = clock64();
            for (int r = 0; r < reps; ++r)
                for (int kk = 0; kk < 2; ++kk)
                    mma_mxf4nvf4(t, smem_desc(smem_u32(s.a4) + 32u * kk, 16, 512, LAYOUT_SW64),
                                 smem_desc(smem_u32(s.b4) + 32u * kk, 16, 512, LAYOUT_SW64), idesc,
                                 t + SFA + 4u * kk, t + SFB + 8u * kk, 1u);
        } else {
            // D fp32, A and B bf16, both K-major
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | (8u << 24);
            c0 = clock64();
            for (int r = 0; r < reps; ++r)
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ss(t, smem_desc(smem_u32(s.a16[ks >> 2]) + 32u * (ks & 3), 16, 1024, LAYOUT_SW128),
                                smem_desc(smem_u32(s.b16[ks >> 2]) + 32u * (ks & 3), 16, 1024, LAYOUT_SW128), idesc,
                                1u);
        }
        tc_commit(smem_u32(&s.bar));
        int abort_flag = 0;
        const bool done = mbar_wait(smem_u32(&s.bar), 0, &abort_flag, status, 4000000000ull);
        if (blockIdx.x == 0) *cycles = done ? clock64() - c0 : -1;
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(t, 512);
    }
}

}  // namespace

cudaError_t launch_mma_rate(int mode, int reps, long long* cycles, int* status, cudaStream_t stream) {
    const size_t smem = sizeof(RateSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    mma_rate_kernel<<<sms, 128, smem, stream>>>(mode, reps, cycles, status);
    return cudaGetLastError();
}

}  // namespace fp4attn
