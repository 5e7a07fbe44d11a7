// NVFP4 operands of the block-scaled tensor-core MMA (tcgen05.mma
// kind::mxf4nvf4), shared by the attention forward and the dQ kernel of the
// training backward: E2M1 code tiles in shared memory and UE4M3 scale factors
// staged through shared-memory atoms into TMEM.
#pragma once
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

// Instruction descriptor of kind::mxf4nvf4: A = B = E2M1 (1 at bits 7 and
// 10), UE4M3 scales, both K-major, M = m rows, N = n columns.
__host__ __device__ constexpr uint32_t idesc_mxf4(int m, int n) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Scales of up to 128 rows (row-major, one uint64 = 8 UE4M3 bytes per row) ->
// two 512-byte atoms (channels 0-63 and 64-127).  Atom line r (16 bytes)
// holds, for rows r, r+32, r+64, r+96, the four scales of that 64-channel
// chunk; tcgen05.cp 32x128b.warpx4 then puts line r in TMEM lane r of every
// sub-partition, so rows 32c.. sit in column c of the chunk's four columns.
// One full warp, lane = line; rows at or beyond n_rows read as zero.  Plain
// 8-byte loads: a row's scales start at any multiple of 8 bytes, which a bulk
// tensor copy could not address.
__device__ __forceinline__ void fetch_scales(const uint64_t* rows, int n_rows, int lane, uint64_t (&w)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int r = lane + 32 * c;
        w[c] = (r < n_rows) ? __ldg(reinterpret_cast<const unsigned long long*>(rows) + r) : 0ull;
    }
}

// The same for rows of srb = 8 or 4 scale bytes (128 or 64 channels): a row of
// 4 bytes reads as its 8-byte form with the upper four scales zero.
__device__ __forceinline__ void fetch_scales_rows(const uint8_t* rows, int srb, int n_rows, int lane,
                                                  uint64_t (&w)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int r = lane + 32 * c;
        if (r >= n_rows) {
            w[c] = 0ull;
        } else if (srb == 8) {
            w[c] = __ldg(reinterpret_cast<const unsigned long long*>(rows) + r);
        } else {
            w[c] = (uint64_t)__ldg(reinterpret_cast<const unsigned int*>(rows) + r);
        }
    }
}

__device__ __forceinline__ void store_scale_atoms(const uint64_t (&w)[4], uint8_t* atom0, uint8_t* atom1, int lane) {
    *reinterpret_cast<uint4*>(atom0 + 16 * lane) =
        make_uint4((uint32_t)w[0], (uint32_t)w[1], (uint32_t)w[2], (uint32_t)w[3]);
    *reinterpret_cast<uint4*>(atom1 + 16 * lane) =
        make_uint4((uint32_t)(w[0] >> 32), (uint32_t)(w[1] >> 32), (uint32_t)(w[2] >> 32), (uint32_t)(w[3] >> 32));
}

__device__ __forceinline__ void load_scale_atoms(const uint64_t* rows, int n_rows, uint8_t* atom0,
                                                 uint8_t* atom1, int lane) {
    uint64_t w[4];
    fetch_scales(rows, n_rows, lane, w);
    store_scale_atoms(w, atom0, atom1, lane);
}

__device__ __forceinline__ uint64_t atom_desc(const void* atom) {
    // K-major, no swizzle: 8-row core matrices of 16-byte rows, 128 B apart.
    return smem_desc(smem_u32(atom), 0, 128, LAYOUT_NONE);
}

__device__ __forceinline__ uint64_t codes_desc(const uint8_t* tile, int kchunk) {
    // K-major 64B swizzle: rows of 64 bytes (128 E2M1), 8-row groups 512 B
    // apart; the second 64-value K chunk starts 32 bytes into each row.
    return smem_desc(smem_u32(tile) + 32u * kchunk, 16, 512, LAYOUT_SW64);
}

// Codes [BH][N][row_bytes] (64 bytes for 128 channels, 32 for 64): 64B-swizzled
// boxes of 64 bytes x box_rows rows, x always 0; bytes of a box past a 32-byte
// row read as zero codes.
inline bool make_code_map(CUtensorMap* m, const uint8_t* base, int BH, int N, uint32_t box_rows,
                          uint32_t row_bytes = 64) {
    const uint64_t dims[3] = {row_bytes, (uint64_t)N, (uint64_t)BH};
    const uint64_t strides[2] = {row_bytes, (uint64_t)N * row_bytes};
    const uint32_t box[3] = {64, box_rows, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace fp4attn
