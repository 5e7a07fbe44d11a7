// Non-causal FP4 attention: O = softmax(scale * Q K^T) V with NVFP4 Q and K
// (block-scaled E2M1, one UE4M3 scale per 16 channels) and BF16 P and V.
//
// Method: FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention":
// queries and keys are quantised for an NVFP4 attention kernel; P and V stay
// in BF16.  This kernel is written for sm_100a:
//   * one CTA per (head, 128-query tile); 4 * COL_GROUPS softmax warps plus
//     two more:
//       softmax    softmax, O correction and epilogue; query row r is TMEM
//                  lane r and is shared by the COL_GROUPS warps w with
//                  w % 4 == r / 32, each owning 128 / COL_GROUPS key columns
//                  of every tile; they exchange partial row maxima through
//                  shared memory every tile;
//       producer   scale-factor atoms (plain loads) and TMA copies of Q
//                  once, then K codes and V tiles of 128 keys into a
//                  STAGES-deep shared-memory ring;
//       MMA        TMEM owner and MMA issuer: stages the scale factors into
//                  TMEM (tcgen05.cp) and issues S = Q K^T with
//                  tcgen05.mma kind::mxf4nvf4 (block16 scales) and
//                  O += P V with tcgen05.mma kind::f16 (P read from TMEM);
//   * TMEM (512 columns): S double buffer [0,128) [128,256) fp32, O [256,384),
//     Q scale factors [384,392), K scale factors 2 x 8 columns from 392; P is
//     written as bf16 pairs over the first 64 columns of its S buffer;
//   * online softmax in the log2 domain with a lazy rescale: the running max
//     only moves when a tile's max exceeds it by more than 8 (so p <= 256),
//     and O is rescaled in TMEM only then; exponentials are split between
//     the MUFU unit and a polynomial on the FMA pipe, with packed fp32x2
//     arithmetic for the scale, the polynomial and the row sums.
// Every wait is bounded; a wait that runs out raises FP4ATTN_ERR_TIMEOUT in
// the status word and the CTA winds down (waiting for its own copies and MMAs)
// instead of hanging.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int STAGES = 4;
// Softmax warps come in COL_GROUPS groups of four (one warp per TMEM
// sub-partition); each warp owns CW of the 128 score columns of its 32 rows.
#ifndef FP4ATTN_COL_GROUPS
#define FP4ATTN_COL_GROUPS 2
#endif
// Of every 8 pairs of exponentials, this many go to the FMA-pipe polynomial
// and the rest to MUFU ex2 (MUFU issues 16 per clock per SM).
#ifndef FP4ATTN_POLY_PAIRS
#define FP4ATTN_POLY_PAIRS 3
#endif
constexpr int COL_GROUPS = FP4ATTN_COL_GROUPS;
static_assert(COL_GROUPS == 2 || COL_GROUPS == 4, "2 or 4 column groups");
constexpr int CW = 128 / COL_GROUPS;  // score columns per softmax warp
constexpr int CW32 = CW / 32;         // 32-column TMEM loads per tile
constexpr int SOFTMAX_WARPS = 4 * COL_GROUPS;
constexpr int FWD_THREADS = 32 * (SOFTMAX_WARPS + 2);
constexpr int WARP_PRODUCER = SOFTMAX_WARPS;
constexpr int WARP_MMA = SOFTMAX_WARPS + 1;
constexpr int POLY_PAIRS_PER_8 = FP4ATTN_POLY_PAIRS;

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0;
constexpr uint32_t TM_O = 256;
constexpr uint32_t TM_SFQ = 384;
constexpr uint32_t TM_SFK = 392;

constexpr uint32_t CODE_TILE_BYTES = 128 * 64;    // 128 rows x 128 E2M1 values
constexpr uint32_t V_PANEL_BYTES = 128 * 64 * 2;  // 128 keys x 64 channels bf16
constexpr uint32_t V_TILE_BYTES = 2 * V_PANEL_BYTES;

// Instruction descriptors.
//  S: kind::mxf4nvf4, A = B = E2M1 (1), UE4M3 scales, K-major, N = 128, M = 128.
constexpr uint32_t IDESC_QK = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);
//  O: kind::f16, fp32 accumulate (1 << 4), A = B = BF16, A K-major (TMEM),
//     B = V MN-major (1 << 16), N = 128 channels, M = 128.
constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct __align__(1024) FwdSmem {
    uint8_t v[STAGES][V_TILE_BYTES];      // two 64-channel panels, 128B swizzle
    uint8_t kc[STAGES][CODE_TILE_BYTES];  // 64B swizzle
    uint8_t qc[CODE_TILE_BYTES];          // 64B swizzle
    uint8_t ks_atom[STAGES][2][512];      // scale-factor atoms for tcgen05.cp
    uint8_t qs_atom[2][512];
    uint64_t bar_q_full;
    uint64_t bar_kv_full[STAGES];
    uint64_t bar_kv_empty[STAGES];
    uint64_t bar_s_full[2];
    uint64_t bar_p_ready[2];      // P of tiles with this parity is in TMEM
    uint64_t bar_o_done;          // O holds the P.V of every tile up to the last commit
    uint64_t bar_o_final;         // the last tile's P.V is done
    uint64_t bar_final;
    uint64_t bar_group[4][2];              // per sub-partition, per tile parity: all partial maxima are in
    float red_max[2][COL_GROUPS][128];     // [tile parity][column group][row] partial row maxima
    float red_sum[COL_GROUPS][128];        // [column group][row] partial row sums, at the end
    uint32_t tmem_base;
    int abort_flag;
};

struct FwdParams {
    const uint64_t* q_scales;  // one uint64 (8 UE4M3 bytes) per row
    const uint64_t* k_scales;
    int N;
    int n_kt;
    float scale_log2;  // softmax_scale * log2(e)
    const float* gq;
    const float* gk;
    __nv_bfloat16* o;
    float* lse;
    int* status;
    uint64_t limit_ns;
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s for the wind-down waits

template <typename T>
__device__ __forceinline__ T* align1024(uint8_t* p) {
    return reinterpret_cast<T*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Warp-uniform bounded wait.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, uint64_t limit) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status, limit);
    return __all_sync(0xffffffffu, ok);
}

// Wait used while winding down: ignores the abort flag, short limit.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
    int dummy_abort = 0;
    return mbar_wait(bar, parity, &dummy_abort, nullptr, kDrainLimitNs);
}

// Scales of 128 rows (row-major, one uint64 = 8 UE4M3 bytes per row) -> two
// 512-byte atoms (channels 0-63 and 64-127).  Atom line r (16 bytes) holds,
// for rows r, r+32, r+64, r+96, the four scales of that 64-channel chunk;
// tcgen05.cp 32x128b.warpx4 then puts line r in TMEM lane r of every
// sub-partition.  One full warp, lane = line; rows at or beyond n_rows read
// as zero.  Plain 8-byte loads: a row's scales start at any multiple of 8
// bytes, which a bulk tensor copy could not address.
__device__ __forceinline__ void fetch_scales(const uint64_t* rows, int n_rows, int lane, uint64_t (&w)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int r = lane + 32 * c;
        w[c] = (r < n_rows) ? __ldg(reinterpret_cast<const unsigned long long*>(rows) + r) : 0ull;
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

__device__ __forceinline__ uint64_t v_desc(const uint8_t* tile, int kstep) {
    // MN-major 128B swizzle: 64-channel panels 16 KB apart (leading byte
    // offset), 8-key groups 1 KB apart (stride byte offset); one MMA covers
    // 16 keys = 2 KB of each panel.
    return smem_desc(smem_u32(tile) + 2048u * kstep, V_PANEL_BYTES, 1024, LAYOUT_SW128);
}

// Issue S = Q K^T for one key tile (two K=64 block-scaled MMAs).
__device__ __forceinline__ void issue_qk(uint32_t tmem, uint32_t s_col, const uint8_t* qc,
                                         const uint8_t* kc, uint32_t sfk_col) {
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        mma_mxf4nvf4(tmem + s_col, codes_desc(qc, kk), codes_desc(kc, kk), IDESC_QK,
                     tmem + TM_SFQ + 4u * kk, tmem + sfk_col + 4u * kk, kk > 0 ? 1u : 0u);
    }
}

// Issue O (+)= P V for one key tile (eight K=16 BF16 MMAs, P from TMEM).
__device__ __forceinline__ void issue_pv(uint32_t tmem, uint32_t p_col, const uint8_t* v,
                                         bool accumulate_first) {
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        mma_bf16_ts(tmem + TM_O, tmem + p_col + 8u * ks, v_desc(v, ks), IDESC_PV,
                    (accumulate_first || ks > 0) ? 1u : 0u);
    }
}

__global__ void __launch_bounds__(FWD_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_qc, const __grid_constant__ CUtensorMap tm_kc,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem& sm = *align1024<FwdSmem>(smem_raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int q0 = blockIdx.x * BM;
    const int T = p.n_kt;
    const int N = p.N;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.bar_q_full), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm.bar_kv_full[s]), 1);
            mbar_init(smem_u32(&sm.bar_kv_empty[s]), 1);
        }
        mbar_init(smem_u32(&sm.bar_s_full[0]), 1);
        mbar_init(smem_u32(&sm.bar_s_full[1]), 1);
        mbar_init(smem_u32(&sm.bar_p_ready[0]), SOFTMAX_WARPS * 32);
        mbar_init(smem_u32(&sm.bar_p_ready[1]), SOFTMAX_WARPS * 32);
        mbar_init(smem_u32(&sm.bar_o_done), 1);
        mbar_init(smem_u32(&sm.bar_o_final), 1);
        mbar_init(smem_u32(&sm.bar_final), 1);
        for (int q = 0; q < 4; ++q) {
            mbar_init(smem_u32(&sm.bar_group[q][0]), 32 * COL_GROUPS);
            mbar_init(smem_u32(&sm.bar_group[q][1]), 32 * COL_GROUPS);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == WARP_PRODUCER && lane == 0) {
        prefetch_tmap(&tm_qc);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;
    const uint64_t limit = p.limit_ns;

    if (warp == WARP_PRODUCER) {
        // ------------------------------------------------------ producer --
        // All 32 lanes stage the scale atoms; lane 0 arms the barrier and
        // issues the bulk tensor copies after the atoms are written.
        const uint64_t* qs_head = p.q_scales + (size_t)bh * N;
        const uint64_t* ks_head = p.k_scales + (size_t)bh * N;
        const uint32_t qf = smem_u32(&sm.bar_q_full);
        load_scale_atoms(qs_head + q0, N - q0, sm.qs_atom[0], sm.qs_atom[1], lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive_expect_tx(qf, CODE_TILE_BYTES);
            tma_load_3d(smem_u32(sm.qc), &tm_qc, 0, q0, bh, qf);
        }
        int issued = 0;
        uint64_t ksc[4];  // the next tile's scales, fetched before its stage is free
        fetch_scales(ks_head, N, lane, ksc);
        for (int j = 0; j < T; ++j) {
            const int s = j % STAGES;
            if (j >= STAGES) {
                if (!warp_wait(smem_u32(&sm.bar_kv_empty[s]), ((j / STAGES) - 1) & 1, abort_flag, p.status,
                               limit))
                    break;
            }
            const int k0 = j * BN;
            store_scale_atoms(ksc, sm.ks_atom[s][0], sm.ks_atom[s][1], lane);
            if (j + 1 < T) fetch_scales(ks_head + k0 + BN, N - k0 - BN, lane, ksc);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const uint32_t full = smem_u32(&sm.bar_kv_full[s]);
                mbar_arrive_expect_tx(full, CODE_TILE_BYTES + V_TILE_BYTES);
                tma_load_3d(smem_u32(sm.kc[s]), &tm_kc, 0, k0, bh, full);
                tma_load_3d(smem_u32(sm.v[s]), &tm_v, 0, k0, bh, full);
                tma_load_3d(smem_u32(sm.v[s]) + V_PANEL_BYTES, &tm_v, 64, k0, bh, full);
            }
            __syncwarp();
            issued = j + 1;
        }
        if (lane == 0 && *abort_flag) {
            // wind down: let this CTA's own copies land before it exits
            drain_wait(qf, 0);
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                drain_wait(smem_u32(&sm.bar_kv_full[i % STAGES]), (i / STAGES) & 1);
        }
    } else if (warp == WARP_MMA) {
        // ----------------------------------------------------------- MMA --
        bool ok = warp_wait(smem_u32(&sm.bar_q_full), 0, abort_flag, p.status, limit);
        if (ok) {
            if (lane == 0) {
                tc_fence_after();
                tmem_cp_32x128b_x4(tmem + TM_SFQ, atom_desc(sm.qs_atom[0]));
                tmem_cp_32x128b_x4(tmem + TM_SFQ + 4, atom_desc(sm.qs_atom[1]));
            }
            __syncwarp();
        }
        auto pv_step = [&](int i) -> bool {
            if (!warp_wait(smem_u32(&sm.bar_p_ready[i & 1]), (i >> 1) & 1, abort_flag, p.status, limit))
                return false;
            if (lane == 0) {
                tc_fence_after();
                issue_pv(tmem, TM_S0 + 128u * (i & 1), sm.v[i % STAGES], i > 0);
                tc_commit(smem_u32(&sm.bar_kv_empty[i % STAGES]));
                tc_commit(smem_u32(&sm.bar_o_done));
                if (i == T - 1) tc_commit(smem_u32(&sm.bar_o_final));
            }
            __syncwarp();
            return true;
        };
        for (int j = 0; ok && j < T; ++j) {
            const int s = j % STAGES;
            const int b = j & 1;
            if (!warp_wait(smem_u32(&sm.bar_kv_full[s]), (j / STAGES) & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                tc_fence_after();
                const uint32_t sfk = TM_SFK + 8u * b;
                tmem_cp_32x128b_x4(tmem + sfk, atom_desc(sm.ks_atom[s][0]));
                tmem_cp_32x128b_x4(tmem + sfk + 4, atom_desc(sm.ks_atom[s][1]));
                issue_qk(tmem, TM_S0 + 128u * b, sm.qc, sm.kc[s], sfk);
                tc_commit(smem_u32(&sm.bar_s_full[b]));
            }
            __syncwarp();
            if (j >= 1 && !pv_step(j - 1)) {
                ok = false;
                break;
            }
        }
        if (ok && T > 0) pv_step(T - 1);
        // every MMA and copy this warp issued must finish before TMEM is freed
        if (lane == 0) {
            tc_commit(smem_u32(&sm.bar_final));
            drain_wait(smem_u32(&sm.bar_final), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax warps --
        const int quad = warp & 3;  // TMEM sub-partition: rows 32*quad ..
        const int grp = warp >> 2;  // score columns CW*grp .. CW*grp+CW-1 of each tile
        const int row = 32 * quad + lane;
        const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
        float gq = 1.0f, gk = 1.0f;
        if (p.gq) gq = *p.gq;
        if (p.gk) gk = *p.gk;
        if (!(gq > 0.0f && gq < INFINITY && gk > 0.0f && gk < INFINITY)) {
            if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)FP4ATTN_ERR_RANGE);
        }
        const float c = p.scale_log2 * gq * gk;
        const float2 c2 = make_float2(c, c);
        float m_run = -INFINITY;
        float2 lacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
        bool ok = true;
        for (int j = 0; j < T; ++j) {
            const int b = j & 1;
            const uint32_t s_addr = tmem + lane_base + TM_S0 + 128u * b;
            if (!warp_wait(smem_u32(&sm.bar_s_full[b]), (j >> 1) & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[CW32][32];
#pragma unroll
            for (int q = 0; q < CW32; ++q) tmem_ld32(s_addr + (uint32_t)(CW * grp + 32 * q), sr[q]);
            tmem_wait_ld();
            const int nvalid = N - j * BN - CW * grp;
            if (nvalid < CW) {
#pragma unroll
                for (int q = 0; q < CW32; ++q)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * q + i >= nvalid) sr[q][i] = __float_as_uint(-INFINITY);
            }
            // partial row max of this warp's columns: a tree of three-input maxima
            float a[CW / 8];
#pragma unroll
            for (int k = 0; k < CW / 8; ++k) {
                const uint32_t* v = &sr[k >> 2][(k & 3) * 8];
                a[k] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                             fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                             fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
            }
            float pmax = a[0];
#pragma unroll
            for (int k = 1; k < CW / 8; ++k) pmax = fmaxf(pmax, a[k]);
            // exchange with the other column groups of the same rows (after this
            // every S read of the tile is done, so P may overwrite S)
            sm.red_max[b][grp][row] = pmax;
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.bar_group[quad][b]));
            if (!warp_wait(smem_u32(&sm.bar_group[quad][b]), (j >> 1) & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float tmax = sm.red_max[b][0][row];
#pragma unroll
            for (int g = 1; g < COL_GROUPS; ++g) tmax = fmaxf(tmax, sm.red_max[b][g][row]);
            const float mx = tmax * c;
            float alpha = 1.0f;
            bool rescale = false;
            if (mx > m_run + 8.0f) {
                alpha = ex2_approx(m_run - mx);
                m_run = mx;
                rescale = true;
                const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                for (int k = 0; k < 4; ++k) lacc[k] = __fmul2_rn(lacc[k], a2);
            }
            const float2 negm = make_float2(-m_run, -m_run);
            uint32_t pk[CW / 2];
#pragma unroll
            for (int k = 0; k < CW / 2; ++k) {
                const float2 s2 = make_float2(__uint_as_float(sr[k >> 4][(2 * k) & 31]),
                                              __uint_as_float(sr[k >> 4][(2 * k + 1) & 31]));
                const float2 x = __ffma2_rn(s2, c2, negm);
                float2 pv;
                if ((k & 7) < POLY_PAIRS_PER_8) {
                    pv = exp2_poly2(x);
                } else {
                    pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                }
                lacc[k & 3] = __fadd2_rn(lacc[k & 3], pv);
                pk[k] = pack_bf16x2(pv.x, pv.y);
            }
            // P (bf16 pairs) over this warp's CW/2 columns of the S buffer
            if constexpr (CW == 64) {
                tmem_st32(s_addr + 32u * grp, *reinterpret_cast<const uint32_t(*)[32]>(pk));
            } else {
                tmem_st16(s_addr + 16u * grp, pk);
            }
            tmem_wait_st();
            // tcgen05.ld/st are warp-collective: the whole warp takes this branch
            // when any of its rows needs it (alpha is 1 elsewhere).  Only then
            // does it wait for tile j-1's P.V: S(j) being ready means every
            // earlier P.V has completed, so that is the only one in flight and
            // the parity wait is unambiguous.
            if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
                if (!warp_wait(smem_u32(&sm.bar_o_done), (j - 1) & 1, abort_flag, p.status, limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t o_addr = tmem + lane_base + TM_O + (uint32_t)(CW * grp);
                const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                for (int q = 0; q < CW32; ++q) {
                    uint32_t r[32];
                    tmem_ld32(o_addr + 32u * q, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float2 o2 =
                            __fmul2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), a2);
                        r[i] = __float_as_uint(o2.x);
                        r[i + 1] = __float_as_uint(o2.y);
                    }
                    tmem_st32(o_addr + 32u * q, r);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.bar_p_ready[b]));
        }
        if (ok && T > 0) {
            // total row sum over the column groups (the group barrier's next phase)
            const float l_part = (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y) + (lacc[2].x + lacc[2].y) +
                                 (lacc[3].x + lacc[3].y);
            sm.red_sum[grp][row] = l_part;
            mbar_arrive(smem_u32(&sm.bar_group[quad][T & 1]));
            ok = warp_wait(smem_u32(&sm.bar_group[quad][T & 1]), (T >> 1) & 1, abort_flag, p.status, limit);
            float l = sm.red_sum[0][row];
#pragma unroll
            for (int g = 1; g < COL_GROUPS; ++g) l += sm.red_sum[g][row];
            if (ok && warp_wait(smem_u32(&sm.bar_o_final), 0, abort_flag, p.status, limit)) {
                tc_fence_after();
                const float inv_l = 1.0f / l;
                const uint32_t o_addr = tmem + lane_base + TM_O + (uint32_t)(CW * grp);
                const int n = q0 + row;
                const size_t orow = (size_t)bh * N + n;
#pragma unroll
                for (int q = 0; q < CW32; ++q) {
                    uint32_t r[32];
                    tmem_ld32(o_addr + 32u * q, r);
                    tmem_wait_ld();
                    if (n < N) {
                        uint4* dst = reinterpret_cast<uint4*>(p.o + orow * 128 + CW * grp + 32 * q);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = 8 * v + 2 * e;
                                w[e] = pack_bf16x2(__uint_as_float(r[i]) * inv_l, __uint_as_float(r[i + 1]) * inv_l);
                            }
                            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (p.lse && n < N && grp == 0) p.lse[orow] = (m_run + __log2f(l)) * 0.69314718055994530942f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------- probes ----

struct ProbeSmem {
    uint8_t v[V_TILE_BYTES];
    uint8_t kc[CODE_TILE_BYTES];
    uint8_t qc[CODE_TILE_BYTES];
    uint8_t ks_atom[2][512];
    uint8_t qs_atom[2][512];
    uint64_t bar_full;
    uint64_t bar_done;
    uint32_t tmem_base;
    int abort_flag;
};

// mode 0: S = Qc Kc^T into out; mode 1: O = P V into out (P given in pbf).
__global__ void __launch_bounds__(160, 1)
    probe_kernel(const __grid_constant__ CUtensorMap tm_qc, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_v, const uint64_t* q_scales, const uint64_t* k_scales,
                 const __nv_bfloat16* pbf, float* out, int mode, int* status) {
    extern __shared__ uint8_t smem_raw[];
    ProbeSmem& sm = *align1024<ProbeSmem>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.bar_full), 1);
        mbar_init(smem_u32(&sm.bar_done), 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;
    const uint32_t full = smem_u32(&sm.bar_full);
    if (mode == 0 && warp == 4) {
        // the same scale staging as the attention kernel's producer warp
        load_scale_atoms(q_scales, 128, sm.qs_atom[0], sm.qs_atom[1], lane);
        load_scale_atoms(k_scales, 128, sm.ks_atom[0], sm.ks_atom[1], lane);
        fence_proxy_async_smem();
        __syncwarp();
    }
    if (threadIdx.x == 128) {
        if (mode == 0) {
            mbar_arrive_expect_tx(full, 2 * CODE_TILE_BYTES);
            tma_load_3d(smem_u32(sm.qc), &tm_qc, 0, 0, 0, full);
            tma_load_3d(smem_u32(sm.kc), &tm_kc, 0, 0, 0, full);
        } else {
            mbar_arrive_expect_tx(full, V_TILE_BYTES);
            tma_load_3d(smem_u32(sm.v), &tm_v, 0, 0, 0, full);
            tma_load_3d(smem_u32(sm.v) + V_PANEL_BYTES, &tm_v, 64, 0, 0, full);
        }
    }
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    if (mode == 1 && warp < 4) {
        // write P into TMEM exactly as the softmax warps do
        const int row = 32 * warp + lane;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(pbf + (size_t)row * 128);
        uint32_t pk[2][32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            pk[0][i] = src[i];
            pk[1][i] = src[32 + i];
        }
        tmem_st32(tmem + lane_base + TM_S0, pk[0]);
        tmem_st32(tmem + lane_base + TM_S0 + 32u, pk[1]);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        ok = warp_wait(full, 0, abort_flag, status, kWaitLimitNs);
        if (ok) {
            if (lane == 0) {
                tc_fence_after();
                if (mode == 0) {
                    tmem_cp_32x128b_x4(tmem + TM_SFQ, atom_desc(sm.qs_atom[0]));
                    tmem_cp_32x128b_x4(tmem + TM_SFQ + 4, atom_desc(sm.qs_atom[1]));
                    tmem_cp_32x128b_x4(tmem + TM_SFK, atom_desc(sm.ks_atom[0]));
                    tmem_cp_32x128b_x4(tmem + TM_SFK + 4, atom_desc(sm.ks_atom[1]));
                    issue_qk(tmem, TM_S0 + 128u, sm.qc, sm.kc, TM_SFK);
                } else {
                    issue_pv(tmem, TM_S0, sm.v, false);
                }
            }
        }
        if (lane == 0) tc_commit(smem_u32(&sm.bar_done));
        __syncwarp();
    }
    if (warp < 4) {
        const int row = 32 * warp + lane;
        const uint32_t col = (mode == 0) ? TM_S0 + 128u : TM_O;
        if (warp_wait(smem_u32(&sm.bar_done), 0, abort_flag, status, kWaitLimitNs)) {
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + col + 32u * q, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) out[(size_t)row * 128 + 32 * q + i] = __uint_as_float(r[i]);
            }
        }
    } else if (lane == 0) {
        drain_wait(smem_u32(&sm.bar_done), 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

__global__ void wait_timeout_kernel(int* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // nothing ever arrives on this barrier: the wait must give up by itself
    warp_wait(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
}

// ---------------------------------------------------------- host side ----

struct Maps {
    CUtensorMap qc, kc, v;
};

// Codes [BH][N][64 bytes]: 64B-swizzled boxes of 128 rows; x is always 0.
bool make_code_map(CUtensorMap* m, const uint8_t* base, int BH, int N) {
    const uint64_t dims[3] = {64, (uint64_t)N, (uint64_t)BH};
    const uint64_t strides[2] = {64, (uint64_t)N * 64};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

// V [BH][N][128 bf16]: 128B-swizzled boxes of 64 channels x 128 keys; x is 0 or 64
// (0 or 128 bytes), so every box starts on a 16-byte boundary.
bool make_v_map(CUtensorMap* m, const __nv_bfloat16* base, int BH, int N) {
    const uint64_t dims[3] = {128, (uint64_t)N, (uint64_t)BH};
    const uint64_t strides[2] = {256, (uint64_t)N * 256};
    const uint32_t box[3] = {64, 128, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(base),
                             dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t fwd_smem_bytes() { return sizeof(FwdSmem) + 1024; }
size_t probe_smem_bytes() { return sizeof(ProbeSmem) + 1024; }

}  // namespace

int launch_forward(const FwdArgs& a, cudaStream_t stream) {
    if (a.BH == 0 || a.N == 0) return FP4ATTN_OK;
    Maps m;
    if (!make_code_map(&m.qc, a.q_codes, a.BH, a.N) || !make_code_map(&m.kc, a.k_codes, a.BH, a.N) ||
        !make_v_map(&m.v, a.v, a.BH, a.N))
        return FP4ATTN_ERR_CUDA;
    static_assert(sizeof(FwdSmem) + 1024 <= 227 * 1024, "shared memory budget");
    const size_t smem = fwd_smem_bytes();
    if (cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return FP4ATTN_ERR_CUDA;
    FwdParams p;
    p.q_scales = reinterpret_cast<const uint64_t*>(a.q_scales);
    p.k_scales = reinterpret_cast<const uint64_t*>(a.k_scales);
    p.N = a.N;
    p.n_kt = (a.N + BN - 1) / BN;
    const float scale = a.softmax_scale > 0.0f ? a.softmax_scale : 0.08838834764831845f;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.gq = a.gq;
    p.gk = a.gk;
    p.o = a.o;
    p.lse = a.lse;
    p.status = a.status;
    p.limit_ns = kWaitLimitNs;
    dim3 grid((a.N + BM - 1) / BM, a.BH);
    fwd_kernel<<<grid, FWD_THREADS, smem, stream>>>(m.qc, m.kc, m.v, p);
    return cudaGetLastError() == cudaSuccess ? FP4ATTN_OK : FP4ATTN_ERR_CUDA;
}

static int launch_probe(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                        const __nv_bfloat16* p, const __nv_bfloat16* v, float* out, int mode,
                        cudaStream_t stream) {
    Maps m;
    if (mode == 0) {
        if (!make_code_map(&m.qc, qc, 1, 128) || !make_code_map(&m.kc, kc, 1, 128)) return FP4ATTN_ERR_CUDA;
        m.v = m.qc;  // unused in this mode
    } else {
        if (!make_v_map(&m.v, v, 1, 128)) return FP4ATTN_ERR_CUDA;
        m.qc = m.kc = m.v;  // unused in this mode
    }
    const size_t smem = probe_smem_bytes();
    if (cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return FP4ATTN_ERR_CUDA;
    probe_kernel<<<1, 160, smem, stream>>>(m.qc, m.kc, m.v, reinterpret_cast<const uint64_t*>(qs),
                                           reinterpret_cast<const uint64_t*>(ks), p, out, mode, nullptr);
    return cudaGetLastError() == cudaSuccess ? FP4ATTN_OK : FP4ATTN_ERR_CUDA;
}

int launch_probe_qk(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                    float* s_out, cudaStream_t stream) {
    return launch_probe(qc, qs, kc, ks, nullptr, nullptr, s_out, 0, stream);
}

int launch_probe_pv(const __nv_bfloat16* p, const __nv_bfloat16* v, float* o_out, cudaStream_t stream) {
    return launch_probe(nullptr, nullptr, nullptr, nullptr, p, v, o_out, 1, stream);
}

int launch_probe_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t stream) {
    wait_timeout_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError() == cudaSuccess ? FP4ATTN_OK : FP4ATTN_ERR_CUDA;
}

}  // namespace fp4attn
