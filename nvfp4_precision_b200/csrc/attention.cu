// Non-causal FP4 attention: O = softmax(scale * Q K^T) V with NVFP4 Q and K
// (block-scaled E2M1, one UE4M3 scale per 16 channels) and BF16 P and V.
//
// Method: FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention":
// queries and keys are quantised for an NVFP4 attention kernel; P and V stay
// in BF16.  This kernel is written for sm_100a:
//   * one CTA per (head, 256 queries) = two 128-row query tiles that share
//     every K/V tile loaded into shared memory; 384 threads:
//       warps 0-3  softmax of query tile 0, warps 4-7 softmax of tile 1 (one
//                  warp per TMEM sub-partition, one query row per thread);
//       warp 8     producer: scale-factor atoms (plain loads) and TMA copies
//                  of both Q tiles once, then K codes and V of 112 keys per
//                  stage into a STAGES-deep shared-memory ring;
//       warp 9     TMEM owner and MMA issuer: stages scale factors into TMEM
//                  (tcgen05.cp), S_i = Q_i K^T with tcgen05.mma
//                  kind::mxf4nvf4 (block16 UE4M3 scales) into TMEM, and
//                  O_i += P_i V with tcgen05.mma kind::f16 from shared memory;
//       warps 10-11 idle: they complete the third warpgroup, whose registers
//                  go to the softmax warpgroups (setmaxnreg 216 / 64);
//   * P_i goes to shared memory (K-major, 32-byte swizzle, one 4 KB panel per
//     16 keys), not back into TMEM, so S_i is free as soon as its softmax
//     warps have loaded it: S_i of the next stage is computed while they
//     still work on this one, and each softmax warp group moves from stage to
//     stage without waiting for the tensor cores;
//   * TMEM (512 columns): S_0 [0,112), S_1 [112,224) fp32, O_0 [224,352),
//     O_1 [352,480), the two Q tiles' scale factors [480,496) and two slots
//     of K scale factors [496,512).  112 keys per stage is what lets four
//     accumulators and the scale factors fit the 512 columns together;
//   * online softmax in the log2 domain with a lazy running max: the max
//     only moves when a stage's max exceeds it by more than 8 (so p <= 256),
//     and only then is O_i rescaled in TMEM, after the previous P_i V has
//     completed.  Exponentials are split between MUFU ex2 and a polynomial on
//     the FMA pipe, with packed fp32x2 arithmetic.  The row sum l is taken
//     over the same bf16-rounded P that enters P V (each bf16 value widened
//     exactly and added in fp32), so O / l is a convex combination of rows of
//     V with the rounded weights: a row dominated by one key gets that key's
//     V row back exactly, whatever the rounding of its p (which the lazy max
//     leaves anywhere in (1, 256]).
// Every wait is bounded; a wait that runs out raises FP4ATTN_ERR_TIMEOUT in
// the status word and the CTA winds down (waiting for its own copies and MMAs)
// instead of hanging.
#include <cuda_bf16.h>

#include "fp4_operands.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int QT = 2;    // query tiles per CTA
constexpr int BN = 112;  // keys per K/V stage
constexpr int STAGES = 4;
constexpr int SOFTMAX_WARPS = 4 * QT;
// Warpgroups 0 and 1 are the softmax warps, warpgroup 2 holds the producer and
// the MMA warp (its last two warps only take part in the register split).
constexpr int FWD_THREADS = 32 * (SOFTMAX_WARPS + 4);
constexpr int WARP_PRODUCER = SOFTMAX_WARPS;
constexpr int WARP_MMA = SOFTMAX_WARPS + 1;
// Register split: three warps share each SM sub-partition's 16384 registers,
// so the launch gets 168 per thread; the producer/MMA warpgroup gives most of
// its share to the softmax warpgroups (2 x 128 x 216 + 128 x 64 <= 384 x 168).
// Measured: the softmax warps spill below 216; 64 for the producer and MMA
// warps beats 56 (fewer spills there) and, oddly, 72.
constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 216, SUPPORT_REGS = 64;
static_assert(2 * 128 * SOFTMAX_REGS + 128 * SUPPORT_REGS <= FWD_THREADS * LAUNCH_REGS, "register split");
static_assert((2 * SOFTMAX_REGS + SUPPORT_REGS) * 32 <= 16384, "registers of one SM sub-partition");
// Of every 8 pairs of exponentials, this many go to the FMA-pipe polynomial
// and the rest to MUFU ex2 (MUFU issues 16 per clock per SM).
#ifndef FP4ATTN_POLY_PAIRS
#define FP4ATTN_POLY_PAIRS 3
#endif
constexpr int POLY_PAIRS_PER_8 = FP4ATTN_POLY_PAIRS;

constexpr uint32_t TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t tm_s(int i) { return (uint32_t)(BN * i); }
__host__ __device__ constexpr uint32_t tm_o(int i) { return (uint32_t)(2 * BN + 128 * i); }
__host__ __device__ constexpr uint32_t tm_sfq(int i) { return (uint32_t)(2 * BN + 256 + 8 * i); }
__host__ __device__ constexpr uint32_t tm_sfk(int slot) { return (uint32_t)(2 * BN + 256 + 16 + 8 * slot); }
static_assert(tm_sfk(1) + 8 == TMEM_COLS, "TMEM budget");

constexpr uint32_t Q_TILE_BYTES = BM * 64;         // 128 rows x 128 E2M1 values
constexpr uint32_t K_TILE_BYTES = BN * 64;         // 112 rows x 128 E2M1 values
constexpr uint32_t V_PANEL_BYTES = BN * 64 * 2;    // 112 keys x 64 channels bf16
constexpr uint32_t V_TILE_BYTES = 2 * V_PANEL_BYTES;
static_assert(K_TILE_BYTES % 1024 == 0 && V_PANEL_BYTES % 1024 == 0, "swizzle atoms stay 1 KB aligned");
// P in shared memory: one panel per 16 keys, 128 rows x 32 bytes (16 bf16),
// K-major with the 32-byte swizzle (the two 16-byte halves of a row swap
// places in rows 4-7 of every 8-row group); 8-row groups 256 B apart.
constexpr uint32_t P_PANEL_BYTES = BM * 32;
constexpr uint32_t P_TILE_BYTES = (BN / 16) * P_PANEL_BYTES;

// Instruction descriptors.
//  S: kind::mxf4nvf4, A = B = E2M1 (1), UE4M3 scales, K-major, M = 128, N = n keys.
__host__ __device__ constexpr uint32_t idesc_qk(int n) { return idesc_mxf4(BM, n); }
//  O: kind::f16, fp32 accumulate (1 << 4), A = B = BF16, A = P K-major,
//     B = V MN-major (1 << 16), N = 128 channels, M = 128.
constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct __align__(1024) FwdSmem {
    uint8_t v[STAGES][V_TILE_BYTES];   // two 64-channel panels, 128B swizzle
    uint8_t kc[STAGES][K_TILE_BYTES];  // 64B swizzle
    uint8_t qc[QT][Q_TILE_BYTES];      // 64B swizzle
    uint8_t pb[QT][P_TILE_BYTES];      // P_i, 32B swizzle
    uint8_t ks_atom[STAGES][2][512];   // scale-factor atoms for tcgen05.cp
    uint8_t qs_atom[QT][2][512];
    uint64_t bar_q_full;
    uint64_t bar_kv_full[STAGES];
    uint64_t bar_kv_empty[STAGES];
    uint64_t bar_s_full[QT];   // S_i of the next stage is in TMEM
    uint64_t bar_s_free[QT];   // the softmax warps of tile i have loaded S_i into registers
    uint64_t bar_p_full[QT];   // P_i of the stage is in shared memory (O_i rescaled if needed)
    uint64_t bar_pv_done[QT];  // O_i += P_i V of the stage has completed (P_i buffer free)
    uint64_t bar_final;        // every MMA and copy of the CTA has completed
    uint32_t tmem_base;
    int abort_flag;
};

struct FwdParams {
    const uint8_t* q_scales;  // srb UE4M3 bytes per row
    const uint8_t* k_scales;
    int srb;                  // scale bytes per row: 8 (128 channels) or 4 (64)
    int o_chunks;             // 32-channel chunks of O to store: 4, or 2 for 64 channels
    int N;
    int n_kt;          // K/V stages of BN keys
    float scale_log2;  // softmax_scale * log2(e)
    const float* gq;
    const float* gk;
    __nv_bfloat16* o;
    long long o_sb, o_sh, o_sn;  // element strides of O ([B,H,N,128], channels contiguous)
    int H;
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

__device__ __forceinline__ uint64_t v_desc(const uint8_t* tile, int kstep, uint32_t panel_bytes) {
    // MN-major 128B swizzle: the two 64-channel panels panel_bytes apart
    // (leading byte offset), 8-key groups 1 KB apart (stride byte offset);
    // one MMA covers 16 keys = 2 KB of each panel.
    return smem_desc(smem_u32(tile) + 2048u * kstep, panel_bytes, 1024, LAYOUT_SW128);
}

__device__ __forceinline__ uint64_t p_desc(const uint8_t* p_tile, int kstep) {
    // K-major 32B swizzle: one panel of 128 rows x 32 bytes per 16 keys,
    // 8-row groups 256 B apart (stride byte offset); the leading byte offset
    // is unused because one MMA's K extent is the swizzle width.
    return smem_desc(smem_u32(p_tile) + P_PANEL_BYTES * kstep, 16, 256, LAYOUT_SW32);
}

// Row `row` of P (NP panels of 16 keys; pk = 8 NP bf16 pairs, key order) into
// the 32B-swizzled layout p_desc reads.  A warp's 32 rows hit all 32 banks
// once per 8 lanes, so each 16-byte store takes the minimum four wavefronts.
template <int NP>
__device__ __forceinline__ void store_p_row(uint8_t* p_tile, int row, const uint32_t* pk) {
    const uint32_t sw = (uint32_t)(row >> 2) & 1u;
    uint8_t* base = p_tile + 32 * row;
#pragma unroll
    for (int ks = 0; ks < NP; ++ks) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t* w = pk + 8 * ks + 4 * h;
            *reinterpret_cast<uint4*>(base + P_PANEL_BYTES * ks + 16u * ((uint32_t)h ^ sw)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// S = Q K^T over all 128 channels for one query tile and n keys: two K=64
// block-scaled MMAs, scale factors of Q at sfq_col, of K at sfk_col.
__device__ __forceinline__ void issue_qk(uint32_t tmem, uint32_t s_col, const uint8_t* qc, const uint8_t* kc,
                                         uint32_t sfq_col, uint32_t sfk_col, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        mma_mxf4nvf4(tmem + s_col, codes_desc(qc, kk), codes_desc(kc, kk), idesc, tmem + sfq_col + 4u * kk,
                     tmem + sfk_col + 4u * kk, kk > 0 ? 1u : 0u);
    }
}

// O (+)= P V over NK keys (NK/16 K=16 BF16 MMAs, P from shared memory).
template <int NK>
__device__ __forceinline__ void issue_pv(uint32_t tmem, uint32_t o_col, const uint8_t* p_tile, const uint8_t* v,
                                         uint32_t v_panel_bytes, bool accumulate_first) {
#pragma unroll
    for (int ks = 0; ks < NK / 16; ++ks) {
        mma_bf16_ss(tmem + o_col, p_desc(p_tile, ks), v_desc(v, ks, v_panel_bytes), IDESC_PV,
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
    const int q0 = blockIdx.x * (QT * BM);
    const int T = p.n_kt;
    const int N = p.N;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.bar_q_full), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm.bar_kv_full[s]), 1);
            mbar_init(smem_u32(&sm.bar_kv_empty[s]), 1);
        }
        for (int i = 0; i < QT; ++i) {
            mbar_init(smem_u32(&sm.bar_s_full[i]), 1);
            mbar_init(smem_u32(&sm.bar_s_free[i]), 128);
            mbar_init(smem_u32(&sm.bar_p_full[i]), 128);
            mbar_init(smem_u32(&sm.bar_pv_done[i]), 1);
        }
        mbar_init(smem_u32(&sm.bar_final), 1);
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
    if (warp >= SOFTMAX_WARPS) {
    setmaxnreg_dec<SUPPORT_REGS>();
    if (warp == WARP_PRODUCER) {
        // ------------------------------------------------------ producer --
        // All 32 lanes stage the scale atoms; lane 0 arms the barrier and
        // issues the bulk tensor copies after the atoms are written.  A query
        // tile that lies past N is copied all the same (the copy fills zeros)
        // and its rows are never stored.
        const int srb = p.srb;
        const uint8_t* qs_head = p.q_scales + (size_t)bh * N * srb;
        const uint8_t* ks_head = p.k_scales + (size_t)bh * N * srb;
        const int v_b = bh / p.H, v_h = bh - v_b * p.H;  // V is addressed as [B][H][N][128]
        const uint32_t qf = smem_u32(&sm.bar_q_full);
#pragma unroll
        for (int i = 0; i < QT; ++i) {
            const int r0 = q0 + BM * i;
            uint64_t w[4];
            fetch_scales_rows(qs_head + (size_t)(r0 < N ? r0 : 0) * srb, srb, N - r0, lane, w);
            store_scale_atoms(w, sm.qs_atom[i][0], sm.qs_atom[i][1], lane);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive_expect_tx(qf, QT * Q_TILE_BYTES);
#pragma unroll
            for (int i = 0; i < QT; ++i) tma_load_3d(smem_u32(sm.qc[i]), &tm_qc, 0, q0 + BM * i, bh, qf);
        }
        int issued = 0;
        uint64_t ksc[4];  // the next stage's scales, fetched before its buffer is free
        fetch_scales_rows(ks_head, srb, N < BN ? N : BN, lane, ksc);
        for (int j = 0; j < T; ++j) {
            const int s = j % STAGES;
            if (j >= STAGES) {
                if (!warp_wait(smem_u32(&sm.bar_kv_empty[s]), ((j / STAGES) - 1) & 1, abort_flag, p.status,
                               limit))
                    break;
            }
            const int k0 = j * BN;
            store_scale_atoms(ksc, sm.ks_atom[s][0], sm.ks_atom[s][1], lane);
            if (j + 1 < T) {
                const int rest = N - k0 - BN;
                fetch_scales_rows(ks_head + (size_t)(k0 + BN) * srb, srb, rest < BN ? rest : BN, lane, ksc);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const uint32_t full = smem_u32(&sm.bar_kv_full[s]);
                mbar_arrive_expect_tx(full, K_TILE_BYTES + V_TILE_BYTES);
                tma_load_3d(smem_u32(sm.kc[s]), &tm_kc, 0, k0, bh, full);
                tma_load_4d(smem_u32(sm.v[s]), &tm_v, 0, k0, v_h, v_b, full);
                tma_load_4d(smem_u32(sm.v[s]) + V_PANEL_BYTES, &tm_v, 64, k0, v_h, v_b, full);
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
        // Issue order: S_0(0) S_1(0) S_0(1) S_1(1), then per stage j
        //   O_0 += P_0(j) V_j,  S_0(j+2),  O_1 += P_1(j) V_j,  S_1(j+2).
        // S_i(j+2) waits until the softmax warps have loaded S_i(j+1), and
        // O_i += P_i(j) V_j until P_i(j) is in shared memory; the softmax
        // warps only ever wait for work issued before, so nothing can wait
        // in a circle.  A K scale-factor slot is refilled for stage j+2 once
        // S_0(j+1) has been loaded: S_0(j+1) was issued after the last reader
        // of the slot (S_1(j)), and tcgen05 operations of one thread complete
        // in order.
        //
        // This warp is on the critical path of both tiles, so it keeps its
        // instruction stream short: every shared-memory descriptor is a base
        // computed once plus a constant (the address field of a descriptor
        // is the byte address / 16 and never carries into the next field,
        // shared memory being below 256 KB), the descriptors live in
        // warp-uniform registers and one elected lane issues, and its waits
        // poll instead of suspending.
        const bool leader = elect_one_sync();
        const uint64_t qd = codes_desc(sm.qc[0], 0);      // tile i: + i*Q_TILE/16, chunk kk: + 2 kk
        const uint64_t kd0 = codes_desc(sm.kc[0], 0);     // stage st: + st*K_TILE/16
        const uint64_t vd0 = v_desc(sm.v[0], 0, V_PANEL_BYTES);  // stage st: + st*V_TILE/16, kstep: + 128
        const uint64_t pd0 = p_desc(sm.pb[0], 0);         // tile i: + i*P_TILE/16, kstep: + P_PANEL/16
        const uint64_t kad0 = atom_desc(sm.ks_atom[0][0]);  // stage st: + 64 st, half h: + 32 h
        constexpr uint64_t QD_TILE = Q_TILE_BYTES >> 4, KD_STAGE = K_TILE_BYTES >> 4,
                           VD_STAGE = V_TILE_BYTES >> 4, PD_TILE = P_TILE_BYTES >> 4,
                           PD_STEP = P_PANEL_BYTES >> 4, AD_STAGE = (2 * 512) >> 4;
        constexpr uint32_t IDESC_S = idesc_qk(BN);
        auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait_spin(bar, parity, abort_flag, p.status, limit));
        };
        // S_i(j): for i == 0 also stage the K scale factors of stage j
        auto qk = [&](int i, int j) {
            const int st = j % STAGES;
            const uint32_t sfk = tm_sfk(j & 1);
            const uint64_t kd = kd0 + KD_STAGE * st;
            if (i == 0) {
                const uint64_t kad = kad0 + AD_STAGE * st;
                tmem_cp_32x128b_x4(tmem + sfk, kad);
                tmem_cp_32x128b_x4(tmem + sfk + 4, kad + 32);
            }
            mma_mxf4nvf4(tmem + tm_s(i), qd + QD_TILE * i, kd, IDESC_S, tmem + tm_sfq(i), tmem + sfk, 0u);
            mma_mxf4nvf4(tmem + tm_s(i), qd + QD_TILE * i + 2, kd + 2, IDESC_S, tmem + tm_sfq(i) + 4,
                         tmem + sfk + 4, 1u);
            tc_commit(smem_u32(&sm.bar_s_full[i]));
        };
        auto pv = [&](int i, int j) {
            const uint64_t vd = vd0 + VD_STAGE * (j % STAGES);
            const uint64_t pd = pd0 + PD_TILE * i;
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks)
                mma_bf16_ss(tmem + tm_o(i), pd + PD_STEP * ks, vd + 128u * ks, IDESC_PV,
                            (ks > 0 || j > 0) ? 1u : 0u);
            tc_commit(smem_u32(&sm.bar_pv_done[i]));
        };
        bool ok = wait(smem_u32(&sm.bar_q_full), 0);
        if (ok && leader) {
            tc_fence_after();
            const uint64_t qad = atom_desc(sm.qs_atom[0][0]);  // tile i: + 64 i, half h: + 32 h
#pragma unroll
            for (int i = 0; i < QT; ++i) {
                tmem_cp_32x128b_x4(tmem + tm_sfq(i), qad + AD_STAGE * i);
                tmem_cp_32x128b_x4(tmem + tm_sfq(i) + 4, qad + AD_STAGE * i + 32);
            }
        }
        __syncwarp();
        // S of the first two stages
        for (int j = 0; ok && j < 2 && j < T; ++j) {
            ok = wait(smem_u32(&sm.bar_kv_full[j]), 0);
            for (int i = 0; ok && i < QT; ++i) {
                if (j == 1) ok = wait(smem_u32(&sm.bar_s_free[i]), 0);
                if (ok && leader) {
                    tc_fence_after();
                    qk(i, j);
                }
                __syncwarp();
            }
        }
        for (int j = 0; ok && j < T; ++j) {
            const int jn = j + 2;  // stage whose S is computed next
            for (int i = 0; i < QT; ++i) {
                if (!wait(smem_u32(&sm.bar_p_full[i]), j & 1)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    tc_fence_after();
                    pv(i, j);
                    if (i == QT - 1) tc_commit(smem_u32(&sm.bar_kv_empty[j % STAGES]));
                }
                __syncwarp();
                if (jn < T) {
                    if (!wait(smem_u32(&sm.bar_s_free[i]), (jn - 1) & 1) ||
                        (i == 0 && !wait(smem_u32(&sm.bar_kv_full[jn % STAGES]), (jn / STAGES) & 1))) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        tc_fence_after();
                        qk(i, jn);
                    }
                    __syncwarp();
                }
            }
        }
        // every MMA and copy this warp issued must finish before TMEM is freed
        if (leader) {
            tc_commit(smem_u32(&sm.bar_final));
            drain_wait(smem_u32(&sm.bar_final), 0);
        }
        __syncwarp();
    }
    } else {
        setmaxnreg_inc<SOFTMAX_REGS>();
        // ------------------------------------------------ softmax warps --
        const int quad = warp & 3;  // TMEM sub-partition: rows 32*quad ..
        const int qt = warp >> 2;   // query tile of this warp group
        const int row = 32 * quad + lane;
        const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
        const uint32_t s_addr = tmem + lane_base + tm_s(qt);
        const uint32_t o_addr = tmem + lane_base + tm_o(qt);
        float gq = 1.0f, gk = 1.0f;
        if (p.gq) gq = *p.gq;
        if (p.gk) gk = *p.gk;
        if (!(gq > 0.0f && gq < INFINITY && gk > 0.0f && gk < INFINITY)) {
            if (threadIdx.x == 0) atomicCAS(p.status, 0, (int)FP4ATTN_ERR_RANGE);
        }
        const float c = p.scale_log2 * gq * gk;
        const float2 c2 = make_float2(c, c);
        float m_run = -INFINITY;  // running max (log2 domain) that P, O and the row sum are relative to
        float2 lacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
        const uint32_t s_full = smem_u32(&sm.bar_s_full[qt]);
        const uint32_t s_free = smem_u32(&sm.bar_s_free[qt]);
        const uint32_t p_full = smem_u32(&sm.bar_p_full[qt]);
        const uint32_t pv_done = smem_u32(&sm.bar_pv_done[qt]);
        uint8_t* p_tile = sm.pb[qt];
        bool ok = true;
        for (int j = 0; j < T; ++j) {
            if (!warp_wait(s_full, j & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[BN];
            tmem_ld32(s_addr, &sr[0]);
            tmem_ld32(s_addr + 32u, &sr[32]);
            tmem_ld32(s_addr + 64u, &sr[64]);
            tmem_ld16(s_addr + 96u, &sr[96]);
            tmem_wait_ld();
            // S_i is in registers: the MMA warp may compute the next stage into it
            tc_fence_before();
            mbar_arrive(s_free);
            const int nvalid = N - j * BN;
            if (nvalid < BN) {
#pragma unroll
                for (int k = 0; k < BN; ++k)
                    if (k >= nvalid) sr[k] = __float_as_uint(-INFINITY);
            }
            // row max of the stage: a tree of three-input maxima
            float a[BN / 8];
#pragma unroll
            for (int g = 0; g < BN / 8; ++g) {
                const uint32_t* v = &sr[8 * g];
                a[g] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                             fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                             fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
            }
            static_assert(BN / 8 == 14, "max tree below covers 14 groups");
            const float mx = fmax3(fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmax3(a[6], a[7], a[8])),
                                   fmax3(a[9], a[10], a[11]), fmaxf(a[12], a[13])) * c;
            // lazy running max: move it only when the stage exceeds it by more than 8
            const float m_new = (mx > m_run + 8.0f) ? mx : m_run;
            const bool moved = m_new != m_run;
            const float alpha = moved ? ex2_approx(m_run - m_new) : 1.0f;  // 0 on the first stage
            if (moved) {
                const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                for (int k = 0; k < 4; ++k) lacc[k] = __fmul2_rn(lacc[k], a2);
            }
            m_run = m_new;
            const float2 negm = make_float2(-m_run, -m_run);
            uint32_t pk[BN / 2];
#pragma unroll
            for (int k = 0; k < BN / 2; ++k) {
                const float2 s2 = make_float2(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
                const float2 x = __ffma2_rn(s2, c2, negm);
                float2 pv;
                if ((k & 7) < POLY_PAIRS_PER_8) {
                    pv = exp2_poly2(x);
                } else {
                    pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                }
                pk[k] = pack_bf16x2(pv.x, pv.y);
                lacc[k & 3] = add_bf16x2_to_f32x2(pk[k], lacc[k & 3]);
            }
            if (j > 0) {
                // the previous P_i V has completed: its P buffer is free and O_i
                // holds every earlier stage
                if (!warp_wait(pv_done, (j - 1) & 1, abort_flag, p.status, limit)) {
                    ok = false;
                    break;
                }
                // rescale O_i when any row of the warp moved its max (whole warp:
                // tcgen05.ld/st are warp-collective; alpha is 1 for other rows)
                if (__any_sync(0xffffffffu, moved)) {
                    tc_fence_after();
                    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t r[32];
                        tmem_ld32(o_addr + 32u * q, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; k += 2) {
                            const float2 o2 =
                                __fmul2_rn(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), a2);
                            r[k] = __float_as_uint(o2.x);
                            r[k + 1] = __float_as_uint(o2.y);
                        }
                        tmem_st32(o_addr + 32u * q, r);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                }
            }
            store_p_row<BN / 16>(p_tile, row, pk);
            fence_proxy_async_smem();  // P is read by the tensor cores (async proxy)
            mbar_arrive(p_full);
        }
        if (ok && T > 0 && warp_wait(pv_done, (T - 1) & 1, abort_flag, p.status, limit)) {
            tc_fence_after();
            const float l = (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y) + (lacc[2].x + lacc[2].y) +
                            (lacc[3].x + lacc[3].y);
            const float inv_l = 1.0f / l;
            const int n = q0 + BM * qt + row;
            const size_t orow = (size_t)bh * N + n;
            const int ob = bh / p.H, oh = bh - ob * p.H;
            __nv_bfloat16* o_row = p.o + ob * p.o_sb + oh * p.o_sh + (long long)n * p.o_sn;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (q >= p.o_chunks) break;  // warp-uniform
                uint32_t r[32];
                tmem_ld32(o_addr + 32u * q, r);
                tmem_wait_ld();
                if (n < N && FP4ATTN_IN_BOUNDS(bh < (int)gridDim.y, p.status)) {
                    uint4* dst = reinterpret_cast<uint4*>(o_row + 32 * q);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 8 * v + 2 * e;
                            w[e] = pack_bf16x2(__uint_as_float(r[k]) * inv_l, __uint_as_float(r[k + 1]) * inv_l);
                        }
                        dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (p.lse && n < N && FP4ATTN_IN_BOUNDS(orow < (size_t)gridDim.y * N, p.status))
                p.lse[orow] = (m_run + __log2f(l)) * 0.69314718055994530942f;
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
// One 128x128 tile through the forward kernel's MMA helpers, descriptors,
// P layout and scale-factor staging (with N = 128 keys).  TMEM: S [128,256),
// O [256,384), scale factors of Q [384,392) and of K [392,400).

constexpr uint32_t PR_S = 128, PR_O = 256, PR_SFQ = 384, PR_SFK = 392;
constexpr uint32_t PR_V_PANEL_BYTES = 128 * 64 * 2;

struct ProbeSmem {
    uint8_t v[2 * PR_V_PANEL_BYTES];
    uint8_t pb[8 * P_PANEL_BYTES];
    uint8_t kc[Q_TILE_BYTES];
    uint8_t qc[Q_TILE_BYTES];
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
            mbar_arrive_expect_tx(full, 2 * Q_TILE_BYTES);
            tma_load_3d(smem_u32(sm.qc), &tm_qc, 0, 0, 0, full);
            tma_load_3d(smem_u32(sm.kc), &tm_kc, 0, 0, 0, full);
        } else {
            mbar_arrive_expect_tx(full, 2 * PR_V_PANEL_BYTES);
            tma_load_4d(smem_u32(sm.v), &tm_v, 0, 0, 0, 0, full);
            tma_load_4d(smem_u32(sm.v) + PR_V_PANEL_BYTES, &tm_v, 64, 0, 0, 0, full);
        }
    }
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    if (mode == 1 && warp < 4) {
        // write P into shared memory exactly as the softmax warps do (bf16 pairs)
        const int row = 32 * warp + lane;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(pbf + (size_t)row * 128);
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) pk[i] = src[i];
        store_p_row<8>(sm.pb, row, pk);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        ok = warp_wait(full, 0, abort_flag, status, kWaitLimitNs);
        if (ok) {
            if (lane == 0) {
                tc_fence_after();
                if (mode == 0) {
                    tmem_cp_32x128b_x4(tmem + PR_SFQ, atom_desc(sm.qs_atom[0]));
                    tmem_cp_32x128b_x4(tmem + PR_SFQ + 4, atom_desc(sm.qs_atom[1]));
                    tmem_cp_32x128b_x4(tmem + PR_SFK, atom_desc(sm.ks_atom[0]));
                    tmem_cp_32x128b_x4(tmem + PR_SFK + 4, atom_desc(sm.ks_atom[1]));
                    issue_qk(tmem, PR_S, sm.qc, sm.kc, PR_SFQ, PR_SFK, idesc_qk(128));
                } else {
                    issue_pv<128>(tmem, PR_O, sm.pb, sm.v, PR_V_PANEL_BYTES, false);
                }
            }
        }
        if (lane == 0) tc_commit(smem_u32(&sm.bar_done));
        __syncwarp();
    }
    if (warp < 4) {
        const int row = 32 * warp + lane;
        const uint32_t col = (mode == 0) ? PR_S : PR_O;
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

// V [B][H][N][d bf16] with element strides st (multiples of 8): 128B-swizzled
// boxes of 64 channels x box_rows keys of one head; x is 0 or 64 (0 or 128
// bytes), so every box starts on a 16-byte boundary.
bool make_v_map(CUtensorMap* m, const __nv_bfloat16* base, int B, int H, int N, Strides st, uint32_t box_rows,
                int d = 128) {
    // with d = 64 the box of channels 64-127 lies past the row: it reads zeros
    const uint64_t dims[4] = {(uint64_t)d, (uint64_t)N, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)st.n * 2, (uint64_t)st.h * 2, (uint64_t)st.b * 2};
    const uint32_t box[4] = {64, box_rows, 1, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(base),
                             dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t fwd_smem_bytes() { return sizeof(FwdSmem) + 1024; }
size_t probe_smem_bytes() { return sizeof(ProbeSmem) + 1024; }

}  // namespace

int launch_forward(const FwdArgs& a, cudaStream_t stream) {
    if (a.BH == 0 || a.N == 0) return FP4ATTN_OK;
    Maps m;
    const uint32_t code_bytes = (uint32_t)a.d / 2;
    if (!make_code_map(&m.qc, a.q_codes, a.BH, a.N, BM, code_bytes) ||
        !make_code_map(&m.kc, a.k_codes, a.BH, a.N, BN, code_bytes) ||
        !make_v_map(&m.v, a.v, a.BH / a.H, a.H, a.N, a.vs, BN, a.d))
        return FP4ATTN_ERR_CUDA;
    static_assert(sizeof(FwdSmem) + 1024 <= 227 * 1024, "shared memory budget");
    const size_t smem = fwd_smem_bytes();
    if (cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return FP4ATTN_ERR_CUDA;
    FwdParams p;
    p.q_scales = a.q_scales;
    p.k_scales = a.k_scales;
    p.srb = a.d / 16;
    p.o_chunks = a.d / 32;
    p.N = a.N;
    p.n_kt = (a.N + BN - 1) / BN;
    const float scale = a.softmax_scale > 0.0f ? a.softmax_scale
                                               : (a.d == 64 ? 0.125f : 0.08838834764831845f);  // 1/sqrt(d)
    p.scale_log2 = scale * 1.4426950408889634f;
    p.gq = a.gq;
    p.gk = a.gk;
    p.o = a.o;
    p.o_sb = a.os.b;
    p.o_sh = a.os.h;
    p.o_sn = a.os.n;
    p.H = a.H;
    p.lse = a.lse;
    p.status = a.status;
    p.limit_ns = kWaitLimitNs;
    dim3 grid((a.N + QT * BM - 1) / (QT * BM), a.BH);
    fwd_kernel<<<grid, FWD_THREADS, smem, stream>>>(m.qc, m.kc, m.v, p);
    return cudaGetLastError() == cudaSuccess ? FP4ATTN_OK : FP4ATTN_ERR_CUDA;
}

static int launch_probe(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                        const __nv_bfloat16* p, const __nv_bfloat16* v, float* out, int mode,
                        cudaStream_t stream) {
    Maps m;
    if (mode == 0) {
        if (!make_code_map(&m.qc, qc, 1, 128, 128) || !make_code_map(&m.kc, kc, 1, 128, 128))
            return FP4ATTN_ERR_CUDA;
        m.v = m.qc;  // unused in this mode
    } else {
        if (!make_v_map(&m.v, v, 1, 1, 128, contiguous_strides(1, 128), 128)) return FP4ATTN_ERR_CUDA;
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
