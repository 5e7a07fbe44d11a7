// Training-time backward of the FP4 attention: fake quantisation with a
// straight-through estimator.
//
// FastVideo "Pika H3 Flex in FastVideo": section "NVFP4 QAD" trains the 4-bit
// student with 4-bit math on from the first step, and the summary list says
// the training-time FP4 attention matches the inference kernel.  The forward
// is the inference path itself (quantise, FP4 attention); the backward takes
// the attention gradients at the dequantised Q^ = gQ Q~ and K^ = gK K~, with
// Q~, K~ the unit-scale values (scale x E2M1: exact in bf16) and the global
// scales folded in as scalars, passes them unchanged through the quantiser
// and differentiates the exact transforms:
//   dS = P * (dP - D),  P = exp(scale Q^K^T - lse),  dP = dO V^T,
//   D_i = sum_c dO_ic O_ic,
//   dQ^ = scale dS K^,  dK^ = scale dS^T Q^,  dV = P^T dO,
//   dq = c H dQ^,  dk = c H (dK^ - mean_n dK^)   (c = 1/sqrt(128)).
//
// Four kernels, the first two on the fifth-generation tensor cores (FP4
// scores, BF16 products, fp32 accumulators in TMEM):
//   bwd_q_kernel  one CTA per (head, 128 queries): D of its rows (written for
//                 the next kernel), then per 64-key stage S = Q~K~^T from the
//                 NVFP4 codes with the forward's block-scaled MMA (the same
//                 scores the forward's lse was taken over, at a quarter of a
//                 BF16 product's cost) and dP = dO V^T (M=128, N=64), dS in
//                 registers written as bf16
//                 over the first 32 columns of S, dQ^ += dS K^ with dS read
//                 from TMEM; epilogue dq = c H (scale dQ^) in registers.
//   bwd_kv_kernel one CTA per (head, 128 keys): per 64-query stage
//                 S^T = K~Q~^T from the codes (block-scaled FP4 MMA) and
//                 dP^T = V dO^T, P^T and dS^T as bf16 over S^T (each compute
//                 warp over the 32 columns it loaded), dV += P^T dO and
//                 dK^ += dS^T Q^ with A from TMEM;
//                 epilogue dv (bf16), scale dK^ (fp32 scratch) and each
//                 warp's column sums of it (for the centring).
//   colsum_kernel the head's column sums, added in a fixed order (so the
//                 gradients are the same bits on every run).
//   ste_k_kernel  one warp per key row: dk = c H (dK^ - colsum/N).
// Warps: the dQ kernel has 4 compute warps (one TMEM lane = one row each),
// then the TMA producer and the TMEM owner / MMA issuer; the dK/dV kernel has
// 8 compute warps (two per TMEM lane quarter, each taking half of a stage's
// queries and half of the epilogue's columns), then the same two.  TMEM (512
// columns): stage buffers b at [64b, 64b+64) for S (S^T); dQ kernel: dP_b at
// [128+64b, ...), dQ^ at [256, 384), the scale factors at [384, 408); dK/dV
// kernel: one dP^T at [128, 192), the scale factors at [192, 216), dV at
// [256, 384) and dK^ at [384, 512).  Every wait is bounded; a wait that runs
// out raises FP4ATTN_ERR_TIMEOUT and the CTA winds down.
#include <cuda_bf16.h>

#include "fp4_operands.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr int BR = 128;     // rows of the resident tile (queries or keys)
constexpr int BS = 64;      // rows of a streamed stage (keys or queries)
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr int WARP_PRODUCER = 4;
constexpr int WARP_MMA = 5;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_X = 0, TM_Y = 128, TM_ACC0 = 256, TM_ACC1 = 384;

constexpr uint32_t PANEL_R = BR * 128;  // 128 rows x 64 channels bf16 (128B swizzle)
constexpr uint32_t TILE_R = 2 * PANEL_R;
constexpr uint32_t PANEL_S = BS * 128;  // 64 rows x 64 channels
constexpr uint32_t TILE_S = 2 * PANEL_S;

// kind::f16 with fp32 accumulation (1 << 4) and BF16 A, B (1 << 7, 1 << 10).
//   IDESC_ST: M = 128, N = 64, both operands K-major (S, dP, S^T, dP^T).
//   IDESC_AC: M = 128, N = 128, A from TMEM, B MN-major (1 << 16) (dQ^, dV, dK^).
constexpr uint32_t IDESC_ST = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BS >> 3) << 17) |
                              ((uint32_t)(BR >> 4) << 24);
constexpr uint32_t IDESC_AC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(128 >> 3) << 17) |
                              ((uint32_t)(BR >> 4) << 24);

constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          uint64_t limit) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status, limit);
    return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
    int dummy_abort = 0;
    return mbar_wait(bar, parity, &dummy_abort, nullptr, kDrainLimitNs);
}

// K-major 128B swizzle (channels along K): 128-byte rows of 64 channels, 8-row
// groups 1 KB apart, the second 64 channels one panel further; K step ks (16
// channels = 32 bytes).
__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* tile) {
    return smem_desc(smem_u32(tile), 16, 1024, LAYOUT_SW128);
}
__host__ __device__ constexpr uint64_t kstep(uint32_t panel, int ks) {
    return (uint64_t)((panel * (uint32_t)(ks >> 2) + 32u * (uint32_t)(ks & 3)) >> 4);
}
// MN-major 128B swizzle (channels along N, rows along K): the two 64-channel
// panels `panel` bytes apart, 8-row groups 1 KB apart; K step (16 rows) 2 KB.
__device__ __forceinline__ uint64_t mn_desc(const uint8_t* tile, uint32_t panel) {
    return smem_desc(smem_u32(tile), panel, 1024, LAYOUT_SW128);
}
constexpr uint64_t MN_KSTEP = 2048 >> 4;

// Element offset of row n of head bh in a [B,H,N,128] tensor with strides (sb, sh, sn).
__device__ __forceinline__ long long row_offset(int bh, int H, int n, long long sb, long long sh, long long sn) {
    const int b = bh / H, h = bh - b * H;
    return b * sb + h * sh + (long long)n * sn;
}

// In-register Walsh-Hadamard transform of 128 values (Sylvester order).
__device__ __forceinline__ void fwht128(float* x) {
#pragma unroll
    for (int h = 1; h < 128; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
            if ((i & h) == 0) {
                const float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
        }
    }
}

struct BwdParams {
    int N, H;
    int n_st;          // streamed stages of BS rows
    float scale;       // softmax scale
    float scale_log2;  // softmax scale * log2(e)
    const float* gq;   // global scales of Q and K (device scalars, nullptr = 1)
    const float* gk;
    const float* lse;  // [BH, N], natural log
    float* dsum;       // [BH, N]: D, written by bwd_q_kernel, read by bwd_kv_kernel
    const __nv_bfloat16* o;
    const __nv_bfloat16* dout;
    __nv_bfloat16* dq;  // [B, H, N, 128], element strides io (as o, dout, dv)
    __nv_bfloat16* dv;
    long long io_sb, io_sh, io_sn;
    float* dk_acc;      // [BH, N, 128] fp32: scale * dK^
    float* partial;     // [BH, key tiles * 4, 128] fp32: column sums of scale * dK^ per warp
    const uint64_t* q_scales;  // [BH, N] NVFP4 scale rows (8 UE4M3 bytes each)
    const uint64_t* k_scales;
    bool hadamard;
    int* status;
    uint64_t limit_ns;
};

// ------------------------------------------------------------- dQ kernel --

constexpr uint32_t QC_BYTES = BR * 64;  // 128 rows of 128 E2M1 codes, 64B swizzle
constexpr uint32_t KC_BYTES = BS * 64;  // 64 rows
constexpr uint32_t TM_SFQ = 384, TM_SFK = 392;  // scale factors: Q [384,392), K slots [392,400), [400,408)
constexpr uint32_t IDESC_S4 = idesc_mxf4(BR, BS);

struct __align__(1024) QSmem {
    uint8_t dout[TILE_R];            // dO tile, K-major
    uint8_t k[STAGES][TILE_S];       // K~ stage (bf16), MN-major for dQ^ += dS K^
    uint8_t v[STAGES][TILE_S];       // V stage, K-major for dP
    uint8_t qc[QC_BYTES];            // Q codes
    uint8_t kc[STAGES][KC_BYTES];    // K codes of the stage
    uint8_t qs_atom[2][512];         // scale-factor atoms for tcgen05.cp
    uint8_t ks_atom[STAGES][2][512];
    uint64_t bar_q_full;
    uint64_t bar_kv_full[STAGES];
    uint64_t bar_kv_empty[STAGES];
    uint64_t bar_s_full[2];   // S_b and dP_b of a stage are in TMEM
    uint64_t bar_p_ready[2];  // dS_b (bf16) is in TMEM
    uint64_t bar_final;       // every MMA of the CTA has completed
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(THREADS, 1)
    bwd_q_kernel(const __grid_constant__ CUtensorMap tm_qc, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    QSmem& sm = *reinterpret_cast<QSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int q0 = blockIdx.x * BR;
    const int T = p.n_st;
    const int N = p.N;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.bar_q_full), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm.bar_kv_full[s]), 1);
            mbar_init(smem_u32(&sm.bar_kv_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm.bar_s_full[b]), 1);
            mbar_init(smem_u32(&sm.bar_p_ready[b]), 128);
        }
        mbar_init(smem_u32(&sm.bar_final), 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;
    const uint64_t limit = p.limit_ns;
    const int hb = bh / p.H, hh = bh - hb * p.H;

    if (warp == WARP_PRODUCER) {
        // Q codes (with their scale atoms) and dO once, then per stage the K
        // codes and scale atoms and the bf16 K~ and V of BS keys.  Rows past N
        // are filled with zeros by the copies (scales: zero bytes).
        const uint32_t qf = smem_u32(&sm.bar_q_full);
        load_scale_atoms(p.q_scales + (size_t)bh * N + q0, N - q0, sm.qs_atom[0], sm.qs_atom[1], lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive_expect_tx(qf, QC_BYTES + 2 * PANEL_R);
            tma_load_3d(smem_u32(sm.qc), &tm_qc, 0, q0, bh, qf);
            tma_load_4d(smem_u32(sm.dout), &tm_do, 0, q0, hh, hb, qf);
            tma_load_4d(smem_u32(sm.dout) + PANEL_R, &tm_do, 64, q0, hh, hb, qf);
        }
        // K scale rows are fetched one stage ahead: their load latency overlaps
        // the wait for a free buffer instead of delaying the stage's copies
        const uint64_t* ks_head = p.k_scales + (size_t)bh * N;
        uint64_t ksc[4];
        fetch_scales(ks_head, N < BS ? N : BS, lane, ksc);
        int issued = 0;
        for (int j = 0; j < T; ++j) {
            const int st = j % STAGES;
            if (j >= STAGES &&
                !warp_wait(smem_u32(&sm.bar_kv_empty[st]), ((j / STAGES) - 1) & 1, abort_flag, p.status, limit))
                break;
            const int k0 = j * BS;
            store_scale_atoms(ksc, sm.ks_atom[st][0], sm.ks_atom[st][1], lane);
            if (j + 1 < T) {
                const int rest = N - k0 - BS;
                fetch_scales(ks_head + k0 + BS, rest < BS ? rest : BS, lane, ksc);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const uint32_t full = smem_u32(&sm.bar_kv_full[st]);
                mbar_arrive_expect_tx(full, KC_BYTES + 2 * TILE_S);
                tma_load_3d(smem_u32(sm.kc[st]), &tm_kc, 0, k0, bh, full);
                tma_load_4d(smem_u32(sm.k[st]), &tm_k, 0, k0, hh, hb, full);
                tma_load_4d(smem_u32(sm.k[st]) + PANEL_S, &tm_k, 64, k0, hh, hb, full);
                tma_load_4d(smem_u32(sm.v[st]), &tm_v, 0, k0, hh, hb, full);
                tma_load_4d(smem_u32(sm.v[st]) + PANEL_S, &tm_v, 64, k0, hh, hb, full);
            }
            __syncwarp();
            issued = j + 1;
        }
        if (lane == 0 && *abort_flag) {
            drain_wait(qf, 0);
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                drain_wait(smem_u32(&sm.bar_kv_full[i % STAGES]), (i / STAGES) & 1);
        }
    } else if (warp == WARP_MMA) {
        const bool leader = elect_one_sync();
        const uint64_t qcd = codes_desc(sm.qc, 0);
        const uint64_t kcd0 = codes_desc(sm.kc[0], 0);     // stage st: + st * KC_BYTES / 16
        const uint64_t kad0 = atom_desc(sm.ks_atom[0][0]);  // stage st: + 64 st, half h: + 32 h
        const uint64_t dod = kmajor_desc(sm.dout);
        const uint64_t vd0 = kmajor_desc(sm.v[0]);          // stage st: + st * TILE_S / 16
        const uint64_t kmn0 = mn_desc(sm.k[0], PANEL_S);
        constexpr uint64_t TD = TILE_S >> 4, KCD = KC_BYTES >> 4, AD = (2 * 512) >> 4;
        auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait_spin(bar, parity, abort_flag, p.status, limit));
        };
        // S_b = Q~ K~^T from the codes (K scale factors of stage j into slot
        // j & 1: the stage two back, which used that slot, was issued before),
        // dP_b = dO V^T
        auto scores = [&](int b, int st, int j) {
            const uint32_t sfk = TM_SFK + 8u * (uint32_t)(j & 1);
            tmem_cp_32x128b_x4(tmem + sfk, kad0 + AD * st);
            tmem_cp_32x128b_x4(tmem + sfk + 4, kad0 + AD * st + 32);
            mma_mxf4nvf4(tmem + TM_X + BS * b, qcd, kcd0 + KCD * st, IDESC_S4, tmem + TM_SFQ, tmem + sfk, 0u);
            mma_mxf4nvf4(tmem + TM_X + BS * b, qcd + 2, kcd0 + KCD * st + 2, IDESC_S4, tmem + TM_SFQ + 4,
                         tmem + sfk + 4, 1u);
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks)
                mma_bf16_ss(tmem + TM_Y + BS * b, dod + kstep(PANEL_R, ks), vd0 + TD * st + kstep(PANEL_S, ks),
                            IDESC_ST, ks > 0 ? 1u : 0u);
            tc_commit(smem_u32(&sm.bar_s_full[b]));
        };
        auto accumulate = [&](int b, int st, bool acc) {  // dQ^ += dS_b K^ (dS from TMEM)
#pragma unroll
            for (int ks = 0; ks < BS / 16; ++ks)
                mma_bf16_ts(tmem + TM_ACC0, tmem + TM_X + BS * b + 8u * ks, kmn0 + TD * st + MN_KSTEP * ks,
                            IDESC_AC, (acc || ks > 0) ? 1u : 0u);
            tc_commit(smem_u32(&sm.bar_kv_empty[st]));
        };
        bool ok = wait(smem_u32(&sm.bar_q_full), 0);
        if (ok && leader) {
            tc_fence_after();
            const uint64_t qad = atom_desc(sm.qs_atom[0]);
            tmem_cp_32x128b_x4(tmem + TM_SFQ, qad);
            tmem_cp_32x128b_x4(tmem + TM_SFQ + 4, qad + 32);
        }
        __syncwarp();
        for (int j = 0; ok && j < T; ++j) {
            const int st = j % STAGES;
            if (!wait(smem_u32(&sm.bar_kv_full[st]), (j / STAGES) & 1)) {
                ok = false;
                break;
            }
            if (leader) {
                tc_fence_after();
                scores(j & 1, st, j);
            }
            __syncwarp();
            if (j > 0) {
                if (!wait(smem_u32(&sm.bar_p_ready[(j - 1) & 1]), ((j - 1) >> 1) & 1)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    tc_fence_after();
                    accumulate((j - 1) & 1, (j - 1) % STAGES, j > 1);
                }
                __syncwarp();
            }
        }
        if (ok && T > 0 && wait(smem_u32(&sm.bar_p_ready[(T - 1) & 1]), ((T - 1) >> 1) & 1)) {
            if (leader) {
                tc_fence_after();
                accumulate((T - 1) & 1, (T - 1) % STAGES, T > 1);
            }
            __syncwarp();
        }
        // the final commit tells the compute warps that dQ^ is complete, and
        // is what this warp waits on before TMEM is freed
        if (leader) {
            tc_commit(smem_u32(&sm.bar_final));
            drain_wait(smem_u32(&sm.bar_final), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ compute warps --
        const int row = 32 * warp + lane;
        const int n = q0 + row;
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        const size_t grow = (size_t)bh * N + n;
        // D = sum_c dO_c O_c of this row, and the row's lse in the log2 domain;
        // rows past N get p = 0 (lse = +inf) and D = 0
        float Dr = 0.0f, lse2 = INFINITY;
        if (n < N) {
            const long long io = row_offset(bh, p.H, n, p.io_sb, p.io_sh, p.io_sn);
            const uint4* po = reinterpret_cast<const uint4*>(p.o + io);
            const uint4* pd = reinterpret_cast<const uint4*>(p.dout + io);
            float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                const uint4 a = po[c], g = pd[c];
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc = __ffma2_rn(make_float2(bf16lo(aw[e]), bf16hi(aw[e])),
                                     make_float2(bf16lo(gw[e]), bf16hi(gw[e])), acc);
            }
            Dr = acc.x + acc.y;
            p.dsum[grow] = Dr;
            lse2 = p.lse[grow] * kLog2e;
        }
        const float gq = p.gq ? *p.gq : 1.0f, gk = p.gk ? *p.gk : 1.0f;
        if (threadIdx.x == 0 && blockIdx.x == 0 && !(gq > 0.0f && gq < INFINITY && gk > 0.0f && gk < INFINITY))
            atomicCAS(p.status, 0, (int)FP4ATTN_ERR_RANGE);
        const float c = p.scale_log2 * gq * gk;  // S = scale gQ gK Q~ K~^T
        const float dq_scale = p.scale * gk;     // dQ^ = scale dS K^ = scale gK dS K~
        bool ok = true;
        for (int j = 0; j < T; ++j) {
            const int b = j & 1;
            if (!warp_wait(smem_u32(&sm.bar_s_full[b]), (j >> 1) & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[BS], dr[BS];
            tmem_ld32(tmem + lane_base + TM_X + BS * b, &sr[0]);
            tmem_ld32(tmem + lane_base + TM_X + BS * b + 32, &sr[32]);
            tmem_ld32(tmem + lane_base + TM_Y + BS * b, &dr[0]);
            tmem_ld32(tmem + lane_base + TM_Y + BS * b + 32, &dr[32]);
            tmem_wait_ld();
            const int nvalid = N - j * BS;  // keys of this stage that exist
            const float2 c2 = make_float2(c, c), nl2 = make_float2(-lse2, -lse2), nd2 = make_float2(-Dr, -Dr);
            uint32_t pk[BS / 2];
#pragma unroll
            for (int k = 0; k < BS / 2; ++k) {
                // exponentials: 3 of every 8 pairs on the FMA-pipe polynomial, the
                // rest on MUFU (as in the forward), packed fp32x2 arithmetic
                const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])),
                                            c2, nl2);
                const float2 pr = ((k & 7) < 3) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                float2 ds = __fmul2_rn(pr, __fadd2_rn(make_float2(__uint_as_float(dr[2 * k]),
                                                                  __uint_as_float(dr[2 * k + 1])), nd2));
                if (2 * k >= nvalid) ds.x = 0.0f;
                if (2 * k + 1 >= nvalid) ds.y = 0.0f;
                pk[k] = pack_bf16x2(ds.x, ds.y);
            }
            tmem_st32(tmem + lane_base + TM_X + BS * b, pk);  // dS over the first 32 columns of S_b
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.bar_p_ready[b]));
        }
        if (ok && T > 0 && warp_wait(smem_u32(&sm.bar_final), 0, abort_flag, p.status, limit)) {
            tc_fence_after();
            float x[128];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + TM_ACC0 + 32u * q, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) x[32 * q + e] = __uint_as_float(r[e]) * dq_scale;
            }
            if (p.hadamard) {
                fwht128(x);
                const float h = __uint_as_float(0x3DB504F3u);  // fp32(1/sqrt(128))
#pragma unroll
                for (int e = 0; e < 128; ++e) x[e] *= h;
            }
            if (n < N) {
                uint4* dst = reinterpret_cast<uint4*>(p.dq + row_offset(bh, p.H, n, p.io_sb, p.io_sh, p.io_sn));
#pragma unroll
                for (int v = 0; v < 16; ++v)
                    dst[v] = make_uint4(pack_bf16x2(x[8 * v], x[8 * v + 1]), pack_bf16x2(x[8 * v + 2], x[8 * v + 3]),
                                        pack_bf16x2(x[8 * v + 4], x[8 * v + 5]),
                                        pack_bf16x2(x[8 * v + 6], x[8 * v + 7]));
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

// ------------------------------------------------------- dK, dV kernel --

// TMEM of the dK/dV kernel: S^T_b [64b, 64b+64) with P^T and dS^T written as
// bf16 over it (each compute warp over the 32 columns it loaded), dP^T
// [128, 192) (one buffer: free once the compute warps have loaded it), scale
// factors of K [192, 200) and two slots of Q's [200, 208), [208, 216); dV
// [256, 384), dK^ [384, 512).
constexpr uint32_t KV_DP = 128, KV_SFK = 192, KV_SFQ = 200;

struct __align__(1024) KVSmem {
    uint8_t v[TILE_R];                // V tile, K-major (A of dP^T)
    uint8_t q[STAGES][TILE_S];        // Q~ stage (bf16): MN-major for dK^ += dS^T Q~
    uint8_t dout[STAGES][TILE_S];     // dO stage: K-major for dP^T, MN-major for dV += P^T dO
    uint8_t kc[QC_BYTES];             // K codes (128 rows): A of S^T
    uint8_t qc[STAGES][KC_BYTES];     // Q codes of the stage (64 rows): B of S^T
    uint8_t ks_atom[2][512];          // scale-factor atoms for tcgen05.cp
    uint8_t qs_atom[STAGES][2][512];
    float lse2[STAGES][BS];           // lse * log2(e) of the stage's queries (+inf past N)
    float dsum[STAGES][BS];           // D of the stage's queries (0 past N)
    uint64_t bar_kv_full;
    uint64_t bar_q_full[STAGES];
    uint64_t bar_q_empty[STAGES];
    uint64_t bar_s_full[2];
    uint64_t bar_dp_free;             // the compute warps have loaded dP^T
    uint64_t bar_p_ready[2];
    uint64_t bar_final;
    uint32_t tmem_base;
    int abort_flag;
};

// Sum of each of NV columns over the 32 lanes of a warp: after five rounds of
// exchanging half of the remaining partial sums, lane l holds the sums of
// columns (NV/32)l .. (NV/32)l + NV/32 - 1 in a[0 .. NV/32 - 1].
template <int NV, int R>
__device__ __forceinline__ void column_sum_round(float* a, int lane) {
    constexpr int half = (NV / 2) >> R;  // partial sums exchanged this round
    const bool upper = (lane >> (4 - R)) & 1;
#pragma unroll
    for (int i = 0; i < half; ++i) {
        const float send = upper ? a[i] : a[i + half];
        const float keep = upper ? a[i + half] : a[i];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16 >> R);
    }
}
template <int NV>
__device__ __forceinline__ void warp_column_sums(float* a, int lane) {
    column_sum_round<NV, 0>(a, lane);
    column_sum_round<NV, 1>(a, lane);
    column_sum_round<NV, 2>(a, lane);
    column_sum_round<NV, 3>(a, lane);
    column_sum_round<NV, 4>(a, lane);
}

// The dK/dV kernel's warps: 0-7 compute, 8 the TMA producer, 9 the MMA issuer.
constexpr int KV_COMPUTE_WARPS = 8;
constexpr int KV_THREADS = 32 * (KV_COMPUTE_WARPS + 2);
constexpr int KV_WARP_PRODUCER = KV_COMPUTE_WARPS;
constexpr int KV_WARP_MMA = KV_COMPUTE_WARPS + 1;
// TMEM column (within S^T_b) of the bf16 P^T for K step ks (16 queries): the
// compute warp of queries 32h .. writes P^T of them to columns 32h .. 32h+15
// and dS^T to 32h+16 .. 32h+31.
__host__ __device__ constexpr uint32_t kv_pcol(int ks) { return 32u * (uint32_t)(ks >> 1) + 8u * (uint32_t)(ks & 1); }

__global__ void __launch_bounds__(KV_THREADS, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_qc, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    KVSmem& sm = *reinterpret_cast<KVSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int k0 = blockIdx.x * BR;
    const int T = p.n_st;
    const int N = p.N;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&sm.bar_kv_full), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm.bar_q_full[s]), 32);  // every producer lane (its lse / D / atom stores)
            mbar_init(smem_u32(&sm.bar_q_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm.bar_s_full[b]), 1);
            mbar_init(smem_u32(&sm.bar_p_ready[b]), 32 * KV_COMPUTE_WARPS);
        }
        mbar_init(smem_u32(&sm.bar_dp_free), 32 * KV_COMPUTE_WARPS);
        mbar_init(smem_u32(&sm.bar_final), 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == KV_WARP_MMA) {
        tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int* abort_flag = &sm.abort_flag;
    const uint64_t limit = p.limit_ns;
    const int hb = bh / p.H, hh = bh - hb * p.H;

    if (warp == KV_WARP_PRODUCER) {
        // K codes (with their scale atoms) and V once; per stage the Q codes and
        // scale atoms, the bf16 Q~ and dO of BS queries, and their lse and D,
        // all but the copies fetched one stage ahead
        const uint32_t kvf = smem_u32(&sm.bar_kv_full);
        load_scale_atoms(p.k_scales + (size_t)bh * N + k0, N - k0, sm.ks_atom[0], sm.ks_atom[1], lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive_expect_tx(kvf, QC_BYTES + TILE_R);
            tma_load_3d(smem_u32(sm.kc), &tm_kc, 0, k0, bh, kvf);
            tma_load_4d(smem_u32(sm.v), &tm_v, 0, k0, hh, hb, kvf);
            tma_load_4d(smem_u32(sm.v) + PANEL_R, &tm_v, 64, k0, hh, hb, kvf);
        }
        const float* lse_head = p.lse + (size_t)bh * N;
        const float* d_head = p.dsum + (size_t)bh * N;
        const uint64_t* qs_head = p.q_scales + (size_t)bh * N;
        float nl[BS / 32], nd[BS / 32];
        uint64_t qsc[4];
        auto fetch = [&](int i) {
#pragma unroll
            for (int e = 0; e < BS / 32; ++e) {
                const int qi = i * BS + lane + 32 * e;
                nl[e] = (qi < N) ? lse_head[qi] * kLog2e : INFINITY;
                nd[e] = (qi < N) ? d_head[qi] : 0.0f;
            }
            const int rest = N - i * BS;
            fetch_scales(qs_head + i * BS, rest < BS ? rest : BS, lane, qsc);
        };
        fetch(0);
        int issued = 0;
        for (int i = 0; i < T; ++i) {
            const int st = i % STAGES;
            if (i >= STAGES &&
                !warp_wait(smem_u32(&sm.bar_q_empty[st]), ((i / STAGES) - 1) & 1, abort_flag, p.status, limit))
                break;
#pragma unroll
            for (int e = 0; e < BS / 32; ++e) {
                sm.lse2[st][lane + 32 * e] = nl[e];
                sm.dsum[st][lane + 32 * e] = nd[e];
            }
            store_scale_atoms(qsc, sm.qs_atom[st][0], sm.qs_atom[st][1], lane);
            if (i + 1 < T) fetch(i + 1);
            fence_proxy_async_smem();
            const uint32_t full = smem_u32(&sm.bar_q_full[st]);
            if (lane == 0) {
                const int r0 = i * BS;
                mbar_arrive_expect_tx(full, KC_BYTES + 2 * TILE_S);
                tma_load_3d(smem_u32(sm.qc[st]), &tm_qc, 0, r0, bh, full);
                tma_load_4d(smem_u32(sm.q[st]), &tm_q, 0, r0, hh, hb, full);
                tma_load_4d(smem_u32(sm.q[st]) + PANEL_S, &tm_q, 64, r0, hh, hb, full);
                tma_load_4d(smem_u32(sm.dout[st]), &tm_do, 0, r0, hh, hb, full);
                tma_load_4d(smem_u32(sm.dout[st]) + PANEL_S, &tm_do, 64, r0, hh, hb, full);
            } else {
                mbar_arrive(full);
            }
            __syncwarp();
            issued = i + 1;
        }
        if (lane == 0 && *abort_flag) {
            drain_wait(kvf, 0);
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                drain_wait(smem_u32(&sm.bar_q_full[i % STAGES]), (i / STAGES) & 1);
        }
    } else if (warp == KV_WARP_MMA) {
        const bool leader = elect_one_sync();
        const uint64_t kcd = codes_desc(sm.kc, 0);
        const uint64_t qcd0 = codes_desc(sm.qc[0], 0);      // stage st: + st * KC_BYTES / 16
        const uint64_t qad0 = atom_desc(sm.qs_atom[0][0]);  // stage st: + 64 st, half h: + 32 h
        const uint64_t vd = kmajor_desc(sm.v);
        const uint64_t dod0 = kmajor_desc(sm.dout[0]);      // stage st: + st * TILE_S / 16
        const uint64_t qmn0 = mn_desc(sm.q[0], PANEL_S);
        const uint64_t domn0 = mn_desc(sm.dout[0], PANEL_S);
        constexpr uint64_t TD = TILE_S >> 4, KCD = KC_BYTES >> 4, AD = (2 * 512) >> 4;
        auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait_spin(bar, parity, abort_flag, p.status, limit));
        };
        // S^T_b = K~ Q~^T from the codes (Q scale factors of stage i into slot
        // i & 1: the stage two back, which used that slot, was issued before)
        auto scores = [&](int b, int st, int i) {
            const uint32_t sfq = KV_SFQ + 8u * (uint32_t)(i & 1);
            tmem_cp_32x128b_x4(tmem + sfq, qad0 + AD * st);
            tmem_cp_32x128b_x4(tmem + sfq + 4, qad0 + AD * st + 32);
            mma_mxf4nvf4(tmem + TM_X + BS * b, kcd, qcd0 + KCD * st, IDESC_S4, tmem + KV_SFK, tmem + sfq, 0u);
            mma_mxf4nvf4(tmem + TM_X + BS * b, kcd + 2, qcd0 + KCD * st + 2, IDESC_S4, tmem + KV_SFK + 4,
                         tmem + sfq + 4, 1u);
        };
        auto dprod = [&](int b, int st) {  // dP^T = V dO^T, then announce S^T_b and dP^T
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks)
                mma_bf16_ss(tmem + KV_DP, vd + kstep(PANEL_R, ks), dod0 + TD * st + kstep(PANEL_S, ks), IDESC_ST,
                            ks > 0 ? 1u : 0u);
            tc_commit(smem_u32(&sm.bar_s_full[b]));
        };
        auto accumulate = [&](int b, int st, bool acc) {  // dV += P^T dO, dK^ += dS^T Q~ (A from TMEM)
#pragma unroll
            for (int ks = 0; ks < BS / 16; ++ks)
                mma_bf16_ts(tmem + TM_ACC0, tmem + TM_X + BS * b + kv_pcol(ks), domn0 + TD * st + MN_KSTEP * ks,
                            IDESC_AC, (acc || ks > 0) ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < BS / 16; ++ks)
                mma_bf16_ts(tmem + TM_ACC1, tmem + TM_X + BS * b + kv_pcol(ks) + 16u, qmn0 + TD * st + MN_KSTEP * ks,
                            IDESC_AC, (acc || ks > 0) ? 1u : 0u);
            tc_commit(smem_u32(&sm.bar_q_empty[st]));
        };
        bool ok = wait(smem_u32(&sm.bar_kv_full), 0);
        if (ok && leader) {
            tc_fence_after();
            const uint64_t kad = atom_desc(sm.ks_atom[0]);
            tmem_cp_32x128b_x4(tmem + KV_SFK, kad);
            tmem_cp_32x128b_x4(tmem + KV_SFK + 4, kad + 32);
        }
        __syncwarp();
        for (int i = 0; ok && i < T; ++i) {
            const int st = i % STAGES;
            if (!wait(smem_u32(&sm.bar_q_full[st]), (i / STAGES) & 1)) {
                ok = false;
                break;
            }
            if (leader) {
                tc_fence_after();
                scores(i & 1, st, i);
            }
            __syncwarp();
            // the single dP^T buffer: the compute warps must have loaded stage i-1's
            if (i > 0 && !wait(smem_u32(&sm.bar_dp_free), (i - 1) & 1)) {
                ok = false;
                break;
            }
            if (leader) {
                tc_fence_after();
                dprod(i & 1, st);
            }
            __syncwarp();
            if (i > 0) {
                if (!wait(smem_u32(&sm.bar_p_ready[(i - 1) & 1]), ((i - 1) >> 1) & 1)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    tc_fence_after();
                    accumulate((i - 1) & 1, (i - 1) % STAGES, i > 1);
                }
                __syncwarp();
            }
        }
        if (ok && T > 0 && wait(smem_u32(&sm.bar_p_ready[(T - 1) & 1]), ((T - 1) >> 1) & 1)) {
            if (leader) {
                tc_fence_after();
                accumulate((T - 1) & 1, (T - 1) % STAGES, T > 1);
            }
            __syncwarp();
        }
        if (leader) {
            tc_commit(smem_u32(&sm.bar_final));
            drain_wait(smem_u32(&sm.bar_final), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ compute warps --
        // warps w and w+4 share TMEM lanes 32(w&3).. (key rows); warp half hc
        // takes queries 32hc .. 32hc+31 of each stage and columns 64hc ..
        // 64hc+63 of the epilogue
        const int quarter = warp & 3, hc = warp >> 2;
        const int row = 32 * quarter + lane;  // key row of the tile
        const int kn = k0 + row;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float gq = p.gq ? *p.gq : 1.0f, gk = p.gk ? *p.gk : 1.0f;
        const float c = p.scale_log2 * gq * gk;  // S^T = scale gQ gK K~ Q~^T
        const float dk_scale = p.scale * gq;     // dK^ = scale dS^T Q^ = scale gQ dS^T Q~
        bool ok = true;
        for (int i = 0; i < T; ++i) {
            const int b = i & 1;
            const int st = i % STAGES;
            // the stage's lse / D (written by the producer lanes) and S^T, dP^T
            if (!warp_wait(smem_u32(&sm.bar_q_full[st]), (i / STAGES) & 1, abort_flag, p.status, limit) ||
                !warp_wait(smem_u32(&sm.bar_s_full[b]), (i >> 1) & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t own = TM_X + BS * b + 32u * hc;  // this warp's 32 columns of S^T_b
            uint32_t sr[32], dr[32];
            tmem_ld32(tmem + lane_base + own, sr);
            tmem_ld32(tmem + lane_base + KV_DP + 32u * hc, dr);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.bar_dp_free));  // dP^T may be overwritten
            const float4* l4 = reinterpret_cast<const float4*>(sm.lse2[st] + 32 * hc);
            const float4* d4 = reinterpret_cast<const float4*>(sm.dsum[st] + 32 * hc);
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float4 lv = l4[g], dv = d4[g];
                const float la[4] = {lv.x, lv.y, lv.z, lv.w}, da[4] = {dv.x, dv.y, dv.z, dv.w};
                float pr[4], ds[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kk = 4 * g + e;
                    pr[e] = ex2_approx(fmaf(__uint_as_float(sr[kk]), c, -la[e]));
                    ds[e] = pr[e] * (__uint_as_float(dr[kk]) - da[e]);
                }
                pk[2 * g] = pack_bf16x2(pr[0], pr[1]);
                pk[2 * g + 1] = pack_bf16x2(pr[2], pr[3]);
                dk[2 * g] = pack_bf16x2(ds[0], ds[1]);
                dk[2 * g + 1] = pack_bf16x2(ds[2], ds[3]);
            }
            // P^T and dS^T of these queries over the warp's own S^T columns
            tmem_st16(tmem + lane_base + own, pk);
            tmem_st16(tmem + lane_base + own + 16, dk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.bar_p_ready[b]));
        }
        if (ok && T > 0 && warp_wait(smem_u32(&sm.bar_final), 0, abort_flag, p.status, limit)) {
            tc_fence_after();
            const size_t grow = (size_t)bh * N + kn;
            const bool valid = kn < N;
            // dV (bf16), columns 64hc ..
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t r[32];
                const uint32_t col = 64u * hc + 32u * q;
                tmem_ld32(tmem + lane_base + TM_ACC0 + col, r);
                tmem_wait_ld();
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(p.dv + row_offset(bh, p.H, kn, p.io_sb, p.io_sh, p.io_sn) +
                                                          col);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(
                            pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                            pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                            pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                            pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
                }
            }
            // scale * dK^ (fp32) of columns 64hc .. and their sums over the valid keys
            float x[64];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + TM_ACC1 + 64u * hc + 32u * q, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) x[32 * q + e] = valid ? __uint_as_float(r[e]) * dk_scale : 0.0f;
            }
            if (valid) {
                float4* dst = reinterpret_cast<float4*>(p.dk_acc + grow * 128 + 64 * hc);
#pragma unroll
                for (int v = 0; v < 16; ++v) dst[v] = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
            }
            warp_column_sums<64>(x, lane);
            float2* part = reinterpret_cast<float2*>(
                p.partial + (((size_t)bh * gridDim.x + blockIdx.x) * 4 + quarter) * 128 + 64 * hc);
            part[lane] = make_float2(x[0], x[1]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == KV_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------- key straight-through --

// Column sums of scale * dK^ of each head: thread c of block bh adds the
// per-warp partial sums of column c in order.
__global__ void __launch_bounds__(128) colsum_kernel(const float* __restrict__ partial, int parts,
                                                     float* __restrict__ colsum) {
    const float* src = partial + (size_t)blockIdx.x * parts * 128 + threadIdx.x;
    float acc = 0.0f;
    for (int i = 0; i < parts; ++i) acc += src[(size_t)i * 128];
    colsum[(size_t)blockIdx.x * 128 + threadIdx.x] = acc;
}

// One warp per key row: dk = c H (scale dK^ - colsum / N) as bf16.  Lane l
// holds channels 4l .. 4l+3; butterfly strides 1 and 2 stay in the lane,
// strides 4 .. 64 pair lanes l and l ^ (stride / 4).
__global__ void __launch_bounds__(256) ste_k_kernel(const float* __restrict__ dk_acc, const float* __restrict__ colsum,
                                                    int N, int H, int64_t rows, bool smooth, bool hadamard,
                                                    __nv_bfloat16* __restrict__ dk, long long sb, long long sh,
                                                    long long sn) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const float nf = (float)N;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nw) {
        const float4 v = reinterpret_cast<const float4*>(dk_acc + r * 128)[lane];
        float x[4] = {v.x, v.y, v.z, v.w};
        if (smooth) {
            const float4 m = reinterpret_cast<const float4*>(colsum + (r / N) * 128)[lane];
            x[0] -= __fdiv_rn(m.x, nf);
            x[1] -= __fdiv_rn(m.y, nf);
            x[2] -= __fdiv_rn(m.z, nf);
            x[3] -= __fdiv_rn(m.w, nf);
        }
        if (hadamard) {
            float a = x[0] + x[1], b = x[0] - x[1], cc = x[2] + x[3], d = x[2] - x[3];
            x[0] = a + cc;
            x[2] = a - cc;
            x[1] = b + d;
            x[3] = b - d;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const bool upper = lane & m;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
                    x[e] = upper ? (o - x[e]) : (x[e] + o);
                }
            }
            const float h = __uint_as_float(0x3DB504F3u);
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] *= h;
        }
        const int bh = (int)(r / N), n = (int)(r - (int64_t)bh * N);
        reinterpret_cast<uint2*>(dk + row_offset(bh, H, n, sb, sh, sn))[lane] =
            make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    }
}

// [B][H][N][128 bf16] with element strides st (multiples of 8): 128B-swizzled
// boxes of 64 channels x box_rows rows of one head (x is 0 or 64: 16-byte
// aligned).
bool make_map(CUtensorMap* m, const __nv_bfloat16* base, int B, int H, int N, uint32_t box_rows, Strides st) {
    const uint64_t dims[4] = {128, (uint64_t)N, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)st.n * 2, (uint64_t)st.h * 2, (uint64_t)st.b * 2};
    const uint32_t box[4] = {64, box_rows, 1, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(base), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

int launch_backward(const BwdArgs& a, cudaStream_t stream) {
    if (a.BH == 0 || a.N == 0) return FP4ATTN_OK;
    const int B = a.BH / a.H;
    // unit-scale Q~, K~ in bf16 (exact) for the dK / dV kernel and the dQ^ product
    const int64_t rows = (int64_t)a.BH * a.N;
    if (launch_dequant_bf16(a.q_codes, a.q_scales, nullptr, rows * 8, a.qhat, stream) != cudaSuccess ||
        launch_dequant_bf16(a.k_codes, a.k_scales, nullptr, rows * 8, a.khat, stream) != cudaSuccess)
        return FP4ATTN_ERR_CUDA;
    CUtensorMap qc_r, kc_s, kc_r, qc_s, do_r, k_s, v_s, v_r, q_s, do_s;
    const Strides cs = contiguous_strides(a.H, a.N);  // Q~, K~: the library's own contiguous tensors
    if (!make_code_map(&qc_r, a.q_codes, a.BH, a.N, BR) || !make_code_map(&kc_s, a.k_codes, a.BH, a.N, BS) ||
        !make_code_map(&kc_r, a.k_codes, a.BH, a.N, BR) || !make_code_map(&qc_s, a.q_codes, a.BH, a.N, BS) ||
        !make_map(&do_r, a.dout, B, a.H, a.N, BR, a.io) ||
        !make_map(&k_s, a.khat, B, a.H, a.N, BS, cs) || !make_map(&v_s, a.v, B, a.H, a.N, BS, a.io) ||
        !make_map(&v_r, a.v, B, a.H, a.N, BR, a.io) ||
        !make_map(&q_s, a.qhat, B, a.H, a.N, BS, cs) || !make_map(&do_s, a.dout, B, a.H, a.N, BS, a.io))
        return FP4ATTN_ERR_CUDA;
    static_assert(sizeof(QSmem) + 1024 <= 227 * 1024, "shared memory budget");
    static_assert(sizeof(KVSmem) + 1024 <= 227 * 1024, "shared memory budget");
    const size_t smem_q = sizeof(QSmem) + 1024, smem_kv = sizeof(KVSmem) + 1024;
    if (cudaFuncSetAttribute(bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv) !=
            cudaSuccess)
        return FP4ATTN_ERR_CUDA;
    BwdParams p;
    p.N = a.N;
    p.H = a.H;
    p.n_st = (a.N + BS - 1) / BS;
    p.scale = a.softmax_scale > 0.0f ? a.softmax_scale : 0.08838834764831845f;
    p.scale_log2 = p.scale * kLog2e;
    p.gq = a.gq;
    p.gk = a.gk;
    p.q_scales = reinterpret_cast<const uint64_t*>(a.q_scales);
    p.k_scales = reinterpret_cast<const uint64_t*>(a.k_scales);
    p.lse = a.lse;
    p.dsum = a.dsum;
    p.o = a.o;
    p.dout = a.dout;
    p.dq = a.dq;
    p.dv = a.dv;
    p.io_sb = a.io.b;
    p.io_sh = a.io.h;
    p.io_sn = a.io.n;
    p.dk_acc = a.dk_acc;
    p.partial = a.partial;
    p.hadamard = !(a.flags & FP4ATTN_NO_HADAMARD);
    p.status = a.status;
    p.limit_ns = kWaitLimitNs;
    const dim3 grid((a.N + BR - 1) / BR, a.BH);
    bwd_q_kernel<<<grid, THREADS, smem_q, stream>>>(qc_r, do_r, kc_s, k_s, v_s, p);
    if (cudaGetLastError() != cudaSuccess) return FP4ATTN_ERR_CUDA;
    bwd_kv_kernel<<<grid, KV_THREADS, smem_kv, stream>>>(kc_r, v_r, qc_s, q_s, do_s, p);
    if (cudaGetLastError() != cudaSuccess) return FP4ATTN_ERR_CUDA;
    if (!(a.flags & FP4ATTN_NO_SMOOTH_K)) {
        colsum_kernel<<<a.BH, 128, 0, stream>>>(a.partial, 4 * (int)grid.x, a.colsum);
        if (cudaGetLastError() != cudaSuccess) return FP4ATTN_ERR_CUDA;
    }
    const int64_t want = (rows + 7) / 8;  // 8 warps per block, one row each
    const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
    ste_k_kernel<<<blocks, 256, 0, stream>>>(a.dk_acc, a.colsum, a.N, a.H, rows, !(a.flags & FP4ATTN_NO_SMOOTH_K),
                                             p.hadamard, a.dk, a.io.b, a.io.h, a.io.n);
    return cudaGetLastError() == cudaSuccess ? FP4ATTN_OK : FP4ATTN_ERR_CUDA;
}

}  // namespace fp4attn
