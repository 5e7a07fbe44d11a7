// Non-causal attention with BF16 Q and K: O = softmax(scale * Q K^T) V, the
// BF16 counterpart of the FP4 kernel in attention.cu.
//
// FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention", keeps two of
// the model's attention blocks in BF16 and measures the FP4 kernel against the
// BF16 one; this kernel is that BF16 path.  It is written for sm_100a:
//   * one CTA per (head, 256 queries) = two 128-row query tiles that share
//     every 128-key K/V stage; 384 threads: warps 0-3 and 4-7 the softmax
//     warps of query tile 0 and 1 (one query row per thread = TMEM lane),
//     warp 8 the TMA producer (both Q tiles once, then K and V of 128 keys
//     per stage into a STAGES-deep ring), warp 9 the TMEM owner and MMA
//     issuer, warps 10-11 only complete the third warpgroup for the register
//     split (softmax warpgroups 224 registers, the rest 56);
//   * TMEM (512 columns): S_0 [0,128), S_1 [128,256) fp32, O_0 [256,384),
//     O_1 [384,512); P_i is written as bf16 pairs over the first 64 columns of
//     S_i and read from there by O_i += P_i V (A operand in TMEM);
//   * S_i = Q_i K^T: eight tcgen05.mma kind::f16 (M=128, N=128, K=16) from
//     128B-swizzled K-major Q and K tiles; O_i += P_i V: eight kind::f16 MMAs
//     with V 128B-swizzled MN-major;
//   * tensor-pipe order per stage j: S_0(j), O_1 += P_1(j-1) V, S_1(j),
//     O_0 += P_0(j) V.  tcgen05 operations of one thread run in issue order,
//     so S_i(j) may overwrite P_i(j-1) right after the MMA that reads it, and
//     the commit that announces S_i(j) also covers O_i += P_i(j-1) V: O_i is
//     complete whenever its softmax warps see S_i, so a rescale needs no extra
//     wait;
//   * online softmax in the log2 domain with a lazy running max (it moves only
//     when a stage's max exceeds it by more than 8, so p <= 256), exponentials
//     split between MUFU ex2 and an FMA-pipe polynomial, packed fp32x2; the
//     row sum is taken over the same bf16-rounded P that enters P V.
// Every wait is bounded; a wait that runs out raises FP4ATTN_ERR_TIMEOUT in the
// status word and the CTA winds down instead of hanging.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int QT = 2;    // query tiles per CTA
constexpr int BN = 128;  // keys per K/V stage
constexpr int STAGES = 2;
constexpr int SOFTMAX_WARPS = 4 * QT;
constexpr int THREADS = 32 * (SOFTMAX_WARPS + 4);
constexpr int WARP_PRODUCER = SOFTMAX_WARPS;
constexpr int WARP_MMA = SOFTMAX_WARPS + 1;
constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 224, SUPPORT_REGS = 56;
static_assert(2 * 128 * SOFTMAX_REGS + 128 * SUPPORT_REGS <= THREADS * LAUNCH_REGS, "register split");
static_assert((2 * SOFTMAX_REGS + SUPPORT_REGS) * 32 <= 16384, "registers of one SM sub-partition");
#ifndef FP4ATTN_POLY_PAIRS
#define FP4ATTN_POLY_PAIRS 3
#endif
constexpr int POLY_PAIRS_PER_8 = FP4ATTN_POLY_PAIRS;  // of every 8 exponential pairs, on the FMA pipe

constexpr uint32_t TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t tm_s(int i) { return (uint32_t)(BN * i); }
__host__ __device__ constexpr uint32_t tm_o(int i) { return (uint32_t)(2 * BN + 128 * i); }
static_assert(tm_o(1) + 128 == TMEM_COLS, "TMEM budget");

constexpr uint32_t PANEL_BYTES = 128 * 128;        // 128 rows x 64 channels bf16, 128B swizzle
constexpr uint32_t TILE_BYTES = 2 * PANEL_BYTES;   // 128 rows x 128 channels

// kind::f16, fp32 accumulate (1 << 4), A = B = BF16 (1 << 7, 1 << 10), M = 128, N = 128.
//  S: A = Q K-major, B = K K-major.  O: A = P (TMEM, K-major), B = V MN-major (1 << 16).
constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(128 >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);

struct __align__(1024) Smem {
    uint8_t q[QT][TILE_BYTES];      // K-major, 128B swizzle: channels 0-63, then 64-127
    uint8_t k[STAGES][TILE_BYTES];  // same layout
    uint8_t v[STAGES][TILE_BYTES];  // same bytes, read as MN-major by O += P V
    uint64_t bar_q_full;
    uint64_t bar_kv_full[STAGES];
    uint64_t bar_kv_empty[STAGES];
    uint64_t bar_s_full[QT];   // S_i of the current stage is in TMEM (and O_i is up to date)
    uint64_t bar_p_ready[QT];  // P_i of the current stage is in TMEM
    uint64_t bar_o_final[QT];  // O_i includes the last stage
    uint64_t bar_final;        // every MMA of the CTA has completed
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    int N;
    int n_kt;
    float scale_log2;  // softmax_scale * log2(e)
    __nv_bfloat16* o;
    long long o_sb, o_sh, o_sn;  // element strides of O ([B,H,N,128], channels contiguous)
    int H;
    float* lse;
    int* status;
    uint64_t limit_ns;
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s for the wind-down waits

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          uint64_t limit) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status, limit);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
    int dummy_abort = 0;
    return mbar_wait(bar, parity, &dummy_abort, nullptr, kDrainLimitNs);
}

// K-major 128B swizzle: 128-byte rows (64 channels), 8-row groups 1 KB apart;
// K step ks (16 channels = 32 bytes) is 32 bytes into the row of panel ks / 4.
__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* tile) {
    return smem_desc(smem_u32(tile), 16, 1024, LAYOUT_SW128);
}
__host__ __device__ constexpr uint64_t kmajor_step(int ks) {
    return (uint64_t)((PANEL_BYTES * (uint32_t)(ks >> 2) + 32u * (uint32_t)(ks & 3)) >> 4);
}
// MN-major 128B swizzle (V as the B operand of O += P V): the two 64-channel
// panels PANEL_BYTES apart, 8-key groups 1 KB apart; K step ks = 16 keys = 2 KB.
__device__ __forceinline__ uint64_t vmn_desc(const uint8_t* tile) {
    return smem_desc(smem_u32(tile), PANEL_BYTES, 1024, LAYOUT_SW128);
}

__global__ void __launch_bounds__(THREADS, 1)
    fwd_bf16qk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
            mbar_init(smem_u32(&sm.bar_p_ready[i]), 128);
            mbar_init(smem_u32(&sm.bar_o_final[i]), 1);
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
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
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
        // A query tile past N is copied all the same (the copy fills zeros)
        // and its rows are never stored.
        const uint32_t qf = smem_u32(&sm.bar_q_full);
        const int hb = bh / p.H, hh = bh - hb * p.H;  // Q, K, V are addressed as [B][H][N][128]
        if (lane == 0) {
            mbar_arrive_expect_tx(qf, QT * TILE_BYTES);
#pragma unroll
            for (int i = 0; i < QT; ++i) {
                tma_load_4d(smem_u32(sm.q[i]), &tm_q, 0, q0 + BM * i, hh, hb, qf);
                tma_load_4d(smem_u32(sm.q[i]) + PANEL_BYTES, &tm_q, 64, q0 + BM * i, hh, hb, qf);
            }
        }
        int issued = 0;
        for (int j = 0; j < T; ++j) {
            const int s = j % STAGES;
            if (j >= STAGES &&
                !warp_wait(smem_u32(&sm.bar_kv_empty[s]), ((j / STAGES) - 1) & 1, abort_flag, p.status, limit))
                break;
            if (lane == 0) {
                const uint32_t full = smem_u32(&sm.bar_kv_full[s]);
                const int k0 = j * BN;
                mbar_arrive_expect_tx(full, 2 * TILE_BYTES);
                tma_load_4d(smem_u32(sm.k[s]), &tm_k, 0, k0, hh, hb, full);
                tma_load_4d(smem_u32(sm.k[s]) + PANEL_BYTES, &tm_k, 64, k0, hh, hb, full);
                tma_load_4d(smem_u32(sm.v[s]), &tm_v, 0, k0, hh, hb, full);
                tma_load_4d(smem_u32(sm.v[s]) + PANEL_BYTES, &tm_v, 64, k0, hh, hb, full);
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
        // Descriptors are bases computed once plus constants (the address
        // field of a descriptor is the byte address / 16 and never carries
        // into the next field, shared memory being below 256 KB); one elected
        // lane issues.
        const bool leader = elect_one_sync();
        const uint64_t qd = kmajor_desc(sm.q[0]);   // tile i: + i*TILE/16
        const uint64_t kd0 = kmajor_desc(sm.k[0]);  // stage st: + st*TILE/16
        const uint64_t vd0 = vmn_desc(sm.v[0]);     // stage st: + st*TILE/16, K step: + 2 KB/16
        constexpr uint64_t TD = TILE_BYTES >> 4;
        auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait_spin(bar, parity, abort_flag, p.status, limit));
        };
        auto qk = [&](int i, int st) {
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks)
                mma_bf16_ss(tmem + tm_s(i), qd + TD * i + kmajor_step(ks), kd0 + TD * st + kmajor_step(ks), IDESC_QK,
                            ks > 0 ? 1u : 0u);
            tc_commit(smem_u32(&sm.bar_s_full[i]));
        };
        auto pv = [&](int i, int st, bool acc) {
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks)
                mma_bf16_ts(tmem + tm_o(i), tmem + tm_s(i) + 8u * ks, vd0 + TD * st + 128u * ks, IDESC_PV,
                            (acc || ks > 0) ? 1u : 0u);
        };
        bool ok = wait(smem_u32(&sm.bar_q_full), 0);
        for (int j = 0; ok && j < T; ++j) {
            const int st = j % STAGES;
            const int sp = (j + STAGES - 1) % STAGES;  // stage of j - 1
            if (!wait(smem_u32(&sm.bar_kv_full[st]), (j / STAGES) & 1)) {
                ok = false;
                break;
            }
            if (leader) {
                tc_fence_after();
                qk(0, st);
            }
            __syncwarp();
            if (j > 0) {
                if (!wait(smem_u32(&sm.bar_p_ready[1]), (j - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    tc_fence_after();
                    pv(1, sp, j > 1);
                    tc_commit(smem_u32(&sm.bar_kv_empty[sp]));
                }
            }
            if (leader) qk(1, st);
            __syncwarp();
            if (!wait(smem_u32(&sm.bar_p_ready[0]), j & 1)) {
                ok = false;
                break;
            }
            if (leader) {
                tc_fence_after();
                pv(0, st, j > 0);
                if (j == T - 1) tc_commit(smem_u32(&sm.bar_o_final[0]));
            }
            __syncwarp();
        }
        if (ok && T > 0 && wait(smem_u32(&sm.bar_p_ready[1]), (T - 1) & 1)) {
            if (leader) {
                tc_fence_after();
                pv(1, (T - 1) % STAGES, T > 1);
                tc_commit(smem_u32(&sm.bar_o_final[1]));
            }
            __syncwarp();
        }
        // every MMA this warp issued must finish before TMEM is freed
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
        const float c = p.scale_log2;
        const float2 c2 = make_float2(c, c);
        float m_run = -INFINITY;  // running max (log2 domain) that P, O and the row sum are relative to
        float2 lacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
        const uint32_t s_full = smem_u32(&sm.bar_s_full[qt]);
        const uint32_t p_ready = smem_u32(&sm.bar_p_ready[qt]);
        bool ok = true;
        for (int j = 0; j < T; ++j) {
            if (!warp_wait(s_full, j & 1, abort_flag, p.status, limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[BN];
#pragma unroll
            for (int q = 0; q < BN / 32; ++q) tmem_ld32(s_addr + 32u * q, &sr[32 * q]);
            tmem_wait_ld();
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
            static_assert(BN / 8 == 16, "max tree below covers 16 groups");
            const float mx = fmax3(fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmax3(a[6], a[7], a[8])),
                                   fmax3(a[9], a[10], a[11]), fmax3(fmax3(a[12], a[13], a[14]), a[15], -INFINITY)) *
                             c;
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
            // P (bf16 pairs) over the first 64 columns of S_i
            tmem_st32(s_addr, &pk[0]);
            tmem_st32(s_addr + 32u, &pk[32]);
            // O_i holds every earlier stage (the commit announcing S_i came after
            // O_i += P_i V of the previous stage).  Rescale it when any row of
            // the warp moved its max (whole warp: tcgen05.ld/st are
            // warp-collective; alpha is 1 for rows that did not move).
            if (j > 0 && __any_sync(0xffffffffu, moved)) {
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
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_ready);
        }
        if (ok && T > 0 && warp_wait(smem_u32(&sm.bar_o_final[qt]), 0, abort_flag, p.status, limit)) {
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
                uint32_t r[32];
                tmem_ld32(o_addr + 32u * q, r);
                tmem_wait_ld();
                if (n < N) {
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
            if (p.lse && n < N) p.lse[orow] = (m_run + __log2f(l)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// [B][H][N][128 bf16] with element strides st (multiples of 8): 128B-swizzled
// boxes of 64 channels x 128 rows of one head; x is 0 or 64 (0 or 128 bytes),
// so every box starts on a 16-byte boundary.
bool make_rows_map(CUtensorMap* m, const __nv_bfloat16* base, int B, int H, int N, Strides st) {
    const uint64_t dims[4] = {128, (uint64_t)N, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)st.n * 2, (uint64_t)st.h * 2, (uint64_t)st.b * 2};
    const uint32_t box[4] = {64, 128, 1, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(base), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

int launch_forward_bf16qk(const FwdBf16Args& a, cudaStream_t stream) {
    if (a.BH == 0 || a.N == 0) return FP4ATTN_OK;
    CUtensorMap tq, tk, tv;
    const int B = a.BH / a.H;
    if (!make_rows_map(&tq, a.q, B, a.H, a.N, a.qs) || !make_rows_map(&tk, a.k, B, a.H, a.N, a.ks) ||
        !make_rows_map(&tv, a.v, B, a.H, a.N, a.vs))
        return FP4ATTN_ERR_CUDA;
    static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget");
    const size_t smem = sizeof(Smem) + 1024;
    if (cudaFuncSetAttribute(fwd_bf16qk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return FP4ATTN_ERR_CUDA;
    Params p;
    p.N = a.N;
    p.n_kt = (a.N + BN - 1) / BN;
    const float scale = a.softmax_scale > 0.0f ? a.softmax_scale : 0.08838834764831845f;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o = a.o;
    p.o_sb = a.os.b;
    p.o_sh = a.os.h;
    p.o_sn = a.os.n;
    p.H = a.H;
    p.lse = a.lse;
    p.status = a.status;
    p.limit_ns = kWaitLimitNs;
    dim3 grid((a.N + QT * BM - 1) / (QT * BM), a.BH);
    fwd_bf16qk_kernel<<<grid, THREADS, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? FP4ATTN_OK : FP4ATTN_ERR_CUDA;
}

}  // namespace fp4attn
