// Quantisation prologue: smooth K + Hadamard + NVFP4 pack of Q and K.
//
// Method: FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention" --
// subtract each head's mean key, rotate Q and K by the same orthonormal
// Hadamard matrix, quantise both to NVFP4 (E2M1 values, one E4M3 scale per 16
// channels, fp32 per-tensor scale).  The fused transform there costs under
// 1 ms per attention call on GB200.
//
// One persistent kernel.  CTAs take 128-row tiles from an atomic ticket queue
// ordered per head as [key-sum tiles][Q tiles][K tiles]:
//   key-sum tile   exact int64 fixed-point column sums of K (sum of
//                  round_half_even(k * 2^24)); order-independent, so atomics
//                  give the same bits as any serial order; then the head's
//                  ready counter is bumped;
//   Q / K tile     two threads per 128-channel row: bf16 -> fp32, (K) minus
//                  the head mean once the head's counter is complete, the 7
//                  butterfly stages of the Walsh-Hadamard transform,
//                  x fp32(1/sqrt(128)), per-16 amax, UE4M3 scale amax/6/g,
//                  E2M1 codes of y * (1/(g*scale)).
// The Q tiles of a head sit between its key-sum and K tiles, so the second
// read of K mostly hits L2 (key-sum loads are marked evict-last, the others
// evict-first).  Q and K may have any [B,H,N,128] strides (a 4-D tensor map).
//
// Dynamic global scales (g = amax / (6*448) of each whole transformed tensor)
// take two launches of the same kernel: the first (AMAX) does the key sums and
// the transform of every Q and K row and reduces the largest magnitude of each
// tensor into two workspace words; the second encodes, with g computed from
// those words, and skips the key sums, which are already complete.  Tiles arrive by TMA (128B swizzle) in a ring of NBUF buffers
// per CTA.  Each tile is first copied from its buffer into registers; after
// one barrier the buffer is refilled with the tile NBUF tickets ahead, so every
// buffer is in flight while a tile is computed.
//
// A row's 128 values live in the registers of two neighbouring lanes as pairs
// (x_i, x_{i+64}), lane h holding i in [32h, 32h+32): the butterfly stages of
// stride 1..16 run on packed fp32x2 instructions inside a lane, stride 32
// between the two lanes (one shuffle per value), stride 64 inside each pair.
// Every fp32 step is an explicit round-to-nearest operation applied in the
// same stage order as the plain CPU definition, so the codes are bit-identical
// to it.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace fp4attn {

namespace {

constexpr float kTwo24 = 16777216.0f;
constexpr float kKeyLimit = 1048576.0f;  // |k| < 2^20 keeps the int64 sum exact for N <= 2^18
constexpr int PRO_THREADS = 256;         // two threads per row of a 128-row tile
constexpr uint32_t HALF_BYTES = 128 * 128;        // 128 rows x 64 channels bf16
constexpr uint32_t TILE_BYTES = 2 * HALF_BYTES;   // 32 KB
constexpr uint64_t kSpinLimitNs = 2000000000ull;

enum TileKind { KIND_KSUM = 0, KIND_Q = 1, KIND_K = 2 };

constexpr int NBUF = 3;  // tile ring depth: NBUF-1 tiles in flight while one is computed

struct __align__(1024) ProSmem {
    uint8_t tile[NBUF][TILE_BYTES];  // channels 0-63 then 64-127, 128B swizzle
    long long kpart[PRO_THREADS / 32][128];  // key-sum partials of the warps
    float2 neg_mean2[64];            // (-m_i, -m_{i+64})
    float inv_scale[128];            // fp32 1 / value of each UE4M3 code (0 for code 0)
    uint64_t bar[NBUF];
    int next_ticket[NBUF];
    int4 next_tile[NBUF];            // the ticket decoded by thread 0: (kind, head, tile, -)
    int mean_head;
    int abort_flag;
};

struct ProArgs {
    uint8_t* codes[2];
    uint8_t* scales[2];
    const float* g[2];
    float* g_out[2];   // encode launch of the dynamic path: receive g of Q and K
    unsigned* amax;    // dynamic path: fp32 bits of the transformed amax of Q and K
    long long* ksum;
    unsigned* head_ready;
    unsigned* ticket;
    float* k_mean;
    int BH, H, N, n_tiles;
    uint32_t flags;
    bool sums_ready;   // the key sums of every head are complete: no key-sum tiles
    int* status;
};

// g = fl32(amax / (6*448)), raised to 2^-64 when smaller, so that g * scale
// and its reciprocal stay finite and normal.
__device__ __forceinline__ float tensor_gscale(float amax) {
    return fmaxf(__fdiv_rn(amax, 2688.0f), 5.42101086242752217e-20f);
}

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                                 int32_t c2, int32_t c3, uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar), "l"(policy)
        : "memory");
}

// Byte offset of 16-byte chunk j (0..7) of row r inside one 128B-swizzled
// half tile: the chunk index is XORed with the row index mod 8, which also
// makes eight consecutive rows reading the same chunk hit distinct banks.
__device__ __forceinline__ uint32_t swz(int r, int j) { return (uint32_t)r * 128u + ((uint32_t)(j ^ (r & 7)) << 4); }

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, f2(-1.0f, -1.0f), a); }

__device__ __forceinline__ float amax16(const float2* p, bool hi) {
    float a[6];
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const float x0 = hi ? p[3 * k].y : p[3 * k].x;
        const float x1 = hi ? p[3 * k + 1].y : p[3 * k + 1].x;
        const float x2 = hi ? p[3 * k + 2].y : p[3 * k + 2].x;
        a[k] = fmax3(fabsf(x0), fabsf(x1), fabsf(x2));
    }
    a[5] = fabsf(hi ? p[15].y : p[15].x);
    return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), 0.0f);
}

// Scale byte and 1/(g*scale) of one block with amax a.
__device__ __forceinline__ void block_scale(float a, float g, bool g_is_one, const float* inv_tab, uint32_t& s,
                                            float& inv) {
    float t = div6_rn(a);
    if (!g_is_one) t = __fdiv_rn(t, g);
    s = cvt_e4m3(t);  // t >= +0: the E4M3 byte is the UE4M3 byte
    if (g_is_one) {
        inv = inv_tab[s];
    } else {
        const float sd = ue4m3_value(s);
        inv = (sd != 0.0f) ? __frcp_rn(__fmul_rn(g, sd)) : 0.0f;
    }
}

// AMAX = true: the first launch of the dynamic-scale path (key sums and the
// transformed amax of Q and K; no codes are written).
template <bool AMAX>
__global__ void __launch_bounds__(PRO_THREADS, 2) prologue_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const ProArgs a) {
    extern __shared__ uint8_t smem_raw[];
    ProSmem& sm = *reinterpret_cast<ProSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int N = a.N;
    const int Th = a.n_tiles;
    const bool smooth = !(a.flags & FP4ATTN_NO_SMOOTH_K);
    const bool hadamard = !(a.flags & FP4ATTN_NO_HADAMARD);
    const int first_kind = (smooth && !a.sums_ready) ? KIND_KSUM : KIND_Q;
    const int per_head = (3 - first_kind) * Th;
    const int total = a.BH * per_head;

    if (tid == 0) {
        for (int b = 0; b < NBUF; ++b) mbar_init(smem_u32(&sm.bar[b]), 1);
        sm.mean_head = -1;
        sm.abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
    }
    if (tid < 128) {
        const float sd = ue4m3_value(tid);  // codes 0..127 cover every scale; 127 (NaN) is never produced
        sm.inv_scale[tid] = (sd != 0.0f) ? __frcp_rn(sd) : 0.0f;
    }
    float gq = 1.0f, gk = 1.0f;
    if (!AMAX && a.amax) {  // encode launch of the dynamic path
        gq = tensor_gscale(__uint_as_float(__ldcg(a.amax)));
        gk = tensor_gscale(__uint_as_float(__ldcg(a.amax + 1)));
        if (blockIdx.x == 0 && tid == 0) {
            if (a.g_out[0]) *a.g_out[0] = gq;
            if (a.g_out[1]) *a.g_out[1] = gk;
        }
    } else if (!AMAX) {
        if (a.g[0]) gq = *a.g[0];
        if (a.g[1]) gk = *a.g[1];
    }
    if (tid == 0 && !(gq > 0.0f && gq < INFINITY && gk > 0.0f && gk < INFINITY)) set_status(a.status, FP4ATTN_ERR_RANGE);
    __syncthreads();

    const uint64_t pol_keep = l2_policy_evict_last();
    const uint64_t pol_stream = l2_policy_evict_first();
    auto decode = [&](int t, int& kind, int& bh, int& tile) {
        bh = t / per_head;
        const int l = t - bh * per_head;
        kind = first_kind + l / Th;
        tile = l % Th;
    };
    auto issue = [&](int t, int buf) {  // thread 0 only; also publishes the decoded ticket
        int kind, bh, tile;
        decode(t, kind, bh, tile);
        sm.next_tile[buf] = make_int4(kind, bh, tile, 0);
        const CUtensorMap* map = (kind == KIND_Q) ? &tm_q : &tm_k;
        const uint64_t pol = (kind == KIND_KSUM) ? pol_keep : pol_stream;
        const uint32_t bar = smem_u32(&sm.bar[buf]);
        const int b = bh / a.H, h = bh - b * a.H;
        mbar_arrive_expect_tx(bar, TILE_BYTES);
        tma_load_4d_hint(smem_u32(sm.tile[buf]), map, 0, tile * 128, h, b, bar, pol);
        tma_load_4d_hint(smem_u32(sm.tile[buf]) + HALF_BYTES, map, 64, tile * 128, h, b, bar, pol);
    };

    uint32_t in_flight = 0u;  // bit b: a copy into buffer b is outstanding (thread 0, which issues them)
    float amax_q = 0.0f, amax_k = 0.0f;  // AMAX: largest |y| of this thread's valid Q and K rows
    if (tid == 0) {
        for (int b = 0; b < NBUF; ++b) {
            const int tk = (int)atomicAdd(a.ticket, 1u);
            sm.next_ticket[b] = tk;
            if (tk < total) {
                issue(tk, b);
                in_flight |= 1u << b;
            }
        }
    }
    __syncthreads();
    int t = sm.next_ticket[0];
    int buf = 0;
    uint32_t phase = 0u;  // bit b: parity of the next phase of buffer b

    // Each tile is first copied from its buffer into registers; after one barrier
    // the buffer is refilled with the tile NBUF iterations ahead, so all NBUF
    // buffers are in flight while the tile is computed.
    auto release = [&](int b) {  // after the barrier that ends the reads of buffer b
        if (tid == 0) {
            const int tn = (int)atomicAdd(a.ticket, 1u);
            sm.next_ticket[b] = tn;
            if (tn < total) {
                issue(tn, b);
                in_flight |= 1u << b;
            }
        }
    };
    while (t < total) {
        const int4 dt = sm.next_tile[buf];  // decoded by thread 0 with the ticket
        const int kind = dt.x, bh = dt.y, tile = dt.z;
        const bool landed = mbar_wait(smem_u32(&sm.bar[buf]), (phase >> buf) & 1u, &sm.abort_flag, a.status, kSpinLimitNs);
        if (__syncthreads_or(!landed)) break;
        phase ^= 1u << buf;
        in_flight &= ~(1u << buf);
        const uint8_t* tb = sm.tile[buf];

        if (kind == KIND_KSUM) {
            // ------------------------------------------------ key sums ----
            // warp w: rows 16w..16w+15; lane l: channels 4l..4l+3 (one 8-byte load
            // per row), four independent int64 accumulators
            const int warp = tid >> 5, lane = tid & 31;
            const uint8_t* hb = tb + (lane >> 4) * HALF_BYTES;
            const int j = (lane & 15) >> 1;
            const uint32_t in_chunk = (uint32_t)(lane & 1) * 8u;
            uint2 kw[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) kw[rr] = *reinterpret_cast<const uint2*>(hb + swz(16 * warp + rr, j) + in_chunk);
            __syncthreads();
            release(buf);
            // |k| is checked once per thread against 2^20 (out-of-range keys make
            // the outputs unspecified and raise the status; non-finite keys are
            // also caught by the K tiles' transform of the same rows)
            long long acc[4] = {0, 0, 0, 0};
            float kmax = 0.0f;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const float v[4] = {bf16lo(kw[rr].x), bf16hi(kw[rr].x), bf16lo(kw[rr].y), bf16hi(kw[rr].y)};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[c] += __float2ll_rn(__fmul_rn(v[c], kTwo24));
                    kmax = fmaxf(kmax, fabsf(v[c]));
                }
            }
            if (!(kmax < kKeyLimit)) set_status(a.status, FP4ATTN_ERR_RANGE);
#pragma unroll
            for (int c = 0; c < 4; ++c) sm.kpart[warp][4 * lane + c] = acc[c];
            __syncthreads();
            if (tid < 128) {
                long long tot = 0;
#pragma unroll
                for (int w = 0; w < PRO_THREADS / 32; ++w) tot += sm.kpart[w][tid];
                atomicAdd(reinterpret_cast<unsigned long long*>(a.ksum + (size_t)bh * D + tid),
                          static_cast<unsigned long long>(tot));
            }
            // the CTA barrier makes every thread's sum visible to thread 0, whose
            // device-scope fence then orders them all before the ready count
            __syncthreads();
            if (tid == 0) {
                __threadfence();
                atomicAdd(a.head_ready + bh, 1u);
            }
        } else {
            const int which = kind - 1;  // 0 = Q, 1 = K
            if (which == 1 && sm.mean_head != bh) {
                // ------------------------------------------ head means ----
                bool ready = true;
                if (smooth && tid == 0) {
                    volatile unsigned* cnt = a.head_ready + bh;
                    const uint64_t t0 = globaltimer_ns();
                    while (*cnt < (unsigned)Th) {
                        if (globaltimer_ns() - t0 > kSpinLimitNs) {
                            set_status(a.status, FP4ATTN_ERR_TIMEOUT);
                            ready = false;
                            break;
                        }
                        __nanosleep(64);
                    }
                    __threadfence();
                }
                if (__syncthreads_or(!ready)) break;
                if (tid < 128) {
                    float m = 0.0f;
                    if (smooth) {
                        const long long S = __ldcg(a.ksum + (size_t)bh * D + tid);
                        m = __double2float_rn(__ddiv_rn(__ll2double_rn(S), (double)N * 16777216.0));
                    }
                    if (tid < 64) sm.neg_mean2[tid].x = -m; else sm.neg_mean2[tid - 64].y = -m;
                    if (a.k_mean && tile == 0) a.k_mean[(size_t)bh * D + tid] = m;
                }
                __syncthreads();
                if (tid == 0) sm.mean_head = bh;
            }
            // ---------------------------------------------- one row ----
            // lanes 2r', 2r'+1 of a warp share row r; lane half h holds the pairs
            // P[k] = (x_i, x_{i+64}), i = 32h + k
            const int r = tid >> 1;
            const int h = tid & 1;
            float2 P[32];
            const bool sub_mean = (which == 1) && smooth;
            bool finite = true;
            uint4 rlo[4], rhi[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                rlo[j] = *reinterpret_cast<const uint4*>(tb + swz(r, 4 * h + j));
                rhi[j] = *reinterpret_cast<const uint4*>(tb + HALF_BYTES + swz(r, 4 * h + j));
            }
            __syncthreads();
            release(buf);
            // chunk j (8 pairs, k = 8j..8j+7): unpack, smooth, and apply the
            // butterfly stages of stride 1, 2, 4, which stay inside the chunk
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 lo = rlo[j], hi = rhi[j];
                const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w};
                const uint32_t wh[4] = {hi.x, hi.y, hi.z, hi.w};
                float2* C = P + 8 * j;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    C[2 * e] = f2(bf16lo(wl[e]), bf16lo(wh[e]));
                    C[2 * e + 1] = f2(bf16hi(wl[e]), bf16hi(wh[e]));
                }
                if (sub_mean) {
                    const float4* nm = reinterpret_cast<const float4*>(sm.neg_mean2 + 32 * h + 8 * j);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 m4 = nm[e];
                        C[2 * e] = __fadd2_rn(C[2 * e], f2(m4.x, m4.y));
                        C[2 * e + 1] = __fadd2_rn(C[2 * e + 1], f2(m4.z, m4.w));
                    }
                }
                if (!hadamard) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) finite &= (fabsf(C[i].x) < INFINITY) && (fabsf(C[i].y) < INFINITY);
                } else {
#pragma unroll
                    for (int st = 1; st < 8; st <<= 1) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if ((i & st) == 0) {
                                const float2 x = C[i], y = C[i + st];
                                C[i] = __fadd2_rn(x, y);
                                C[i + st] = sub2(x, y);
                            }
                        }
                    }
                }
            }
            if (hadamard) {
                // strides 8 and 16 across chunks
#pragma unroll
                for (int st = 8; st < 32; st <<= 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if ((i & st) == 0) {
                            const float2 x = P[i], y = P[i + st];
                            P[i] = __fadd2_rn(x, y);
                            P[i + st] = sub2(x, y);
                        }
                    }
                }
                // stride 32 between the two lanes of the row: lane 0 keeps
                // x_i + x_{i+32}, lane 1 keeps x_i - x_{i+32}
                const float sg = h ? -1.0f : 1.0f;  // fl(other + sg * own): the sum or the difference, one rounding
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float ox = __shfl_xor_sync(0xffffffffu, P[k].x, 1);
                    const float oy = __shfl_xor_sync(0xffffffffu, P[k].y, 1);
                    P[k] = __ffma2_rn(P[k], f2(sg, sg), f2(ox, oy));
                }
                // stride 64 inside each pair
#pragma unroll
                for (int k = 0; k < 32; ++k) P[k] = f2(__fadd_rn(P[k].x, P[k].y), __fsub_rn(P[k].x, P[k].y));
                // y_0 (lane 0, P[0].x) is the sum of all 128 inputs: it is finite iff
                // they all are (barring overflow of the sum itself)
                finite = (h != 0) || (fabsf(P[0].x) < INFINITY);
                const float c = __uint_as_float(0x3DB504F3u);  // fp32(1/sqrt(128))
#pragma unroll
                for (int k = 0; k < 32; ++k) P[k] = __fmul2_rn(P[k], f2(c, c));
            }

            const bool valid = (tile * 128 + r) < N;
            if (!finite && valid) set_status(a.status, FP4ATTN_ERR_RANGE);
            if constexpr (AMAX) {
                // rows past N hold the copy's zero fill (minus the mean for K): skip them
                if (valid) {
                    float m = 0.0f;
#pragma unroll
                    for (int k = 0; k < 32; ++k) m = fmax3(m, fabsf(P[k].x), fabsf(P[k].y));
                    if (which) amax_k = fmaxf(amax_k, m); else amax_q = fmaxf(amax_q, m);
                }
            } else {
            // NVFP4 pack.  This lane holds blocks 2h, 2h+1 (the .x lanes of
            // P[0..15], P[16..31]) and 4+2h, 5+2h (the .y lanes); block b's codes
            // are bytes 8b..8b+7 of the row.
            const float gw = which ? gk : gq;
            const bool g_is_one = (gw == 1.0f);
            const size_t row = (size_t)bh * N + (size_t)tile * 128 + r;
            uint32_t s_b[4];  // scale bytes of blocks 2h, 2h+1, 4+2h, 5+2h
            uint32_t w_lo[4], w_hi[4];
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                float inv_lo, inv_hi;
                block_scale(amax16(P + 16 * bb, false), gw, g_is_one, sm.inv_scale, s_b[bb], inv_lo);
                block_scale(amax16(P + 16 * bb, true), gw, g_is_one, sm.inv_scale, s_b[2 + bb], inv_hi);
                const float2 inv2 = f2(inv_lo, inv_hi);
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    float2 R[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) R[k] = __fmul2_rn(P[16 * bb + 8 * h8 + k], inv2);
                    w_lo[2 * bb + h8] = cvt_e2m1x8(R[0].x, R[1].x, R[2].x, R[3].x, R[4].x, R[5].x, R[6].x, R[7].x);
                    w_hi[2 * bb + h8] = cvt_e2m1x8(R[0].y, R[1].y, R[2].y, R[3].y, R[4].y, R[5].y, R[6].y, R[7].y);
                }
            }
            // scale bytes: lane 0 writes blocks 0-3, lane 1 blocks 4-7
            const uint32_t mine_lo = s_b[0] | (s_b[1] << 8), mine_hi = s_b[2] | (s_b[3] << 8);
            const uint32_t other = __shfl_xor_sync(0xffffffffu, h ? mine_lo : mine_hi, 1);
            const uint32_t sword = h ? (other | (mine_hi << 16)) : (mine_lo | (other << 16));
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>((which ? a.codes[1] : a.codes[0]) + row * 64);
                dst[h] = make_uint4(w_lo[0], w_lo[1], w_lo[2], w_lo[3]);
                dst[2 + h] = make_uint4(w_hi[0], w_hi[1], w_hi[2], w_hi[3]);
                *reinterpret_cast<uint32_t*>((which ? a.scales[1] : a.scales[0]) + row * 8 + 4 * h) = sword;
            }
            }  // pack
        }
        // the next buffer's ticket was written at least one barrier ago
        buf = (buf + 1) % NBUF;
        t = sm.next_ticket[buf];
    }
    if constexpr (AMAX) {
        // magnitudes are >= 0, so their fp32 bit patterns order like the values
        const unsigned wq = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_q));
        const unsigned wk = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_k));
        if ((tid & 31) == 0) {
            if (wq) atomicMax(a.amax, wq);
            if (wk) atomicMax(a.amax + 1, wk);
        }
    }
    // wind down after an abort: let this CTA's own copies land before exiting
    if (tid == 0) {
        int dummy = 0;
        for (int b = 0; b < NBUF; ++b)
            if (in_flight & (1u << b)) mbar_wait(smem_u32(&sm.bar[b]), (phase >> b) & 1u, &dummy, nullptr, 200000000ull);
    }
}

size_t pro_smem_bytes() { return sizeof(ProSmem) + 1024; }

// [B][H][N][128 bf16] with element strides st: 128B-swizzled boxes of 64
// channels x 128 rows of one head; x is 0 or 64 (0 or 128 bytes), so every box
// starts on a 16-byte boundary.  The strides must be multiples of 8 elements.
bool make_rows_map(CUtensorMap* m, const __nv_bfloat16* base, int B, int H, int N, Strides st) {
    const uint64_t dims[4] = {128, (uint64_t)N, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)st.n * 2, (uint64_t)st.h * 2, (uint64_t)st.b * 2};
    const uint32_t box[4] = {64, 128, 1, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(base), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <bool AMAX>
cudaError_t launch_pass(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ProArgs& a, cudaStream_t stream) {
    static_assert(sizeof(ProSmem) + 1024 <= 227 * 1024, "shared memory budget");
    const size_t smem = pro_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(prologue_kernel<AMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prologue_kernel<AMAX>, PRO_THREADS, smem)) !=
        cudaSuccess)
        return e;
    const bool sum_tiles = !(a.flags & FP4ATTN_NO_SMOOTH_K) && !a.sums_ready;
    const long long tiles = (long long)a.BH * a.n_tiles * (sum_tiles ? 3 : 2);
    long long grid = (long long)sms * (per_sm > 0 ? per_sm : 1);
    if (grid > tiles) grid = tiles;
    prologue_kernel<AMAX><<<(unsigned)grid, PRO_THREADS, smem, stream>>>(tm_q, tm_k, a);
    return cudaGetLastError();
}

__global__ void store_gscales_kernel(float* gq, float* gk) {
    *gq = tensor_gscale(0.0f);
    *gk = tensor_gscale(0.0f);
}

}  // namespace

cudaError_t launch_store_gscales(float* gq, float* gk, cudaStream_t stream) {
    store_gscales_kernel<<<1, 1, 0, stream>>>(gq, gk);
    return cudaGetLastError();
}

cudaError_t launch_quantize_qk(const QuantArgs& q, cudaStream_t stream) {
    if (q.BH == 0 || q.N == 0) return cudaSuccess;
    const int B = q.BH / q.H;
    CUtensorMap tm_q, tm_k;
    if (!make_rows_map(&tm_q, q.q, B, q.H, q.N, q.qs) || !make_rows_map(&tm_k, q.k, B, q.H, q.N, q.ks))
        return cudaErrorInvalidValue;
    ProArgs a{};
    a.codes[0] = q.q_codes;
    a.codes[1] = q.k_codes;
    a.scales[0] = q.q_scales;
    a.scales[1] = q.k_scales;
    a.g[0] = q.gq;
    a.g[1] = q.gk;
    a.ksum = q.ksum;
    a.head_ready = q.counters;
    a.ticket = q.ticket;
    a.k_mean = q.k_mean;
    a.BH = q.BH;
    a.H = q.H;
    a.N = q.N;
    a.n_tiles = (q.N + 127) / 128;
    a.flags = q.flags & ~QUANT_DYNAMIC_G;
    a.status = q.status;
    if (!(q.flags & QUANT_DYNAMIC_G)) return launch_pass<false>(tm_q, tm_k, a, stream);
    // dynamic global scales: amax pass (with the key sums), then the encode pass
    ProArgs m = a;
    m.amax = q.amax;
    m.k_mean = nullptr;
    cudaError_t e = launch_pass<true>(tm_q, tm_k, m, stream);
    if (e != cudaSuccess) return e;
    a.amax = q.amax;
    a.g_out[0] = q.g_out[0];
    a.g_out[1] = q.g_out[1];
    a.ticket = q.ticket + 1;
    a.sums_ready = true;
    return launch_pass<false>(tm_q, tm_k, a, stream);
}

}  // namespace fp4attn
