// Quantisation prologue: smooth K + Hadamard + NVFP4 pack of Q and K.
//
// Method: FastVideo "Pika H3 Flex in FastVideo", section "FP4 attention" --
// subtract each head's mean key, rotate Q and K by the same orthonormal
// Hadamard matrix, quantise both to NVFP4 (E2M1 values, one E4M3 scale per 16
// channels, fp32 per-tensor scale).  The fused transform there costs under
// 1 ms per attention call on GB200.
//
// One persistent, warp-specialised kernel per launch.  A tile is 16*W rows of
// one head; tiles come from an atomic ticket queue (in runs of consecutive
// tickets, one atomic per run) in which every head contributes three runs:
// key-sum tiles (exact int64 fixed-point column sums of K, the sum of
// round_half_even(k * 2^24), order-independent), Q tiles and K tiles.  The
// key sums of head h+L are placed between the Q and the K tiles of head h,
// with the lead L the smallest that keeps every CTA's unfinished tickets
// from reaching a head's K tiles before its sums are complete, so a K tile
// does not wait, while K is still in L2 for its second read (key-sum loads
// are marked evict-last, the others evict-first).
//
// Warp W of each CTA is the producer: it takes tickets and moves each tile by
// TMA (two 128B-swizzled boxes of 64 channels) into a ring of NSLOT shared-
// memory slots, each with a "full" and an "empty" mbarrier.  Consumer warp w
// (0 <= w < W) owns rows 16w..16w+15 of every tile: it waits for the slot to
// fill, copies its rows into registers, arrives on the slot's empty barrier
// and computes.  No CTA-wide barrier is taken after the set-up, so the
// consumer warps drift freely within the depth of the ring.  The producer
// takes a ticket only when a slot is free and asks for the next run with the
// last ticket of the current one, so a CTA holds at most NSLOT + run
// unfinished tickets; the lead L is sized from that at launch.
//
// Key-sum rows: lane l sums channels 4l..4l+3 of the warp's 16 rows into four
// int64 registers.  A warp keeps summing while its tiles stay on one head;
// when that run of tiles ends, the W warps of the CTA combine their sums in
// shared memory and the last of them adds the run's 128 sums to the
// workspace with 64-bit atomics, then a device fence and the head's count of
// 16-row chunks.  A K tile follows every key-sum tile of its head in the
// ticket order, and a warp reaches a K tile only after its run has ended, so
// a warp that waits for a head's sums never holds any of them back.  A K row
// needs its head's means: the consumer warp waits for the head's count to
// reach every chunk, then computes the 128 means once per head into its own
// shared memory.  With key sums, a warp copies its rows and releases the
// slot before it flushes a run or waits for a head's means, so neither
// holds up the ring.
//
// Q / K rows: two lanes per row.  Lane h holds the pairs (x_i, x_{i+64}) for
// i in [32h, 32h+32) as 32 packed fp32x2 registers: the butterflies of stride
// 1..16 run on packed fp32x2 instructions inside a lane, stride 32 between
// the two lanes (each lane receives the partner's 64 values and keeps the sum
// or the difference, as fl(other + sign * own), one rounding), stride 64
// inside each pair, then x fp32(1/sqrt(128)).  Every fp32 step is an explicit
// round-to-nearest operation in the same stage order as the plain CPU
// definition, so the codes are bit-identical to it, signed zeros included.
// Each lane then owns four whole 16-value blocks: per-block amax, the UE4M3
// scale amax/6/g, E2M1 codes of y * (1/(g * scale)).  The kernel comes in one
// instance per setting of the two transforms, and the packing in one version
// for g == 1 (scale reciprocals from a table) and one for other g.
//
// Dynamic global scales (g = amax / (6*448) of each whole transformed tensor)
// take two launches of the same kernel: the first (AMAX) does the key sums and
// the transform of every Q and K row and reduces the largest magnitude of each
// tensor into two workspace words; the second encodes, with g computed from
// those words, and skips the key sums, which are already complete.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

#ifndef FP4ATTN_PRO_W
#define FP4ATTN_PRO_W 15       // consumer warps per CTA (16 rows each per tile)
#endif
#ifndef FP4ATTN_PRO_NSLOT
#define FP4ATTN_PRO_NSLOT 3    // tile slots in the ring
#endif
#ifndef FP4ATTN_PRO_CTAS
#define FP4ATTN_PRO_CTAS 1     // resident CTAs per SM the kernel is built for
#endif
#ifndef FP4ATTN_PRO_RUN
#define FP4ATTN_PRO_RUN 8      // most consecutive tiles per ticket request
#endif
#ifndef FP4ATTN_PRO_LEAD
#define FP4ATTN_PRO_LEAD 1     // least lead of the key sums over the K tiles (0: ahead of Q(h))
#endif

namespace fp4attn {

namespace {

constexpr float kTwo24 = 16777216.0f;
constexpr float kSumLimit = 17592186044416.0f;  // 2^44: |k| < 2^20 keeps the int64 sum exact for N <= 2^18
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;

constexpr int W = FP4ATTN_PRO_W;
constexpr int NSLOT = FP4ATTN_PRO_NSLOT;
constexpr int CTAS_PER_SM = FP4ATTN_PRO_CTAS;
constexpr int MAX_TICKET_RUN = FP4ATTN_PRO_RUN;
constexpr int PRO_THREADS = 32 * (W + 1);
constexpr int TILE_ROWS = 16 * W;
constexpr uint32_t HALF_BYTES = TILE_ROWS * 128;  // TILE_ROWS rows x 64 channels bf16
constexpr uint32_t TILE_BYTES = 2 * HALF_BYTES;
static_assert(NSLOT <= 16 && TILE_ROWS <= 256, "ring bookkeeping and TMA box limits");

enum TileKind { KIND_KSUM = 0, KIND_Q = 1, KIND_K = 2, KIND_END = 3 };

struct __align__(1024) ProSmem {
    uint8_t tile[NSLOT][TILE_BYTES];  // channels 0-63 then 64-127, 128B swizzle
    float2 neg_mean2[W][64];          // per consumer warp: (-m_i, -m_{i+64}) of its current K head
    float inv_scale[128];             // fp32 1 / value of each UE4M3 code (0 for code 0)
    int4 meta[NSLOT];                 // (kind, head, tile, -) of the tile in each slot
    uint64_t full[NSLOT];
    uint64_t empty[NSLOT];
    unsigned long long csum[2][128];  // key sums of the CTA's current run, two runs in turn
    int run_warps[2];                 // consumer warps that have added their share to csum[b]
    int run_gen[2];                   // runs completed through csum[b]
    int abort_flag;
};

struct ProArgs {
    uint8_t* codes[2];
    uint8_t* scales[2];
    const float* g[2];
    float* g_out[2];   // encode launch of the dynamic path: receive g of Q and K
    unsigned* amax;    // dynamic path: fp32 bits of the transformed amax of Q and K
    long long* ksum;
    unsigned* head_ready;  // per head: 16-row key-sum chunks summed
    unsigned* ticket;
    float* k_mean;
    int BH, H, N, n_tiles;
    uint32_t flags;
    bool sums_ready;   // the key sums of every head are complete: no key-sum tiles
    bool withhold_sums;  // test hook: K tiles wait for key sums that no tile computes
    int lead;          // L >= 1: key sums of head h+L between Q(h) and K(h); 0: ahead of Q(h)
    int run;           // consecutive tiles per ticket request
    uint64_t spin_limit_ns;
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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
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

// Scale byte and 1/(g*scale) of one 16-value block with amax a >= 0.  The
// quotient a/6 is fl(a * fl(1/6)) corrected by one FMA: equal to the IEEE
// quotient for every a >= 2^-123 (checked over all fp32 patterns).  Below
// that, a/6/g < 2^-61 for every admissible g (g >= 2^-64), far under half of
// the smallest UE4M3 step (2^-9), so the byte is 0 whatever the low bits of
// the quotient and no exact-divide path is needed; the sign bit is cleared
// so that a -0 could not give the byte 0x80.
template <bool G1>
__device__ __forceinline__ void block_scale(float a, float g, const float* inv_tab, uint32_t& s, float& inv) {
    float t = div6_refined(a);
    if (!G1) t = __fdiv_rn(t, g);
    s = cvt_e4m3(t) & 0x7Fu;
    if (G1) {
        inv = inv_tab[s];
    } else {
        const float sd = ue4m3_value(s);
        inv = (sd != 0.0f) ? __frcp_rn(__fmul_rn(g, sd)) : 0.0f;
    }
}

// NVFP4 pack of a lane's four blocks: group q = P[16q..16q+15], its .x values
// one block and its .y values another; sb receives the four scale bytes (.x
// of groups 0, 1, then .y), wx / wy the code words (block order as sb).
template <bool G1>
__device__ __forceinline__ void pack_blocks(const float2* P, float g, const float* inv_tab, uint32_t (&sb)[4],
                                            uint32_t (&wx)[2][2], uint32_t (&wy)[2][2]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        float inv_x, inv_y;
        block_scale<G1>(amax16(P + 16 * q, false), g, inv_tab, sb[q], inv_x);
        block_scale<G1>(amax16(P + 16 * q, true), g, inv_tab, sb[2 + q], inv_y);
        const float2 inv2 = f2(inv_x, inv_y);
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            float2 R[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) R[k] = __fmul2_rn(P[16 * q + 8 * h8 + k], inv2);
            wx[q][h8] = cvt_e2m1x8(R[0].x, R[1].x, R[2].x, R[3].x, R[4].x, R[5].x, R[6].x, R[7].x);
            wy[q][h8] = cvt_e2m1x8(R[0].y, R[1].y, R[2].y, R[3].y, R[4].y, R[5].y, R[6].y, R[7].y);
        }
    }
}

// Ticket t -> (kind, flat head, tile).  With key sums (sums), lead L >= 1:
// the key sums of heads 0..L-1 first, then per head h [Q(h)][key sums of
// h+L][K(h)] (the last L heads without the middle run); lead 0:
// [key sums of h][Q(h)][K(h)].
__device__ __forceinline__ void decode_ticket(int t, int Th, int BH, bool sums, int lead, int& kind, int& bh,
                                              int& tile) {
    if (!sums) {
        bh = t / (2 * Th);
        const int l = t - bh * 2 * Th;
        kind = l < Th ? KIND_Q : KIND_K;
        tile = l < Th ? l : l - Th;
        return;
    }
    if (lead == 0) {
        bh = t / (3 * Th);
        const int l = t - bh * 3 * Th;
        const int part = l / Th;
        kind = part == 0 ? KIND_KSUM : (part == 1 ? KIND_Q : KIND_K);
        tile = l - part * Th;
        return;
    }
    const int first = lead < BH ? lead : BH;  // heads whose key sums come first
    if (t < first * Th) {
        kind = KIND_KSUM;
        bh = t / Th;
        tile = t - bh * Th;
        return;
    }
    t -= first * Th;
    const int inner = BH - first;  // heads with a run of later key sums inside
    if (t < inner * 3 * Th) {
        const int h = t / (3 * Th), l = t - h * 3 * Th;
        if (l < Th) {
            kind = KIND_Q;
            bh = h;
            tile = l;
        } else if (l < 2 * Th) {
            kind = KIND_KSUM;
            bh = h + lead;
            tile = l - Th;
        } else {
            kind = KIND_K;
            bh = h;
            tile = l - 2 * Th;
        }
        return;
    }
    t -= inner * 3 * Th;
    const int h = inner + t / (2 * Th), l = t - (h - inner) * 2 * Th;
    kind = l < Th ? KIND_Q : KIND_K;
    bh = h;
    tile = l < Th ? l : l - Th;
}

// AMAX = true: the first launch of the dynamic-scale path (key sums and the
// transformed amax of Q and K; no codes are written).
template <bool AMAX, bool HAD, bool SMOOTH>
__global__ void __launch_bounds__(PRO_THREADS, CTAS_PER_SM) prologue_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                          const __grid_constant__ CUtensorMap tm_k,
                                                                          const ProArgs a) {
    extern __shared__ uint8_t smem_raw[];
    ProSmem& sm = *reinterpret_cast<ProSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int N = a.N;
    const int Th = a.n_tiles;
    constexpr bool smooth = SMOOTH;  // one instance per setting of the two transforms
    constexpr bool hadamard = HAD;
    const bool sums = smooth && !a.sums_ready && !a.withhold_sums;
    const int total = a.BH * Th * (sums ? 3 : 2);

    if (tid == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), W);
        }
        sm.abort_flag = 0;
        for (int b = 0; b < 2; ++b) sm.run_warps[b] = sm.run_gen[b] = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
    }
    if (tid < 128) {
        sm.csum[0][tid] = sm.csum[1][tid] = 0ull;
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

    if (warp == W) {
        // ------------------------------------------------------ producer ----
        if (lane == 0) {
            const uint64_t pol_keep = l2_policy_evict_last();
            const uint64_t pol_stream = l2_policy_evict_first();
            uint32_t filled = 0u, parity = 0u;  // per slot: ever filled; parity of its last fill
            // tickets come in runs of a.run consecutive tiles.  A ticket is
            // taken only when its slot is free, and the next run is requested
            // with the last ticket of the current one and read after the next
            // slot frees, so the atomic's round trip overlaps that wait and a
            // CTA never holds more than NSLOT + a.run tickets it has not
            // finished: few enough that a head's key sums are complete before
            // its K tiles are handed out (the lead is sized from it).
            const int run_len = a.run;
            int run = (int)atomicAdd(a.ticket, (unsigned)run_len);
            int run_next = 0;
            int in_run = 0;
            for (int i = 0;; ++i) {
                const int s = i % NSLOT;
                const uint32_t ph = (uint32_t)(i / NSLOT) & 1u;
                if (i >= NSLOT &&
                    !mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, &sm.abort_flag, a.status, kWaitLimitNs))
                    break;
                if (in_run == run_len) {
                    run = run_next;
                    in_run = 0;
                }
                const int t = run + in_run++;
                if (in_run == run_len && t < total) run_next = (int)atomicAdd(a.ticket, (unsigned)run_len);
                const uint32_t fb = smem_u32(&sm.full[s]);
                filled |= 1u << s;
                parity = (parity & ~(1u << s)) | (ph << s);
                if (t >= total) {  // no work left: every consumer sees this slot's end marker
                    sm.meta[s] = make_int4(KIND_END, 0, 0, 0);
                    mbar_arrive(fb);
                    break;
                }
                int kind, bh, tile;
                decode_ticket(t, Th, a.BH, sums, a.lead, kind, bh, tile);
                if (!FP4ATTN_IN_BOUNDS(bh >= 0 && bh < a.BH && tile >= 0 && tile < Th && kind <= KIND_K, a.status)) {
                    sm.abort_flag = 1;
                    break;
                }
                sm.meta[s] = make_int4(kind, bh, tile, 0);
                const CUtensorMap* map = (kind == KIND_Q) ? &tm_q : &tm_k;
                const uint64_t pol = (kind == KIND_KSUM) ? pol_keep : pol_stream;
                const int b = bh / a.H, h = bh - b * a.H;
                mbar_arrive_expect_tx(fb, TILE_BYTES);
                tma_load_4d_hint(smem_u32(sm.tile[s]), map, 0, tile * TILE_ROWS, h, b, fb, pol);
                tma_load_4d_hint(smem_u32(sm.tile[s]) + HALF_BYTES, map, 64, tile * TILE_ROWS, h, b, fb, pol);
            }
            // wind down: the last phase of every slot this warp armed (the end
            // marker's included) must complete, so this CTA's own copies have
            // landed before it exits; after a normal run they all have
            int dummy = 0;
            for (int s = 0; s < NSLOT; ++s)
                if (filled & (1u << s))
                    mbar_wait(smem_u32(&sm.full[s]), (parity >> s) & 1u, &dummy, nullptr, kDrainLimitNs);
        }
        return;
    }

    // -------------------------------------------------------- consumers ----
    const int h = lane & 1;                    // which half of the row this lane holds
    const int r = 16 * warp + (lane >> 1);     // row within the tile
    const float sg = h ? -1.0f : 1.0f;         // stride-32 sign: lane 0 the sum, lane 1 the difference
    const float c = __uint_as_float(0x3DB504F3u);  // fp32(1/sqrt(128))
    // lane h holds channels i in [32h, 32h+32) and i+64: its register groups
    // P[0..15] and P[16..31] are blocks 2h and 2h+1 (.x) and 2h+4, 2h+5 (.y),
    // with or without the rotation.  The selector interleaves the two lanes'
    // scale bytes (lane 0: blocks 0,1,4,5; lane 1: 2,3,6,7) into the row's.
    const int blk[4] = {2 * h, 2 * h + 1, 2 * h + 4, 2 * h + 5};
    const uint32_t ssel = h ? 0x3276u : 0x5410u;

    long long acc[4] = {0, 0, 0, 0};  // key sums of channels 4*lane..4*lane+3, not yet flushed
    int pend_bh = -1, pend_cnt = 0;
    float umax = 0.0f;
    int mean_head = -1;
    float amax_q = 0.0f, amax_k = 0.0f;  // AMAX: largest |y| of this thread's valid Q and K rows

    // Key sums: every consumer warp sees the same tiles, so the runs of
    // key-sum tiles of one head end at the same place for all of them.  At
    // the end of a run each warp adds its partial sums into the CTA's
    // shared-memory accumulator (two of them, used by alternate runs); the
    // last warp to do so moves the run's sums to the workspace with 128
    // 64-bit atomics, then a device fence and the head's count of 16-row
    // chunks.  A warp more than one run ahead waits (bounded) for its buffer.
    int runs = 0;
    auto flush = [&]() -> bool {  // warp-uniform; false after an abort
        const int b = runs & 1;
        bool ok = true;
        if (lane == 0) {
            volatile int* gen = &sm.run_gen[b];
            if (*gen != (runs >> 1)) {
                const uint64_t t0 = globaltimer_ns();
                while (*gen != (runs >> 1)) {
                    if (*reinterpret_cast<volatile int*>(&sm.abort_flag) ||
                        globaltimer_ns() - t0 > a.spin_limit_ns) {
                        set_status(a.status, FP4ATTN_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    __nanosleep(64);
                }
            }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
            sm.abort_flag = 1;
            return false;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            atomicAdd(&sm.csum[b][4 * lane + cc], static_cast<unsigned long long>(acc[cc]));
            acc[cc] = 0;
        }
        if (!(umax < kSumLimit)) set_status(a.status, FP4ATTN_ERR_RANGE);
        umax = 0.0f;
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            __threadfence_block();
            last = (atomicAdd(&sm.run_warps[b], 1) == W - 1);
        }
        if (__shfl_sync(0xffffffffu, last, 0) && FP4ATTN_IN_BOUNDS(pend_bh >= 0 && pend_bh < a.BH, a.status)) {
            __threadfence_block();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const unsigned long long v = atomicExch(&sm.csum[b][4 * lane + cc], 0ull);
                atomicAdd(reinterpret_cast<unsigned long long*>(a.ksum + (size_t)pend_bh * D + 4 * lane + cc), v);
            }
            // the warp barrier orders every lane's sums before lane 0's device
            // fence, which orders them (cumulatively) before the count
            __syncwarp();
            if (lane == 0) {
                sm.run_warps[b] = 0;
                __threadfence();
                atomicAdd(a.head_ready + pend_bh, (unsigned)(W * pend_cnt));
                __threadfence_block();
                atomicAdd(&sm.run_gen[b], 1);
            }
        }
        ++runs;
        pend_cnt = 0;
        return true;
    };

    for (int i = 0;; ++i) {
        const int s = i % NSLOT;
        const uint32_t ph = (uint32_t)(i / NSLOT) & 1u;
        const uint32_t fb = smem_u32(&sm.full[s]);
        {
            const bool ok = mbar_wait(fb, ph, &sm.abort_flag, a.status, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) break;
        }
        const int4 mt = sm.meta[s];
        if (mt.x == KIND_END) break;
        const int kind = mt.x, bh = mt.y, tile = mt.z;
        const uint8_t* tb = sm.tile[s];
        const uint32_t eb = smem_u32(&sm.empty[s]);

        if (kind == KIND_KSUM) {
            // -------------------------------------------------- key sums ----
            const uint8_t* hb = tb + (lane >> 4) * HALF_BYTES;
            const int j = (lane & 15) >> 1;
            const uint32_t in_chunk = (uint32_t)(lane & 1) * 8u;
            uint2 kw[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) kw[rr] = *reinterpret_cast<const uint2*>(hb + swz(16 * warp + rr, j) + in_chunk);
            __syncwarp();
            if (lane == 0) mbar_arrive(eb);
            // a run of another head ends here: flushed after the slot is
            // released, so the ring refills meanwhile
            if (pend_cnt && pend_bh != bh && !flush()) break;
            const float2 two24 = f2(kTwo24, kTwo24);
#pragma unroll
            for (int rr = 0; rr < 16; rr += 2) {
                const float2 a0 = __fmul2_rn(f2(bf16lo(kw[rr].x), bf16hi(kw[rr].x)), two24);
                const float2 a1 = __fmul2_rn(f2(bf16lo(kw[rr].y), bf16hi(kw[rr].y)), two24);
                const float2 b0 = __fmul2_rn(f2(bf16lo(kw[rr + 1].x), bf16hi(kw[rr + 1].x)), two24);
                const float2 b1 = __fmul2_rn(f2(bf16lo(kw[rr + 1].y), bf16hi(kw[rr + 1].y)), two24);
                acc[0] += __float2ll_rn(a0.x) + __float2ll_rn(b0.x);
                acc[1] += __float2ll_rn(a0.y) + __float2ll_rn(b0.y);
                acc[2] += __float2ll_rn(a1.x) + __float2ll_rn(b1.x);
                acc[3] += __float2ll_rn(a1.y) + __float2ll_rn(b1.y);
                umax = fmax3(umax, fmax3(fabsf(a0.x), fabsf(a0.y), fabsf(a1.x)),
                             fmax3(fabsf(a1.y), fmax3(fabsf(b0.x), fabsf(b0.y), fabsf(b1.x)), fabsf(b1.y)));
            }
            pend_bh = bh;
            ++pend_cnt;
            continue;
        }
        // with key sums (a flush or a wait for a head's means may come
        // next), the row goes into registers and the slot is released first,
        // so that neither holds a slot; without, the copy comes just before
        // the arithmetic
        uint4 rlo[4], rhi[4];
        auto load_row = [&]() {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int cj = 4 * h + j;
                rlo[j] = *reinterpret_cast<const uint4*>(tb + swz(r, cj));
                rhi[j] = *reinterpret_cast<const uint4*>(tb + HALF_BYTES + swz(r, cj));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(eb);
        };
        if constexpr (SMOOTH) load_row();
        if (pend_cnt && !flush()) break;
        const int which = kind - 1;  // 0 = Q, 1 = K
        const bool sub_mean = (which == 1) && smooth;
        if (which == 1 && mean_head != bh) {
            // ---------------------------------------------- head means ----
            float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // channels lane, lane+32, lane+64, lane+96
            if (smooth) {
                bool ready = true;
                if (lane == 0) {
                    volatile unsigned* cnt = a.head_ready + bh;
                    const unsigned need = (unsigned)(W * Th);
                    if (*cnt < need) {
                        const uint64_t t0 = globaltimer_ns();
                        while (*cnt < need) {
                            if (*reinterpret_cast<volatile int*>(&sm.abort_flag) || globaltimer_ns() - t0 > a.spin_limit_ns) {
                                set_status(a.status, FP4ATTN_ERR_TIMEOUT);
                                ready = false;
                                break;
                            }
                            __nanosleep(128);
                        }
                    }
                    __threadfence();
                }
                if (!__shfl_sync(0xffffffffu, ready, 0)) {
                    sm.abort_flag = 1;
                    break;
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const long long S = __ldcg(a.ksum + (size_t)bh * D + lane + 32 * q4);
                    m[q4] = __double2float_rn(__ddiv_rn(__ll2double_rn(S), (double)N * 16777216.0));
                }
                sm.neg_mean2[warp][lane] = f2(-m[0], -m[2]);
                sm.neg_mean2[warp][lane + 32] = f2(-m[1], -m[3]);
            }
            if (a.k_mean && tile == 0 && warp == 0) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) a.k_mean[(size_t)bh * D + lane + 32 * q4] = m[q4];
            }
            __syncwarp();
            mean_head = bh;
        }
        // ------------------------------------------------------- one row ----

        if constexpr (!SMOOTH) load_row();
        float2 P[32];
        bool finite = true;
        // chunk j (8 pairs): unpack, smooth, and the butterflies of stride
        // 1, 2, 4, which stay inside the chunk
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
                const float4* nm = reinterpret_cast<const float4*>(sm.neg_mean2[warp] + 8 * (4 * h + j));
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 m4 = nm[e];
                    C[2 * e] = __fadd2_rn(C[2 * e], f2(m4.x, m4.y));
                    C[2 * e + 1] = __fadd2_rn(C[2 * e + 1], f2(m4.z, m4.w));
                }
            }
            if (!hadamard) {
#pragma unroll
                for (int q = 0; q < 8; ++q) finite &= (fabsf(C[q].x) < INFINITY) && (fabsf(C[q].y) < INFINITY);
            } else {
#pragma unroll
                for (int st = 1; st < 8; st <<= 1) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if ((q & st) == 0) {
                            const float2 x = C[q], y = C[q + st];
                            C[q] = __fadd2_rn(x, y);
                            C[q + st] = sub2(x, y);
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
                for (int q = 0; q < 32; ++q) {
                    if ((q & st) == 0) {
                        const float2 x = P[q], y = P[q + st];
                        P[q] = __fadd2_rn(x, y);
                        P[q + st] = sub2(x, y);
                    }
                }
            }
            // stride 32 between the two lanes of the row: lane 0 keeps
            // x_i + x_{i+32}, lane 1 keeps x_i - x_{i+32}, each as
            // fl(other + sg * own), one rounding
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const float ox = __shfl_xor_sync(0xffffffffu, P[q].x, 1);
                const float oy = __shfl_xor_sync(0xffffffffu, P[q].y, 1);
                P[q] = __ffma2_rn(P[q], f2(sg, sg), f2(ox, oy));
            }
            // stride 64 inside each pair, then x fp32(1/sqrt(128))
#pragma unroll
            for (int q = 0; q < 32; ++q) P[q] = f2(__fadd_rn(P[q].x, P[q].y), __fsub_rn(P[q].x, P[q].y));
#pragma unroll
            for (int q = 0; q < 32; ++q) P[q] = __fmul2_rn(P[q], f2(c, c));
            // y_0 (lane 0, P[0].x) is c times the sum of all 128 inputs: it is
            // finite iff they all are (barring overflow of the sum itself)
            finite = (h != 0) || (fabsf(P[0].x) < INFINITY);
        }

        const bool valid = (tile * TILE_ROWS + r) < N;
        if (!finite && valid) set_status(a.status, FP4ATTN_ERR_RANGE);
        if constexpr (AMAX) {
            // rows past N hold the copy's zero fill (minus the mean for K): skip them
            if (valid) {
                float mx = 0.0f;
#pragma unroll
                for (int q = 0; q < 32; ++q) mx = fmax3(mx, fabsf(P[q].x), fabsf(P[q].y));
                if (which) amax_k = fmaxf(amax_k, mx); else amax_q = fmaxf(amax_q, mx);
            }
        } else {
            // NVFP4 pack of the lane's four blocks: group g = P[16g..16g+15],
            // its .x values form block blk[g], its .y values block blk[2+g];
            // block b's codes are bytes 8b..8b+7 of the row
            const float gw = which ? gk : gq;
            const size_t row = (size_t)bh * N + (size_t)tile * TILE_ROWS + r;
            uint8_t* crow = (which ? a.codes[1] : a.codes[0]) + row * 64;
            uint32_t sb[4];
            uint32_t wx[2][2], wy[2][2];
            if (gw == 1.0f)
                pack_blocks<true>(P, gw, sm.inv_scale, sb, wx, wy);
            else
                pack_blocks<false>(P, gw, sm.inv_scale, sb, wx, wy);
            const uint32_t mine = sb[0] | (sb[1] << 8) | (sb[2] << 16) | (sb[3] << 24);
            const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
            if (valid && FP4ATTN_IN_BOUNDS(row < (size_t)a.BH * N, a.status)) {
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    *reinterpret_cast<uint2*>(crow + 8 * blk[g]) = make_uint2(wx[g][0], wx[g][1]);
                    *reinterpret_cast<uint2*>(crow + 8 * blk[2 + g]) = make_uint2(wy[g][0], wy[g][1]);
                }
                *reinterpret_cast<uint32_t*>((which ? a.scales[1] : a.scales[0]) + row * 8 + 4 * h) =
                    prmt(mine, other, ssel);
            }
        }
    }
    if (pend_cnt) flush();
    if constexpr (AMAX) {
        // magnitudes are >= 0, so their fp32 bit patterns order like the values
        const unsigned wq = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_q));
        const unsigned wk = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_k));
        if (lane == 0) {
            if (wq) atomicMax(a.amax, wq);
            if (wk) atomicMax(a.amax + 1, wk);
        }
    }
}

size_t pro_smem_bytes() { return sizeof(ProSmem) + 1024; }

// [B][H][N][128 bf16] with element strides st: 128B-swizzled boxes of 64
// channels x TILE_ROWS rows of one head; x is 0 or 64 (0 or 128 bytes), so
// every box starts on a 16-byte boundary.  The strides must be multiples of 8
// elements.
bool make_rows_map(CUtensorMap* m, const __nv_bfloat16* base, int B, int H, int N, Strides st) {
    const uint64_t dims[4] = {128, (uint64_t)N, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)st.n * 2, (uint64_t)st.h * 2, (uint64_t)st.b * 2};
    const uint32_t box[4] = {64, TILE_ROWS, 1, 1};
    return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(base), dims,
                             strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <bool AMAX, bool HAD, bool SMOOTH>
cudaError_t launch_inst(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ProArgs& a, cudaStream_t stream) {
    static_assert(sizeof(ProSmem) + 1024 <= 227 * 1024, "shared memory budget");
    const size_t smem = pro_smem_bytes();
    const auto kernel = prologue_kernel<AMAX, HAD, SMOOTH>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, PRO_THREADS, smem)) != cudaSuccess)
        return e;
    const bool sum_tiles = !(a.flags & FP4ATTN_NO_SMOOTH_K) && !a.sums_ready && !a.withhold_sums;
    const long long tiles = (long long)a.BH * a.n_tiles * (sum_tiles ? 3 : 2);
    long long grid = (long long)sms * (per_sm > 0 ? per_sm : 1);
    if (grid > tiles) grid = tiles;
    ProArgs b = a;
    if (sum_tiles && b.lead > 0) {
        // A head's K tiles are handed out about 3 * lead * n_tiles tickets
        // after its last key-sum tile, and the CTAs hold at most
        // grid * (NSLOT + run) tickets they have not finished: the smallest
        // lead that keeps the first a quarter above the second lets no K tile
        // wait for its sums, while K is still in L2 for its second read.
        const long long held = grid * (NSLOT + b.run);
        while (b.lead < b.BH && 3LL * b.lead * b.n_tiles < held + held / 4) ++b.lead;
    }
    kernel<<<(unsigned)grid, PRO_THREADS, smem, stream>>>(tm_q, tm_k, b);
    return cudaGetLastError();
}

template <bool AMAX>
cudaError_t launch_pass(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const ProArgs& a, cudaStream_t stream) {
    const bool had = !(a.flags & FP4ATTN_NO_HADAMARD), smooth = !(a.flags & FP4ATTN_NO_SMOOTH_K);
    if (had) return smooth ? launch_inst<AMAX, true, true>(tm_q, tm_k, a, stream)
                           : launch_inst<AMAX, true, false>(tm_q, tm_k, a, stream);
    return smooth ? launch_inst<AMAX, false, true>(tm_q, tm_k, a, stream)
                  : launch_inst<AMAX, false, false>(tm_q, tm_k, a, stream);
}

__global__ void store_gscales_kernel(float* gq, float* gk) {
    *gq = tensor_gscale(0.0f);
    *gk = tensor_gscale(0.0f);
}

ProArgs base_args(const QuantArgs& q) {
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
    a.n_tiles = (q.N + TILE_ROWS - 1) / TILE_ROWS;
    a.flags = q.flags & ~QUANT_DYNAMIC_G;
    a.lead = FP4ATTN_PRO_LEAD;
    // runs of about n_tiles / 48 tiles, 1 to MAX_TICKET_RUN (the lead, set at
    // launch, grows with the tickets the CTAs can hold)
    a.run = a.n_tiles / 48;
    if (a.run < 1) a.run = 1;
    if (a.run > MAX_TICKET_RUN) a.run = MAX_TICKET_RUN;
    a.spin_limit_ns = kWaitLimitNs;
    a.status = q.status;
    return a;
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
    ProArgs a = base_args(q);
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

// Test hook: the prologue with the key-sum tiles withheld, so the first K tile
// of every head waits for sums that never arrive; the wait must give up after
// spin_limit_ns with FP4ATTN_ERR_TIMEOUT in the status word and the kernel
// must return (every CTA winds down, waiting for its own copies).
cudaError_t launch_quantize_qk_withheld_sums(const QuantArgs& q, uint64_t spin_limit_ns, cudaStream_t stream) {
    if (q.BH == 0 || q.N == 0) return cudaSuccess;
    const int B = q.BH / q.H;
    CUtensorMap tm_q, tm_k;
    if (!make_rows_map(&tm_q, q.q, B, q.H, q.N, q.qs) || !make_rows_map(&tm_k, q.k, B, q.H, q.N, q.ks))
        return cudaErrorInvalidValue;
    ProArgs a = base_args(q);
    a.flags &= ~(uint32_t)FP4ATTN_NO_SMOOTH_K;
    a.withhold_sums = true;
    a.spin_limit_ns = spin_limit_ns;
    return launch_pass<false>(tm_q, tm_k, a, stream);
}

}  // namespace fp4attn
