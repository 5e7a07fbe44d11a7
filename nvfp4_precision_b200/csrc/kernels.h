// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime_api.h>

namespace fp4attn {

constexpr int D = 128;

// Bounds-checked build (-DFP4ATTN_BOUNDS_CHECK): the kernels test each global
// store, atomic and tile coordinate against the sizes of their buffers; a
// failed test records FP4ATTN_ERR_RANGE in the status word and skips the
// access instead of touching memory it does not own.  Without the macro
// every check is the constant true and compiles away.
#ifdef FP4ATTN_BOUNDS_CHECK
#define FP4ATTN_IN_BOUNDS(cond, status)                                                   \
    ((cond) ? true : (((status) ? (void)atomicCAS((status), 0, (int)FP4ATTN_ERR_RANGE) : (void)0), false))
#else
#define FP4ATTN_IN_BOUNDS(cond, status) true
#endif

// Workspace layout: [0,4) status word, [64,68) and [68,72) tile ticket
// counters of the two prologue launches, [128,136) fp32 bit patterns of the
// transformed amax of Q and K (dynamic global scales), rest of [0,256) spare;
// [256, 256 + 8*BH*128) int64 key column sums; then one uint32 per head
// (key-sum tiles completed).
constexpr size_t WS_STATUS_BYTES = 256;
constexpr size_t WS_TICKET_OFFSET = 64;
constexpr size_t WS_AMAX_OFFSET = 128;
inline size_t ws_ksum_offset() { return WS_STATUS_BYTES; }
inline size_t ws_counter_offset(int64_t BH) { return WS_STATUS_BYTES + (size_t)BH * D * 8; }
inline size_t ws_bytes(int64_t BH) {
    size_t b = ws_counter_offset(BH) + (size_t)BH * 4;
    return (b + 255) / 256 * 256;
}

// Element strides of a [B,H,N,128] bf16 tensor (the channel stride is 1).
struct Strides {
    int64_t b, h, n;
};
inline Strides contiguous_strides(int H, int N, int d = D) {
    return Strides{(int64_t)H * N * d, (int64_t)N * d, (int64_t)d};
}

// Flag of QuantArgs: compute g of Q and K from the transformed amax.
constexpr uint32_t QUANT_DYNAMIC_G = 4u;

struct QuantArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    Strides qs, ks;
    int BH, H, N;
    const float* gq;  // device scalar or nullptr (1.0); ignored with QUANT_DYNAMIC_G
    const float* gk;
    float* g_out[2];  // QUANT_DYNAMIC_G: receive the computed g of Q and K
    unsigned* amax;   // QUANT_DYNAMIC_G: two zeroed words (fp32 bits of the amax)
    uint32_t flags;
    uint8_t* q_codes;
    uint8_t* q_scales;
    uint8_t* k_codes;
    uint8_t* k_scales;
    float* k_mean;  // may be nullptr
    long long* ksum;
    unsigned* counters;
    unsigned* ticket;
    int* status;
};

cudaError_t launch_quantize_qk(const QuantArgs& a, cudaStream_t stream);

// Heads of 64 channels (codes [B,H,N,32], scales [B,H,N,4], key mean [B,H,64]);
// static global scales only.  The key sums use the first 64 slots of each
// head's 128 in the workspace.
struct Prologue64Args {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    Strides qs, ks;
    int BH, H, N;
    uint32_t flags;
    const float* gq;
    const float* gk;
    uint8_t* q_codes;
    uint8_t* q_scales;
    uint8_t* k_codes;
    uint8_t* k_scales;
    float* k_mean;
    long long* ksum;
    int* status;
};
cudaError_t launch_quantize_qk64(const Prologue64Args& a, cudaStream_t stream);
// Test hook: the prologue with its key-sum tiles withheld (K tiles time out).
cudaError_t launch_quantize_qk_withheld_sums(const QuantArgs& a, uint64_t spin_limit_ns, cudaStream_t stream);
// Dynamic global scales of empty tensors (amax 0): store the smallest g, 2^-64.
cudaError_t launch_store_gscales(float* gq, float* gk, cudaStream_t stream);

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t nblocks,
                           float* out, cudaStream_t stream);
cudaError_t launch_div6_check(unsigned* res, cudaStream_t stream);
cudaError_t launch_mma_rate(int mode, int reps, long long* cycles, int* status, cudaStream_t stream);
cudaError_t launch_encode_f32(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                              cudaStream_t stream);

// Tensor-map encoder (driver entry point cuTensorMapEncodeTiled, looked up at
// run time so the library needs no link to libcuda).
bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

struct FwdArgs {
    const uint8_t* q_codes;
    const uint8_t* q_scales;
    const uint8_t* k_codes;
    const uint8_t* k_scales;
    const float* gq;
    const float* gk;
    const __nv_bfloat16* v;
    Strides vs, os;
    int BH, H, N;
    int d;  // 128, or 64: codes [.., 32], scales [.., 4], V and O [.., 64]
    float softmax_scale;
    __nv_bfloat16* o;
    float* lse;
    int* status;
};

struct FwdBf16Args {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    Strides qs, ks, vs, os;
    int BH, H, N;
    float softmax_scale;
    __nv_bfloat16* o;
    float* lse;
    int* status;
};

// Backward workspace: [0,256) status word and spare; then D [BH*N] fp32,
// column sums [BH*128] fp32, per-warp column sums [BH*ceil(N/128)*4*128] fp32,
// scale * dK^ [BH*N*128] fp32, unit-scale Q~ and K~ [BH*N*128] bf16 each
// (each 256-aligned).
inline size_t bws_align(size_t b) { return (b + 255) / 256 * 256; }
inline size_t bws_dsum_offset() { return WS_STATUS_BYTES; }
inline size_t bws_colsum_offset(int64_t BH, int64_t N) { return bws_dsum_offset() + bws_align((size_t)(BH * N) * 4); }
inline size_t bws_partial_offset(int64_t BH, int64_t N) {
    return bws_colsum_offset(BH, N) + bws_align((size_t)BH * D * 4);
}
inline size_t bws_dk_offset(int64_t BH, int64_t N) {
    return bws_partial_offset(BH, N) + bws_align((size_t)BH * ((N + 127) / 128) * 4 * D * 4);
}
inline size_t bws_qt_offset(int64_t BH, int64_t N) { return bws_dk_offset(BH, N) + bws_align((size_t)(BH * N) * D * 4); }
inline size_t bws_kt_offset(int64_t BH, int64_t N) { return bws_qt_offset(BH, N) + bws_align((size_t)(BH * N) * D * 2); }
inline size_t bws_bytes(int64_t BH, int64_t N) { return bws_kt_offset(BH, N) + bws_align((size_t)(BH * N) * D * 2); }

struct BwdArgs {
    const uint8_t* q_codes;     // the forward's NVFP4 Q and K ([B,H,N,64] codes, [B,H,N,8] scales)
    const uint8_t* q_scales;
    const uint8_t* k_codes;
    const uint8_t* k_scales;
    __nv_bfloat16* qhat;        // workspace: unit-scale dequantised Q and K, [B,H,N,128]
    __nv_bfloat16* khat;
    const float* gq;            // global scales (device scalars) or nullptr for 1
    const float* gk;
    const __nv_bfloat16* v;
    const __nv_bfloat16* o;
    const __nv_bfloat16* dout;
    Strides io;        // element strides of v, o, dout, dq, dk, dv
    const float* lse;  // [B,H,N]
    int BH, H, N;
    float softmax_scale;
    uint32_t flags;  // FP4ATTN_NO_SMOOTH_K / FP4ATTN_NO_HADAMARD of the forward
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* dsum;
    float* colsum;
    float* partial;
    float* dk_acc;
    int* status;
};

// Returns 0 on success, else an fp4attn_status code.
int launch_backward(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_dequant_bf16(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t nblocks,
                                __nv_bfloat16* out, cudaStream_t stream);
int launch_forward(const FwdArgs& a, cudaStream_t stream);
int launch_forward_bf16qk(const FwdBf16Args& a, cudaStream_t stream);
int launch_probe_qk(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                    float* s_out, cudaStream_t stream);
int launch_probe_pv(const __nv_bfloat16* p, const __nv_bfloat16* v, float* o_out,
                    cudaStream_t stream);
int launch_probe_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t stream);

}  // namespace fp4attn
