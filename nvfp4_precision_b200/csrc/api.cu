// C ABI of the FP4 attention library: argument validation, workspace
// handling, tensor-map encoding and kernel launches on the caller's stream.
// See include/fp4attn.h for the contract of each entry point.
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "fp4attn.h"
#include "kernels.h"

namespace fp4attn {

namespace {

constexpr int32_t kMaxN = 262144;  // 2^18: keeps |sum of k * 2^24| < 2^62 for |k| < 2^20

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// d = 128, or 64 for the entry points that take narrow heads (allow64)
int check_shape(fp4attn_shape s, bool allow64 = false) {
    if (s.B < 0 || s.H < 0 || s.N < 0 || s.D <= 0) return FP4ATTN_ERR_INVALID_ARG;
    if (s.D != D && !(allow64 && s.D == 64)) return FP4ATTN_ERR_UNSUPPORTED;
    if (s.N > kMaxN) return FP4ATTN_ERR_UNSUPPORTED;
    const int64_t bh = (int64_t)s.B * s.H;
    if (bh > 65535 || bh * (int64_t)s.N >= ((int64_t)1 << 31)) return FP4ATTN_ERR_UNSUPPORTED;
    return FP4ATTN_OK;
}

int64_t heads(fp4attn_shape s) { return (int64_t)s.B * s.H; }

// Strides of a [B,H,N,D] bf16 tensor: positive multiples of 8 elements
// (16 bytes, the tensor-copy rule) below 2^39 elements (2^40 bytes); a
// dimension of size 1 takes the contiguous stride instead of the caller's.
bool normalise_strides(fp4attn_shape s, fp4attn_strides in, Strides* out) {
    const Strides c = contiguous_strides(s.H, s.N, s.D);
    const int64_t v[3] = {s.B == 1 ? c.b : in.b, s.H == 1 ? c.h : in.h, s.N == 1 ? c.n : in.n};
    for (int64_t x : v)
        if (x <= 0 || (x & 7) || x >= ((int64_t)1 << 39)) return false;
    *out = Strides{v[0], v[1], v[2]};
    return true;
}

fp4attn_strides contiguous(fp4attn_shape s) {
    const Strides c = contiguous_strides(s.H, s.N, s.D);
    return fp4attn_strides{c.b, c.h, c.n};
}
bool empty(fp4attn_shape s) { return heads(s) == 0 || s.N == 0; }

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

int launch_status(cudaError_t e) {
    if (e == cudaSuccess) return FP4ATTN_OK;
    (void)cudaGetLastError();
    return FP4ATTN_ERR_CUDA;
}

}  // namespace

bool encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle) {
    auto fn = get_encode();
    if (!fn) return false;
    cuuint64_t gdim[5] = {0, 0, 0, 0, 0}, gstride[5] = {0, 0, 0, 0, 0};
    cuuint32_t bdim[5] = {0, 0, 0, 0, 0}, estride[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        if (i + 1 < rank) gstride[i] = strides_bytes[i];
    }
    // the strides array is always passed, even for rank 1 where it is unused
    CUresult r = fn(map, dtype, (cuuint32_t)rank, base, gdim, gstride, bdim, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS && std::getenv("FP4ATTN_DEBUG")) {
        std::fprintf(stderr, "fp4attn: cuTensorMapEncodeTiled failed (CUresult %d): dtype %d rank %d dims",
                     (int)r, (int)dtype, rank);
        for (int i = 0; i < rank; ++i) std::fprintf(stderr, " %llu", (unsigned long long)gdim[i]);
        std::fprintf(stderr, " box");
        for (int i = 0; i < rank; ++i) std::fprintf(stderr, " %u", bdim[i]);
        std::fprintf(stderr, " swizzle %d\n", (int)swizzle);
    }
    return r == CUDA_SUCCESS;
}

}  // namespace fp4attn

using namespace fp4attn;

extern "C" {

size_t fp4attn_workspace_bytes(fp4attn_shape s) {
    int64_t bh = heads(s);
    if (bh < 0) bh = 0;
    return ws_bytes(bh);
}

int fp4attn_quantize_qk_ex(const void* q, fp4attn_strides q_strides, const void* k, fp4attn_strides k_strides,
                           fp4attn_shape s, float* gq, float* gk, uint32_t flags, uint8_t* q_codes,
                           uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales, float* k_mean,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    int st = check_shape(s, true);
    if (st != FP4ATTN_OK) return st;
    if (flags & ~(uint32_t)(FP4ATTN_NO_SMOOTH_K | FP4ATTN_NO_HADAMARD | FP4ATTN_DYNAMIC_GSCALE))
        return FP4ATTN_ERR_INVALID_ARG;
    const bool dynamic = (flags & FP4ATTN_DYNAMIC_GSCALE) != 0;
    if (dynamic && s.D != D) return FP4ATTN_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < fp4attn_workspace_bytes(s) || !aligned16(workspace))
        return FP4ATTN_ERR_WORKSPACE;
    if ((gq && ((uintptr_t)gq & 3)) || (gk && ((uintptr_t)gk & 3))) return FP4ATTN_ERR_INVALID_ARG;
    if (dynamic && (!gq || !gk)) return FP4ATTN_ERR_INVALID_ARG;
    Strides qs{}, ks{};
    if (!empty(s)) {
        const void* ptrs[] = {q, k, q_codes, q_scales, k_codes, k_scales};
        for (const void* p : ptrs)
            if (!p || !aligned16(p)) return FP4ATTN_ERR_INVALID_ARG;
        if (k_mean && !aligned16(k_mean)) return FP4ATTN_ERR_INVALID_ARG;
        if (!normalise_strides(s, q_strides, &qs) || !normalise_strides(s, k_strides, &ks))
            return FP4ATTN_ERR_INVALID_ARG;
    }
    cudaError_t e = cudaMemsetAsync(workspace, 0, fp4attn_workspace_bytes(s), stream);
    if (e != cudaSuccess) return launch_status(e);
    if (empty(s)) return dynamic ? launch_status(launch_store_gscales(gq, gk, stream)) : FP4ATTN_OK;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (s.D == 64) {
        Prologue64Args b{};
        b.q = static_cast<const __nv_bfloat16*>(q);
        b.k = static_cast<const __nv_bfloat16*>(k);
        b.qs = qs;
        b.ks = ks;
        b.BH = (int)heads(s);
        b.H = s.H;
        b.N = s.N;
        b.flags = flags;
        b.gq = gq;
        b.gk = gk;
        b.q_codes = q_codes;
        b.q_scales = q_scales;
        b.k_codes = k_codes;
        b.k_scales = k_scales;
        b.k_mean = k_mean;
        b.ksum = reinterpret_cast<long long*>(ws + ws_ksum_offset());
        b.status = reinterpret_cast<int*>(ws);
        return launch_status(launch_quantize_qk64(b, stream));
    }
    QuantArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.qs = qs;
    a.ks = ks;
    a.BH = (int)heads(s);
    a.H = s.H;
    a.N = s.N;
    a.gq = dynamic ? nullptr : gq;
    a.gk = dynamic ? nullptr : gk;
    a.g_out[0] = dynamic ? gq : nullptr;
    a.g_out[1] = dynamic ? gk : nullptr;
    a.amax = reinterpret_cast<unsigned*>(ws + WS_AMAX_OFFSET);
    a.flags = (flags & ~(uint32_t)FP4ATTN_DYNAMIC_GSCALE) | (dynamic ? QUANT_DYNAMIC_G : 0u);
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.k_codes = k_codes;
    a.k_scales = k_scales;
    a.k_mean = k_mean;
    a.ksum = reinterpret_cast<long long*>(ws + ws_ksum_offset());
    a.counters = reinterpret_cast<unsigned*>(ws + ws_counter_offset(heads(s)));
    a.ticket = reinterpret_cast<unsigned*>(ws + WS_TICKET_OFFSET);
    a.status = reinterpret_cast<int*>(ws);
    return launch_status(launch_quantize_qk(a, stream));
}

int fp4attn_quantize_qk(const void* q, const void* k, fp4attn_shape s, const float* gq, const float* gk,
                        uint32_t flags, uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales,
                        float* k_mean, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (flags & FP4ATTN_DYNAMIC_GSCALE) return FP4ATTN_ERR_INVALID_ARG;  // its scale pointers are inputs
    return fp4attn_quantize_qk_ex(q, contiguous(s), k, contiguous(s), s, const_cast<float*>(gq),
                                  const_cast<float*>(gk), flags, q_codes, q_scales, k_codes, k_scales, k_mean,
                                  workspace, workspace_bytes, stream);
}

int fp4attn_forward_ex(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                       const uint8_t* k_scales, const float* gq, const float* gk, const void* v,
                       fp4attn_strides v_strides, fp4attn_shape s, float softmax_scale, void* o,
                       fp4attn_strides o_strides, float* lse, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
    int st = check_shape(s, true);
    if (st != FP4ATTN_OK) return st;
    if (!workspace || workspace_bytes < fp4attn_workspace_bytes(s) || !aligned16(workspace))
        return FP4ATTN_ERR_WORKSPACE;
    if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f) return FP4ATTN_ERR_INVALID_ARG;
    if (empty(s)) return FP4ATTN_OK;
    const void* ptrs[] = {q_codes, q_scales, k_codes, k_scales, v, o};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return FP4ATTN_ERR_INVALID_ARG;
    if (lse && ((uintptr_t)lse & 3)) return FP4ATTN_ERR_INVALID_ARG;
    FwdArgs a;
    if (!normalise_strides(s, v_strides, &a.vs) || !normalise_strides(s, o_strides, &a.os))
        return FP4ATTN_ERR_INVALID_ARG;
    a.H = s.H;
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.k_codes = k_codes;
    a.k_scales = k_scales;
    a.gq = gq;
    a.gk = gk;
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.BH = (int)heads(s);
    a.N = s.N;
    a.d = s.D;
    a.softmax_scale = softmax_scale;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.status = static_cast<int*>(workspace);
    st = launch_forward(a, stream);
    if (st != FP4ATTN_OK) (void)cudaGetLastError();
    return st;
}

int fp4attn_forward(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                    const uint8_t* k_scales, const float* gq, const float* gk, const void* v,
                    fp4attn_shape s, float softmax_scale, void* o, float* lse, void* workspace,
                    size_t workspace_bytes, cudaStream_t stream) {
    return fp4attn_forward_ex(q_codes, q_scales, k_codes, k_scales, gq, gk, v, contiguous(s), s, softmax_scale, o,
                              contiguous(s), lse, workspace, workspace_bytes, stream);
}

int fp4attn_forward_bf16qk_ex(const void* q, fp4attn_strides q_strides, const void* k, fp4attn_strides k_strides,
                              const void* v, fp4attn_strides v_strides, fp4attn_shape s, float softmax_scale,
                              void* o, fp4attn_strides o_strides, float* lse, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    int st = check_shape(s);
    if (st != FP4ATTN_OK) return st;
    if (!workspace || workspace_bytes < fp4attn_workspace_bytes(s) || !aligned16(workspace))
        return FP4ATTN_ERR_WORKSPACE;
    if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f) return FP4ATTN_ERR_INVALID_ARG;
    if (empty(s)) return FP4ATTN_OK;
    const void* ptrs[] = {q, k, v, o};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return FP4ATTN_ERR_INVALID_ARG;
    if (lse && ((uintptr_t)lse & 3)) return FP4ATTN_ERR_INVALID_ARG;
    FwdBf16Args a;
    if (!normalise_strides(s, q_strides, &a.qs) || !normalise_strides(s, k_strides, &a.ks) ||
        !normalise_strides(s, v_strides, &a.vs) || !normalise_strides(s, o_strides, &a.os))
        return FP4ATTN_ERR_INVALID_ARG;
    a.H = s.H;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.BH = (int)heads(s);
    a.N = s.N;
    a.softmax_scale = softmax_scale;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.status = static_cast<int*>(workspace);
    st = launch_forward_bf16qk(a, stream);
    if (st != FP4ATTN_OK) (void)cudaGetLastError();
    return st;
}

int fp4attn_forward_bf16qk(const void* q, const void* k, const void* v, fp4attn_shape s, float softmax_scale,
                           void* o, float* lse, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return fp4attn_forward_bf16qk_ex(q, contiguous(s), k, contiguous(s), v, contiguous(s), s, softmax_scale, o,
                                     contiguous(s), lse, workspace, workspace_bytes, stream);
}

size_t fp4attn_backward_workspace_bytes(fp4attn_shape s) {
    int64_t bh = heads(s);
    if (bh < 0) bh = 0;
    return bws_bytes(bh, s.N > 0 ? s.N : 0);
}

int fp4attn_backward_ex(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                        const uint8_t* k_scales, const float* gq, const float* gk, const void* v, const void* o,
                        const void* dout, fp4attn_strides io_strides, const float* lse, fp4attn_shape s,
                        float softmax_scale, uint32_t flags, void* dq, void* dk, void* dv, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
    int st = check_shape(s);
    if (st != FP4ATTN_OK) return st;
    if (flags & ~(uint32_t)(FP4ATTN_NO_SMOOTH_K | FP4ATTN_NO_HADAMARD)) return FP4ATTN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < fp4attn_backward_workspace_bytes(s) || !aligned16(workspace))
        return FP4ATTN_ERR_WORKSPACE;
    if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f) return FP4ATTN_ERR_INVALID_ARG;
    if (!empty(s)) {
        const void* ptrs[] = {q_codes, q_scales, k_codes, k_scales, v, o, dout, lse, dq, dk, dv};
        for (const void* p : ptrs)
            if (!p || !aligned16(p)) return FP4ATTN_ERR_INVALID_ARG;
    }
    if ((gq && ((uintptr_t)gq & 3)) || (gk && ((uintptr_t)gk & 3))) return FP4ATTN_ERR_INVALID_ARG;
    Strides io{};
    if (!empty(s) && !normalise_strides(s, io_strides, &io)) return FP4ATTN_ERR_INVALID_ARG;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t BH = heads(s);
    cudaError_t e = cudaMemsetAsync(ws, 0, WS_STATUS_BYTES, stream);
    if (e != cudaSuccess) return launch_status(e);
    if (empty(s)) return FP4ATTN_OK;
    BwdArgs a;
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.k_codes = k_codes;
    a.k_scales = k_scales;
    a.qhat = reinterpret_cast<__nv_bfloat16*>(ws + bws_qt_offset(BH, s.N));
    a.khat = reinterpret_cast<__nv_bfloat16*>(ws + bws_kt_offset(BH, s.N));
    a.gq = gq;
    a.gk = gk;
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.o = static_cast<const __nv_bfloat16*>(o);
    a.dout = static_cast<const __nv_bfloat16*>(dout);
    a.io = io;
    a.lse = lse;
    a.BH = (int)BH;
    a.H = s.H;
    a.N = s.N;
    a.softmax_scale = softmax_scale;
    a.flags = flags;
    a.dq = static_cast<__nv_bfloat16*>(dq);
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dv = static_cast<__nv_bfloat16*>(dv);
    a.dsum = reinterpret_cast<float*>(ws + bws_dsum_offset());
    a.colsum = reinterpret_cast<float*>(ws + bws_colsum_offset(BH, s.N));
    a.partial = reinterpret_cast<float*>(ws + bws_partial_offset(BH, s.N));
    a.dk_acc = reinterpret_cast<float*>(ws + bws_dk_offset(BH, s.N));
    a.status = reinterpret_cast<int*>(ws);
    st = launch_backward(a, stream);
    if (st != FP4ATTN_OK) (void)cudaGetLastError();
    return st;
}

int fp4attn_backward(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                     const uint8_t* k_scales, const float* gq, const float* gk, const void* v, const void* o,
                     const void* dout, const float* lse, fp4attn_shape s, float softmax_scale, uint32_t flags,
                     void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return fp4attn_backward_ex(q_codes, q_scales, k_codes, k_scales, gq, gk, v, o, dout, contiguous(s), lse, s,
                               softmax_scale, flags, dq, dk, dv, workspace, workspace_bytes, stream);
}

int fp4attn_dequant_bf16(const uint8_t* codes, const uint8_t* scales, const float* g, fp4attn_shape s, void* out,
                         cudaStream_t stream) {
    int st = check_shape(s, true);
    if (st != FP4ATTN_OK) return st;
    if (empty(s)) return FP4ATTN_OK;
    if (!codes || !scales || !out || !aligned16(codes) || !aligned16(out) ||
        ((uintptr_t)scales & (uintptr_t)(s.D / 16 - 1)))  // a row's scales: 8 bytes (4 for 64 channels)
        return FP4ATTN_ERR_INVALID_ARG;
    if (g && ((uintptr_t)g & 3)) return FP4ATTN_ERR_INVALID_ARG;
    return launch_status(launch_dequant_bf16(codes, scales, g, heads(s) * s.N * (s.D / 16),
                                             static_cast<__nv_bfloat16*>(out), stream));
}

int fp4attn_dequant(const uint8_t* codes, const uint8_t* scales, const float* g, fp4attn_shape s,
                    float* out, cudaStream_t stream) {
    int st = check_shape(s, true);
    if (st != FP4ATTN_OK) return st;
    if (empty(s)) return FP4ATTN_OK;
    if (!codes || !scales || !out || !aligned16(codes) || !aligned16(out) ||
        ((uintptr_t)scales & (uintptr_t)(s.D / 16 - 1)))  // a row's scales: 8 bytes (4 for 64 channels)
        return FP4ATTN_ERR_INVALID_ARG;
    return launch_status(launch_dequant(codes, scales, g, heads(s) * s.N * (s.D / 16), out, stream));
}

int fp4attn_read_status(const void* workspace, cudaStream_t stream, int* device_status) {
    if (!workspace || !device_status) return FP4ATTN_ERR_INVALID_ARG;
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return launch_status(e);
    *device_status = v;
    return FP4ATTN_OK;
}

int fp4attn_reset_status(void* workspace, cudaStream_t stream) {
    if (!workspace) return FP4ATTN_ERR_INVALID_ARG;
    return launch_status(cudaMemsetAsync(workspace, 0, sizeof(int), stream));
}

const char* fp4attn_status_string(int code) {
    switch (code) {
        case FP4ATTN_OK: return "ok";
        case FP4ATTN_ERR_INVALID_ARG: return "invalid argument";
        case FP4ATTN_ERR_UNSUPPORTED: return "unsupported shape or option";
        case FP4ATTN_ERR_CUDA: return "CUDA call failed";
        case FP4ATTN_ERR_RANGE: return "input out of range (non-finite value, |k| >= 2^20 or bad global scale)";
        case FP4ATTN_ERR_TIMEOUT: return "a bounded device wait ran out";
        case FP4ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        default: return "unknown status";
    }
}

int fp4attn_encode_f32(const float* x, int64_t n, uint8_t* e2m1, uint8_t* e4m3, cudaStream_t stream) {
    if (n < 0 || (n > 0 && !x)) return FP4ATTN_ERR_INVALID_ARG;
    return launch_status(launch_encode_f32(x, n, e2m1, e4m3, stream));
}

int fp4attn_probe_qk_tile(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                          float* s_out, cudaStream_t stream) {
    const void* ptrs[] = {qc, qs, kc, ks, s_out};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return FP4ATTN_ERR_INVALID_ARG;
    int st = launch_probe_qk(qc, qs, kc, ks, s_out, stream);
    if (st != FP4ATTN_OK) (void)cudaGetLastError();
    return st;
}

int fp4attn_probe_pv_tile(const void* p, const void* v, float* o_out, cudaStream_t stream) {
    if (!p || !v || !o_out || !aligned16(p) || !aligned16(v) || !aligned16(o_out))
        return FP4ATTN_ERR_INVALID_ARG;
    int st = launch_probe_pv(static_cast<const __nv_bfloat16*>(p), static_cast<const __nv_bfloat16*>(v),
                             o_out, stream);
    if (st != FP4ATTN_OK) (void)cudaGetLastError();
    return st;
}

int fp4attn_probe_div6(uint32_t* result, cudaStream_t stream) {
    if (!result || ((uintptr_t)result & 3)) return FP4ATTN_ERR_INVALID_ARG;
    uint32_t init[2] = {0u, 0xFFFFFFFFu};
    cudaError_t e = cudaMemcpyAsync(result, init, sizeof init, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = launch_div6_check(result, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    return launch_status(e);
}

int fp4attn_probe_mma_rate(int mode, int reps, long long* cycles, int* status, cudaStream_t stream) {
    if ((mode != 0 && mode != 1) || reps < 1 || reps > 1000000 || !cycles || ((uintptr_t)cycles & 7) || !status ||
        ((uintptr_t)status & 3))
        return FP4ATTN_ERR_INVALID_ARG;
    return launch_status(launch_mma_rate(mode, reps, cycles, status, stream));
}

int fp4attn_probe_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t stream) {
    if (!status || limit_ns > 10000000000ull) return FP4ATTN_ERR_INVALID_ARG;
    return launch_probe_wait_timeout(status, limit_ns, stream);
}

int fp4attn_probe_withheld_key_sums(const void* q, const void* k, fp4attn_shape s, uint8_t* q_codes,
                                    uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales, void* workspace,
                                    size_t workspace_bytes, uint64_t limit_ns, cudaStream_t stream) {
    int st = check_shape(s);
    if (st != FP4ATTN_OK) return st;
    if (empty(s) || limit_ns > 10000000000ull) return FP4ATTN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < fp4attn_workspace_bytes(s) || !aligned16(workspace))
        return FP4ATTN_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, q_codes, q_scales, k_codes, k_scales};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return FP4ATTN_ERR_INVALID_ARG;
    cudaError_t e = cudaMemsetAsync(workspace, 0, fp4attn_workspace_bytes(s), stream);
    if (e != cudaSuccess) return launch_status(e);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    QuantArgs a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.qs = a.ks = contiguous_strides(s.H, s.N);
    a.BH = (int)heads(s);
    a.H = s.H;
    a.N = s.N;
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.k_codes = k_codes;
    a.k_scales = k_scales;
    a.ksum = reinterpret_cast<long long*>(ws + ws_ksum_offset());
    a.counters = reinterpret_cast<unsigned*>(ws + ws_counter_offset(heads(s)));
    a.ticket = reinterpret_cast<unsigned*>(ws + WS_TICKET_OFFSET);
    a.status = reinterpret_cast<int*>(ws);
    return launch_status(launch_quantize_qk_withheld_sums(a, limit_ns, stream));
}

}  // extern "C"
