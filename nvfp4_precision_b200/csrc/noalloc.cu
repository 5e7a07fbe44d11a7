// fp4attn_quantize_qk_noalloc: the quantisation prologue for callers that
// cannot allocate device memory.
//
// The prologue needs a little scratch memory (a status word, a tile ticket,
// per-head int64 key sums and ready counters).  fp4attn_quantize_qk takes it
// from a caller-provided workspace.  Some callers have no way to provide one:
// cudaMalloc/cudaFree may synchronise the whole device, which a latency-bound
// caller (a serving loop sharing the GPU with other streams) cannot afford,
// and some callers run where another allocator owns the device memory budget
// and raw allocations are not allowed.  This variant uses a fixed scratch
// array in the library's own device memory instead: every GPU that loads the
// library holds it (about 1 MB) until the process exits.
#include <cuda_runtime_api.h>

#include <mutex>

#include "fp4attn.h"
#include "kernels.h"

namespace fp4attn {
namespace {

constexpr int kNoAllocMaxHeads = 1024;  // B * H limit of the variant
constexpr size_t kNoAllocScratchBytes = (WS_STATUS_BYTES + (size_t)kNoAllocMaxHeads * D * 8 +
                                         (size_t)kNoAllocMaxHeads * 4 + 255) / 256 * 256;

// The scratch itself.  Host code must not pass this symbol to a kernel: on the
// host it is only a stand-in, so its device address is looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached for the life of the
// process.  The cache does not survive a teardown of the device's primary
// context (cudaDeviceReset): the module, and the array with it, may then be
// loaded at another address.
int scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return FP4ATTN_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return FP4ATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_dev[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return FP4ATTN_ERR_CUDA;
        }
        g_scratch_dev[dev] = p;
    }
    *out = g_scratch_dev[dev];
    return FP4ATTN_OK;
}

}  // namespace
}  // namespace fp4attn

using namespace fp4attn;

extern "C" int fp4attn_quantize_qk_noalloc(const void* q_bf16, const void* k_bf16, fp4attn_shape s,
                                           const float* q_gscale, const float* k_gscale, uint32_t flags,
                                           uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes,
                                           uint8_t* k_scales, float* k_mean, int* status_dev,
                                           cudaStream_t stream) {
    // reject shapes whose key sums do not fit the fixed scratch, before any CUDA call
    if (s.B > 0 && s.H > 0 && (int64_t)s.B * s.H > kNoAllocMaxHeads) return FP4ATTN_ERR_UNSUPPORTED;
    if (fp4attn_workspace_bytes(s) > kNoAllocScratchBytes) return FP4ATTN_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    int st = scratch_on_current_device(&scratch);
    if (st != FP4ATTN_OK) return st;
    // the existing entry point validates the arguments, clears the scratch it
    // uses (status, ticket, key sums, counters) on the stream, and launches
    st = fp4attn_quantize_qk(q_bf16, k_bf16, s, q_gscale, k_gscale, flags, q_codes, q_scales, k_codes, k_scales,
                             k_mean, scratch, kNoAllocScratchBytes, stream);
    if (st != FP4ATTN_OK) return st;
    if (status_dev) {
        if (cudaMemcpyAsync(status_dev, scratch, sizeof(int), cudaMemcpyDeviceToDevice, stream) != cudaSuccess) {
            (void)cudaGetLastError();
            return FP4ATTN_ERR_CUDA;
        }
    }
    return FP4ATTN_OK;
}
