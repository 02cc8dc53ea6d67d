// sikv_sparse_attn_static: sparse attention for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc at all, so they cannot provide the
// workspace that sikv_sparse_attn takes.  Examples: a serving engine whose
// device memory is carved up once at start-up and may not grow inside the
// decode loop, or a plugin host that hands a kernel only its input and output
// buffers.  This entry point runs the same attention kernels, but their
// scratch (the split-k partials and the device status word) lives in a
// fixed-size array compiled into the library, so the call allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.  Host code
// cannot use the variable's name as a device address (it is only a host-side
// handle), so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current, and caches it.
#include <mutex>

#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attn_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device (looked up once per
// device).  Returns nullptr and sets *err when the lookup fails.
void *scratch_address(cudaError_t *err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        *err = cudaGetSymbolAddress(&ptr, g_attn_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" sikv_status sikv_sparse_attn_static(const sikv_params *p, const void *q, const void *K,
                                               const void *V, const uint8_t *codes, const float *codebook,
                                               const float *mu, const int32_t *idx, const int32_t *k_per_seq,
                                               const int32_t *seq_lens, void *out, int32_t *device_flags,
                                               sikv_stream_t stream) {
    using namespace sikv;
    // Same parameter rules as sikv_sparse_attn (its workspace-size function
    // returns 0 for any invalid or unsupported parameters).
    if (sikv_sparse_attn_workspace_size(p) == 0) return SIKV_ERR_INVALID_ARG;
    const uintptr_t align_mask = 15u;
    if (!q || !K || !V || !codes || !codebook || !mu || !k_per_seq || !seq_lens || !out) return SIKV_ERR_INVALID_ARG;
    if (p->max_topk > 0 && !idx) return SIKV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) |
         reinterpret_cast<uintptr_t>(codes) | reinterpret_cast<uintptr_t>(codebook) |
         reinterpret_cast<uintptr_t>(mu) | reinterpret_cast<uintptr_t>(out)) & align_mask)
        return SIKV_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(k_per_seq) |
         reinterpret_cast<uintptr_t>(seq_lens) | reinterpret_cast<uintptr_t>(device_flags)) & 3u)
        return SIKV_ERR_UNSUPPORTED;
    // The partials must fit in the fixed array.
    if (attn_layout(*p, kHeaderBytes).total > kStaticScratchBytes) return SIKV_ERR_WORKSPACE;

    cudaError_t err = cudaSuccess;
    char *scratch = static_cast<char *>(scratch_address(&err));
    if (!scratch) return SIKV_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t *status = reinterpret_cast<int32_t *>(scratch);
    // The array keeps the previous call's contents: only the status word has
    // to start at zero (every partial the kernels read is written first).
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return SIKV_ERR_CUDA;
    const sikv_status st = launch_sparse_attn(*p, q, K, V, nullptr, codes, codebook, mu, idx, k_per_seq, seq_lens, out,
                                              scratch, kHeaderBytes, status, s);
    if (st != SIKV_OK) return st;
    if (device_flags &&
        cudaMemcpyAsync(device_flags, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return SIKV_ERR_CUDA;
    return SIKV_OK;
}
