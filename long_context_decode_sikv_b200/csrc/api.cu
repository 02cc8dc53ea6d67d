// Public C ABI of libsikv: argument validation, workspace sizing and the
// entry points declared in sikv.h.
#include <math.h>
#include <string.h>

#include "sikv_common.cuh"
#include "sikv_internal.h"

using namespace sikv;

namespace {

constexpr int32_t kVersion = 100;   // 0.1.0

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

sikv_status check_params(const sikv_params *p) {
    if (!p) return SIKV_ERR_INVALID_ARG;
    if (p->dtype != SIKV_DTYPE_F32 && p->dtype != SIKV_DTYPE_BF16) return SIKV_ERR_UNSUPPORTED;
    if (p->head_dim != kHeadDim) return SIKV_ERR_UNSUPPORTED;
    if (p->batch < 1 || p->num_kv_heads < 1 || p->num_q_heads < 1) return SIKV_ERR_INVALID_ARG;
    if (p->num_q_heads % p->num_kv_heads != 0) return SIKV_ERR_INVALID_ARG;
    if (p->num_q_heads / p->num_kv_heads > kMaxGroup) return SIKV_ERR_UNSUPPORTED;
    if (p->max_seq_len < 1 || p->num_sinks < 0 || p->max_topk < 0) return SIKV_ERR_INVALID_ARG;
    if (p->reserved[0] || p->reserved[1] || p->reserved[2]) return SIKV_ERR_INVALID_ARG;
    if (!(p->softmax_scale <= 0.f || isfinite(p->softmax_scale))) return SIKV_ERR_INVALID_ARG;
    const long long segs = static_cast<long long>(p->batch) * p->num_kv_heads;
    if (segs > 65535) return SIKV_ERR_UNSUPPORTED;                      // grid.y limit
    if (static_cast<long long>(p->max_seq_len) > (1ll << 30)) return SIKV_ERR_UNSUPPORTED;
    if (static_cast<long long>(p->num_sinks) + p->max_topk > (1ll << 30)) return SIKV_ERR_UNSUPPORTED;
    return SIKV_OK;
}

sikv_status check_ws(void *ws, size_t bytes, size_t need) {
    if (!ws) return SIKV_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SIKV_ERR_WORKSPACE;
    if (bytes < need) return SIKV_ERR_WORKSPACE;
    return SIKV_OK;
}

#define SIKV_TRY(expr)                        \
    do {                                      \
        const sikv_status _st = (expr);       \
        if (_st != SIKV_OK) return _st;       \
    } while (0)

#define SIKV_REQUIRE_PTR(ptr)                                   \
    do {                                                        \
        if (!(ptr)) return SIKV_ERR_INVALID_ARG;                \
        if (!aligned16(ptr)) return SIKV_ERR_UNSUPPORTED;       \
    } while (0)

#define SIKV_REQUIRE_PTR4(ptr)                                      \
    do {                                                            \
        if (!(ptr)) return SIKV_ERR_INVALID_ARG;                    \
        if ((reinterpret_cast<uintptr_t>(ptr) & 3u) != 0)           \
            return SIKV_ERR_UNSUPPORTED;                            \
    } while (0)

}  // namespace

namespace sikv {

DecodeLayout decode_layout(const sikv_params &p) {
    DecodeLayout L;
    const size_t segs = static_cast<size_t>(p.batch) * p.num_kv_heads;
    size_t off = kHeaderBytes;
    L.scores = off;
    off = align_up(off + segs * p.max_seq_len * sizeof(float), 256);
    L.idx = off;
    off = align_up(off + segs * (p.max_topk > 0 ? p.max_topk : 1) * sizeof(int32_t), 256);
    L.attn = off;
    L.a = attn_layout(p, off);
    L.fused = L.a.total;
    L.total = fused_layout(p, L.fused).total;
    return L;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace sikv

extern "C" {

int32_t sikv_version(void) { return kVersion; }

const char *sikv_status_string(sikv_status status) {
    switch (status) {
        case SIKV_OK: return "SIKV_OK";
        case SIKV_ERR_INVALID_ARG: return "SIKV_ERR_INVALID_ARG: null pointer, bad shape or size";
        case SIKV_ERR_UNSUPPORTED: return "SIKV_ERR_UNSUPPORTED: head_dim, group size, dtype or alignment not supported";
        case SIKV_ERR_WORKSPACE: return "SIKV_ERR_WORKSPACE: workspace null, not 256-byte aligned or too small";
        case SIKV_ERR_CUDA: return "SIKV_ERR_CUDA: a CUDA call or kernel launch failed";
        case SIKV_ERR_DEVICE: return "SIKV_ERR_DEVICE: a device-side check failed (see the status word)";
    }
    return "SIKV_ERR_UNKNOWN";
}

sikv_status sikv_workspace_init(void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_ws(workspace, workspace_bytes, kHeaderBytes));
    return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SIKV_OK
               : SIKV_ERR_CUDA;
}

sikv_status sikv_check_device_status(void *workspace, size_t workspace_bytes, sikv_stream_t stream,
                                     int32_t *device_flags) {
    SIKV_TRY(check_ws(workspace, workspace_bytes, kHeaderBytes));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t flags = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SIKV_ERR_CUDA;
    if (cudaMemcpy(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess) return SIKV_ERR_CUDA;
    if (flags != 0 && cudaMemset(workspace, 0, sizeof(flags)) != cudaSuccess) return SIKV_ERR_CUDA;
    if (device_flags) *device_flags = flags;
    return flags ? SIKV_ERR_DEVICE : SIKV_OK;
}

size_t sikv_encode_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return encode_layout(*p).total;
}

size_t sikv_score_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return kHeaderBytes;
}

size_t sikv_topk_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return topk_layout(*p).total;
}

size_t sikv_sparse_attn_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return attn_layout(*p, kHeaderBytes).total;
}

size_t sikv_decode_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return decode_layout(*p).total;
}

int32_t sikv_decode_launches(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    if (fused_plan(*p).ok) return 1;               // one cooperative kernel
    return 1 + (p->max_topk > 0 ? 1 : 0) + 2;     // score, top-k, attention partials + combine
}

sikv_status sikv_encode_keys(const sikv_params *p, const void *K, const int32_t *seq_lens, float *mu,
                             uint8_t *codes, float *codebook, int32_t *counts, void *workspace,
                             size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    if (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)) return SIKV_ERR_UNSUPPORTED;
    SIKV_TRY(check_ws(workspace, workspace_bytes, encode_layout(*p).total));
    return launch_encode(*p, K, seq_lens, mu, codes, codebook, counts, static_cast<char *>(workspace),
                         reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_score(const sikv_params *p, const void *q, const uint8_t *codes, const float *codebook,
                       const float *mu, const int32_t *seq_lens, float *scores, void *workspace,
                       size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR4(scores);
    SIKV_TRY(check_ws(workspace, workspace_bytes, kHeaderBytes));
    return launch_score(*p, q, codes, codebook, mu, seq_lens, scores, static_cast<int32_t *>(workspace),
                        reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_topk(const sikv_params *p, const float *scores, const int32_t *seq_lens,
                      const int32_t *k_per_seq, int32_t *idx, void *workspace, size_t workspace_bytes,
                      sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR4(scores);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR4(k_per_seq);
    if (p->max_topk > 0) SIKV_REQUIRE_PTR4(idx);
    SIKV_TRY(check_ws(workspace, workspace_bytes, topk_layout(*p).total));
    if (p->max_topk == 0 && !idx) return SIKV_OK;
    return launch_topk(*p, scores, seq_lens, k_per_seq, idx, static_cast<int32_t *>(workspace),
                       reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_sparse_attn(const sikv_params *p, const void *q, const void *K, const void *V,
                             const uint8_t *codes, const float *codebook, const float *mu,
                             const int32_t *idx, const int32_t *k_per_seq, const int32_t *seq_lens,
                             void *out, void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    SIKV_REQUIRE_PTR(mu);
    if (p->max_topk > 0) SIKV_REQUIRE_PTR4(idx);
    SIKV_REQUIRE_PTR4(k_per_seq);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR(out);
    SIKV_TRY(check_ws(workspace, workspace_bytes, attn_layout(*p, kHeaderBytes).total));
    return launch_sparse_attn(*p, q, K, V, codes, codebook, mu, idx, k_per_seq, seq_lens, out,
                              static_cast<char *>(workspace), kHeaderBytes, static_cast<int32_t *>(workspace),
                              reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_decode(const sikv_params *p, const void *q, const void *K, const void *V,
                        const uint8_t *codes, const float *codebook, const float *mu,
                        const int32_t *seq_lens, const int32_t *k_per_seq, void *out, int32_t *idx_out,
                        float *scores_out, void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR4(k_per_seq);
    SIKV_REQUIRE_PTR(out);
    if (idx_out) SIKV_REQUIRE_PTR4(idx_out);
    if (scores_out) SIKV_REQUIRE_PTR4(scores_out);
    const DecodeLayout L = decode_layout(*p);
    SIKV_TRY(check_ws(workspace, workspace_bytes, L.total));
    char *ws = static_cast<char *>(workspace);
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const FusedPlan plan = fused_plan(*p);
    if (plan.ok)
        return launch_decode_fused(*p, plan, q, K, V, codes, codebook, mu, seq_lens, k_per_seq, out, idx_out,
                                   scores_out, ws, L.fused, status, s);
    float *sc = scores_out ? scores_out : reinterpret_cast<float *>(ws + L.scores);
    int32_t *ix = idx_out ? idx_out : reinterpret_cast<int32_t *>(ws + L.idx);
    SIKV_TRY(launch_score(*p, q, codes, codebook, mu, seq_lens, sc, status, s));
    if (p->max_topk > 0) SIKV_TRY(launch_topk(*p, sc, seq_lens, k_per_seq, ix, status, s));
    return launch_sparse_attn(*p, q, K, V, codes, codebook, mu, ix, k_per_seq, seq_lens, out, ws, L.attn,
                              status, s);
}

}  // extern "C"
