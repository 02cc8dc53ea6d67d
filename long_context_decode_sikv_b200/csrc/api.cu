// Public C ABI of libsikv: argument validation, workspace sizing and the
// entry points declared in sikv.h.
#include <math.h>
#include <atomic>
#include <string.h>

#include <new>
#include <vector>

#include "sikv_common.cuh"
#include "sikv_internal.h"

using namespace sikv;

// A captured host-facing decode step (sikv_decode_host_plan_*): the graph
// [query copy -> decode kernels -> output copy] on the plan's workspace, and
// the two copy nodes that each run re-points.
struct sikv_host_plan {
    sikv_params p;
    const void *K, *V;
    const uint8_t *codes;
    const float *codebook, *mu;
    const int32_t *seq_lens, *k_per_seq;
    char *ws;
    size_t ws_bytes;
    uint4 *q_slot, *out_slot;           // the workspace's device copies of q and of the output
    int n16;                            // 16-byte words of one q (= one output) tensor
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    cudaGraphNode_t up, down;
    cudaKernelNodeParams up_kp, down_kp;
};

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
    if (p->decode_path < SIKV_DECODE_AUTO || p->decode_path > SIKV_DECODE_COMPOSED) return SIKV_ERR_INVALID_ARG;
    if (p->reserved[0] || p->reserved[1]) return SIKV_ERR_INVALID_ARG;
    if (!(p->softmax_scale <= 0.f || isfinite(p->softmax_scale))) return SIKV_ERR_INVALID_ARG;
    const long long segs = static_cast<long long>(p->batch) * p->num_kv_heads;
    if (segs > 65535) return SIKV_ERR_UNSUPPORTED;                      // grid.y limit
    if (static_cast<long long>(p->max_seq_len) > (1ll << 30)) return SIKV_ERR_UNSUPPORTED;
    if (static_cast<long long>(p->num_sinks) + p->max_topk > (1ll << 30)) return SIKV_ERR_UNSUPPORTED;
    return SIKV_OK;
}

// The kernels a decode step runs (sikv_decode_path; 0 when a forced path
// does not apply).  The automatic choice follows measurements on B200: the
// cooperative kernel when one launch covers the batch, except for segments
// that a cluster of at most two CTAs covers (short contexts); the cluster
// kernel when the cooperative one would need several launches (large ragged
// batches); the three composed kernels otherwise.
int resolve_decode_path(const sikv_params &p, bool vq) {
    const int path = p.decode_path;
    if (path == SIKV_DECODE_CLUSTER) return cluster_plan(p, vq).ok ? SIKV_DECODE_CLUSTER : 0;
    if (path == SIKV_DECODE_COOPERATIVE)
        return (fused_plan(p, vq).ok || fused_sub_batch(p, vq) > 0) ? SIKV_DECODE_COOPERATIVE : 0;
    if (path == SIKV_DECODE_COMPOSED) return SIKV_DECODE_COMPOSED;
    const ClusterPlan cp = cluster_plan(p, vq);
    const bool single = fused_plan(p, vq).ok;
    if (single && !(cp.ok && cp.csize <= 2)) return SIKV_DECODE_COOPERATIVE;
    if (cp.ok) return SIKV_DECODE_CLUSTER;
    if (fused_sub_batch(p, vq) > 0) return SIKV_DECODE_COOPERATIVE;
    return SIKV_DECODE_COMPOSED;
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
    // per device, 0 until first asked; concurrent first calls store the same value
    static std::atomic<int> cached[64];
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Workspace of sikv_decode_host: the decode workspace, then the device copies
// of the query and of the output.
struct HostLayout {
    size_t bytes = 0, q = 0, out = 0, total = 0;   // bytes: one query (= one output) tensor
};

HostLayout host_layout(const sikv_params &p, size_t decode_total) {
    HostLayout H;
    const size_t eb = p.dtype == SIKV_DTYPE_F32 ? 4 : 2;
    H.bytes = static_cast<size_t>(p.batch) * p.num_q_heads * p.head_dim * eb;
    H.q = align_up(decode_total, 256);
    H.out = align_up(H.q + H.bytes, 256);
    H.total = align_up(H.out + H.bytes, 256);
    return H;
}

// Copies n16 16-byte words between host-mapped and device memory: each word
// crosses the host link once, and a warp moves 512 contiguous bytes.
__global__ void __launch_bounds__(256) copy16_kernel(const uint4 *src, uint4 *dst, int n16) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += gridDim.x * blockDim.x) dst[i] = src[i];
}

int copy16_grid(int n16) { return std::min((n16 + 255) / 256, 64); }

// The device address of a page-locked host buffer, or null for pageable
// memory (which then goes through a staged copy).
void *device_view(const void *host) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
    return at.devicePointer;
}

// One decode step on device buffers (arguments checked here, except q and
// out, which the callers check).
sikv_status decode_step(const sikv_params &pp, const void *q, const void *K, const void *V, const uint8_t *vq,
                        const uint8_t *codes, const float *codebook, const float *mu, const int32_t *seq_lens,
                        const int32_t *k_per_seq, void *out, int32_t *idx_out, float *scores_out, void *workspace,
                        size_t workspace_bytes, cudaStream_t s) {
    const sikv_params *p = &pp;
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR4(k_per_seq);
    const DecodeLayout L = decode_layout(*p);
    SIKV_TRY(check_ws(workspace, workspace_bytes, L.total));
    char *ws = static_cast<char *>(workspace);
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    const bool qv = vq != nullptr;
    const int path = resolve_decode_path(*p, qv);
    if (path == 0) return SIKV_ERR_UNSUPPORTED;
    if (path == SIKV_DECODE_CLUSTER) {
        const ClusterPlan cp = cluster_plan(*p, qv);
        if (cp.ok) {
            const FusedLayout FL = fused_layout(*p, L.fused);
            return launch_decode_cluster(*p, cp, q, K, V, vq, codes, codebook, mu, seq_lens, k_per_seq, out, idx_out,
                                         scores_out, reinterpret_cast<uint2 *>(ws + FL.cand), fused_cand_cap(*p),
                                         status, s);
        }
        return SIKV_ERR_UNSUPPORTED;
    }
    const FusedPlan plan = path == SIKV_DECODE_COMPOSED ? FusedPlan() : fused_plan(*p, qv);
    if (plan.ok)
        return launch_decode_fused(*p, plan, fused_layout(*p, L.fused), q, K, V, vq, codes, codebook, mu, seq_lens,
                                   k_per_seq, out, idx_out, scores_out, ws, status, s);
    // Too many segments for one co-resident launch: run the single-launch
    // kernel on sub-batches of sequences that fit, one after the other on the
    // stream (each launch leaves the coordination state zeroed for the next).
    const int bsub = path == SIKV_DECODE_COMPOSED ? 0 : fused_sub_batch(*p, qv);
    if (path == SIKV_DECODE_COOPERATIVE && bsub == 0) return SIKV_ERR_UNSUPPORTED;
    if (bsub > 0) {
        // one coordination layout, the largest sub-batch's, for every
        // sub-launch: a layout sized by each launch's own batch would place
        // one launch's counters and candidates over another's histograms,
        // which no launch then clears
        sikv_params pmax = *p;
        pmax.batch = bsub;
        const FusedLayout FL = fused_layout(pmax, L.fused);
        const size_t eb = p->dtype == SIKV_DTYPE_F32 ? 4 : 2;
        const size_t hq = p->num_q_heads, hkv = p->num_kv_heads, nmax = p->max_seq_len, d = p->head_dim;
        for (int b0 = 0; b0 < p->batch; b0 += bsub) {
            sikv_params ps = *p;
            ps.batch = std::min(bsub, p->batch - b0);
            const FusedPlan pl = fused_plan(ps, qv);
            if (!pl.ok) return SIKV_ERR_UNSUPPORTED;      // cannot happen: fused_sub_batch checked it
            const size_t bq = static_cast<size_t>(b0) * hq * d * eb, bkv = static_cast<size_t>(b0) * hkv * nmax * d * eb;
            SIKV_TRY(launch_decode_fused(
                ps, pl, FL, static_cast<const char *>(q) + bq, static_cast<const char *>(K) + bkv,
                static_cast<const char *>(V) + bkv,
                qv ? vq + static_cast<size_t>(b0) * hkv * nmax * kVqRowBytes : nullptr,
                codes + static_cast<size_t>(b0) * hkv * nmax * (d / 8),
                codebook + static_cast<size_t>(b0) * hkv * kSubspaces * kClusters * 4,
                mu + static_cast<size_t>(b0) * hkv * d, seq_lens + b0, k_per_seq + b0, static_cast<char *>(out) + bq,
                idx_out ? idx_out + static_cast<size_t>(b0) * hkv * (p->max_topk > 0 ? p->max_topk : 0) : nullptr,
                scores_out ? scores_out + static_cast<size_t>(b0) * hkv * nmax : nullptr, ws, status, s));
        }
        return SIKV_OK;
    }
    float *sc = scores_out ? scores_out : reinterpret_cast<float *>(ws + L.scores);
    int32_t *ix = idx_out ? idx_out : reinterpret_cast<int32_t *>(ws + L.idx);
    SIKV_TRY(launch_score(*p, q, codes, codebook, mu, seq_lens, sc, status, s));
    if (p->max_topk > 0) SIKV_TRY(launch_topk(*p, sc, seq_lens, k_per_seq, ix, status, s));
    return launch_sparse_attn(*p, q, K, V, vq, codes, codebook, mu, ix, k_per_seq, seq_lens, out, ws, L.attn,
                              status, s);
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
    return encode_layout(*p, device_sm_count()).total;
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

size_t sikv_dense_attn_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return sikv::dense_attn_layout(*p, kHeaderBytes).total;
}

sikv_status sikv_dense_score(const sikv_params *p, const void *q, const void *K, const int32_t *seq_lens,
                             float *scores, void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR4(scores);
    SIKV_TRY(check_ws(workspace, workspace_bytes, kHeaderBytes));
    return sikv::launch_dense_score(*p, q, K, seq_lens, scores, reinterpret_cast<int32_t *>(workspace),
                                    reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_dense_attn(const sikv_params *p, const void *q, const void *K, const void *V,
                            const int32_t *seq_lens, void *out, void *workspace, size_t workspace_bytes,
                            sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR(out);
    const sikv::DenseAttnLayout L = sikv::dense_attn_layout(*p, kHeaderBytes);
    SIKV_TRY(check_ws(workspace, workspace_bytes, L.total));
    char *ws = static_cast<char *>(workspace);
    return sikv::launch_dense_attn(*p, q, K, V, seq_lens, out, ws, kHeaderBytes, reinterpret_cast<int32_t *>(ws),
                                   reinterpret_cast<cudaStream_t>(stream));
}

size_t sikv_append_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return kHeaderBytes;
}

sikv_status sikv_append_codes(const sikv_params *p, const void *K, const int32_t *start, const int32_t *count,
                              const float *mu, uint8_t *codes, void *workspace, size_t workspace_bytes,
                              sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR4(start);
    SIKV_REQUIRE_PTR4(count);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR(codes);
    SIKV_TRY(check_ws(workspace, workspace_bytes, kHeaderBytes));
    int32_t *status = reinterpret_cast<int32_t *>(workspace);
    return sikv::launch_append(*p, K, start, count, mu, codes, status, reinterpret_cast<cudaStream_t>(stream));
}

size_t sikv_kmeans_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return sikv::kmeans_layout(*p, device_sm_count()).total;
}

sikv_status sikv_kmeans_codebook(const sikv_params *p, const void *K, const int32_t *seq_lens, const float *mu,
                                 const int32_t *init_idx, int32_t iters, uint8_t *codes, float *codebook,
                                 int32_t *counts, void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR4(init_idx);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    if (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)) return SIKV_ERR_UNSUPPORTED;
    if (iters < 1 || iters > 1000) return SIKV_ERR_INVALID_ARG;
    const sikv::KmeansLayout L = sikv::kmeans_layout(*p, device_sm_count());
    SIKV_TRY(check_ws(workspace, workspace_bytes, L.total));
    return sikv::launch_kmeans(*p, L, K, seq_lens, mu, init_idx, iters, codes, codebook, counts,
                               static_cast<char *>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

size_t sikv_decode_host_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return sikv::host_layout(*p, decode_layout(*p).total).total;
}

int32_t sikv_decode_resolved_path(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return resolve_decode_path(*p, false);
}

int32_t sikv_decode_launches(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    switch (resolve_decode_path(*p, false)) {
        case SIKV_DECODE_CLUSTER: return 1;                      // one cluster launch
        case SIKV_DECODE_COOPERATIVE: {
            if (fused_plan(*p).ok) return 1;                     // one cooperative kernel
            const int bsub = fused_sub_batch(*p);
            return (p->batch + bsub - 1) / bsub;                 // one per sub-batch
        }
        case SIKV_DECODE_COMPOSED: return 1 + (p->max_topk > 0 ? 1 : 0) + 2;   // score, top-k, attention + combine
        default: return 0;
    }
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
    const EncodeLayout L = encode_layout(*p, device_sm_count());
    SIKV_TRY(check_ws(workspace, workspace_bytes, L.total));
    return launch_encode(*p, L, K, seq_lens, mu, codes, codebook, counts, static_cast<char *>(workspace),
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
    return launch_sparse_attn(*p, q, K, V, nullptr, codes, codebook, mu, idx, k_per_seq, seq_lens, out,
                              static_cast<char *>(workspace), kHeaderBytes, static_cast<int32_t *>(workspace),
                              reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_sparse_attn_qv(const sikv_params *p, const void *q, const void *K, const void *V, const uint8_t *vq,
                                const uint8_t *codes, const float *codebook, const float *mu, const int32_t *idx,
                                const int32_t *k_per_seq, const int32_t *seq_lens, void *out, void *workspace,
                                size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR(vq);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    SIKV_REQUIRE_PTR(mu);
    if (p->max_topk > 0) SIKV_REQUIRE_PTR4(idx);
    SIKV_REQUIRE_PTR4(k_per_seq);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR(out);
    SIKV_TRY(check_ws(workspace, workspace_bytes, attn_layout(*p, kHeaderBytes).total));
    return launch_sparse_attn(*p, q, K, V, vq, codes, codebook, mu, idx, k_per_seq, seq_lens, out,
                              static_cast<char *>(workspace), kHeaderBytes, static_cast<int32_t *>(workspace),
                              reinterpret_cast<cudaStream_t>(stream));
}

size_t sikv_quantize_values_workspace_size(const sikv_params *p) {
    if (check_params(p) != SIKV_OK) return 0;
    return kHeaderBytes;
}

sikv_status sikv_quantize_values(const sikv_params *p, const void *V, const int32_t *seq_lens, uint8_t *vq,
                                 void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR(vq);
    SIKV_TRY(check_ws(workspace, workspace_bytes, kHeaderBytes));
    return sikv::launch_quantize_values(*p, V, seq_lens, vq, static_cast<int32_t *>(workspace),
                                        reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_decode(const sikv_params *p, const void *q, const void *K, const void *V,
                        const uint8_t *codes, const float *codebook, const float *mu,
                        const int32_t *seq_lens, const int32_t *k_per_seq, void *out, int32_t *idx_out,
                        float *scores_out, void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(out);
    if (idx_out) SIKV_REQUIRE_PTR4(idx_out);
    if (scores_out) SIKV_REQUIRE_PTR4(scores_out);
    return sikv::decode_step(*p, q, K, V, nullptr, codes, codebook, mu, seq_lens, k_per_seq, out, idx_out,
                             scores_out, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_decode_qv(const sikv_params *p, const void *q, const void *K, const void *V, const uint8_t *vq,
                           const uint8_t *codes, const float *codebook, const float *mu, const int32_t *seq_lens,
                           const int32_t *k_per_seq, void *out, int32_t *idx_out, float *scores_out, void *workspace,
                           size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(q);
    SIKV_REQUIRE_PTR(out);
    SIKV_REQUIRE_PTR(vq);
    if (idx_out) SIKV_REQUIRE_PTR4(idx_out);
    if (scores_out) SIKV_REQUIRE_PTR4(scores_out);
    return sikv::decode_step(*p, q, K, V, vq, codes, codebook, mu, seq_lens, k_per_seq, out, idx_out, scores_out,
                             workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

sikv_status sikv_decode_host(const sikv_params *p, const void *q_host, const void *K, const void *V,
                             const uint8_t *codes, const float *codebook, const float *mu,
                             const int32_t *seq_lens, const int32_t *k_per_seq, void *out_host,
                             void *workspace, size_t workspace_bytes, sikv_stream_t stream) {
    SIKV_TRY(check_params(p));
    if (!q_host || !out_host) return SIKV_ERR_INVALID_ARG;
    const size_t decode_total = decode_layout(*p).total;
    const sikv::HostLayout H = sikv::host_layout(*p, decode_total);
    SIKV_TRY(check_ws(workspace, workspace_bytes, H.total));
    char *ws = static_cast<char *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // Page-locked host buffers are device-addressable (unified addressing).
    // The query is read by every CTA of its segment, so it is brought into the
    // workspace first: by a copy kernel that reads each byte of the host
    // buffer once (a 32 KB DMA copy costs more, in latency), or, for pageable
    // or unaligned buffers, by cudaMemcpyAsync.  The output, written once, goes
    // to a page-locked buffer in place.
    const void *q_view = sikv::device_view(q_host);
    void *out_dev = sikv::device_view(out_host);
    char *q_dev = ws + H.q;
    if (q_view && (reinterpret_cast<uintptr_t>(q_view) & 15u) == 0 && H.bytes % 16 == 0) {
        const int n16 = static_cast<int>(H.bytes / 16);
        sikv::copy16_kernel<<<sikv::copy16_grid(n16), 256, 0, s>>>(static_cast<const uint4 *>(q_view),
                                                                   reinterpret_cast<uint4 *>(q_dev), n16);
        if (cudaGetLastError() != cudaSuccess) return SIKV_ERR_CUDA;
    } else if (cudaMemcpyAsync(q_dev, q_host, H.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        return SIKV_ERR_CUDA;
    }
    SIKV_TRY(sikv::decode_step(*p, q_dev, K, V, nullptr, codes, codebook, mu, seq_lens, k_per_seq,
                               out_dev ? out_dev : ws + H.out, nullptr, nullptr, workspace, decode_total, s));
    if (!out_dev &&
        cudaMemcpyAsync(out_host, ws + H.out, H.bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SIKV_ERR_CUDA;
    return SIKV_OK;
}

void sikv_decode_host_plan_destroy(sikv_host_plan *plan) {
    if (!plan) return;
    if (plan->exec) cudaGraphExecDestroy(plan->exec);
    if (plan->graph) cudaGraphDestroy(plan->graph);
    delete plan;
}

sikv_status sikv_decode_host_plan_create(const sikv_params *p, const void *K, const void *V, const uint8_t *codes,
                                         const float *codebook, const float *mu, const int32_t *seq_lens,
                                         const int32_t *k_per_seq, void *workspace, size_t workspace_bytes,
                                         sikv_host_plan **plan) {
    if (!plan) return SIKV_ERR_INVALID_ARG;
    *plan = nullptr;
    SIKV_TRY(check_params(p));
    SIKV_REQUIRE_PTR(K);
    SIKV_REQUIRE_PTR(V);
    SIKV_REQUIRE_PTR(codes);
    SIKV_REQUIRE_PTR(codebook);
    SIKV_REQUIRE_PTR(mu);
    SIKV_REQUIRE_PTR4(seq_lens);
    SIKV_REQUIRE_PTR4(k_per_seq);
    const size_t decode_total = decode_layout(*p).total;
    const sikv::HostLayout H = sikv::host_layout(*p, decode_total);
    SIKV_TRY(check_ws(workspace, workspace_bytes, H.total));
    if (H.bytes % 16 != 0) return SIKV_ERR_UNSUPPORTED;
    // the launch facts the decode kernels need are computed now, outside the capture
    if (resolve_decode_path(*p, false) == 0) return SIKV_ERR_UNSUPPORTED;

    sikv_host_plan *pl = new (std::nothrow) sikv_host_plan();
    if (!pl) return SIKV_ERR_CUDA;
    pl->p = *p;
    pl->K = K;
    pl->V = V;
    pl->codes = codes;
    pl->codebook = codebook;
    pl->mu = mu;
    pl->seq_lens = seq_lens;
    pl->k_per_seq = k_per_seq;
    pl->ws = static_cast<char *>(workspace);
    pl->ws_bytes = workspace_bytes;
    pl->q_slot = reinterpret_cast<uint4 *>(pl->ws + H.q);
    pl->out_slot = reinterpret_cast<uint4 *>(pl->ws + H.out);
    pl->n16 = static_cast<int>(H.bytes / 16);

    // capture on a private stream: nothing runs now.  The copies are captured
    // with placeholder host ends (the workspace slots themselves) that every
    // run replaces.
    cudaStream_t cs = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) {
        delete pl;
        return SIKV_ERR_CUDA;
    }
    sikv_status st = SIKV_OK;
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        st = SIKV_ERR_CUDA;
    } else {
        const int g = sikv::copy16_grid(pl->n16);
        sikv::copy16_kernel<<<g, 256, 0, cs>>>(pl->q_slot, pl->q_slot, pl->n16);
        st = sikv::decode_step(*p, pl->q_slot, K, V, nullptr, codes, codebook, mu, seq_lens, k_per_seq, pl->out_slot,
                               nullptr, nullptr, workspace, decode_total, cs);
        sikv::copy16_kernel<<<g, 256, 0, cs>>>(pl->out_slot, pl->out_slot, pl->n16);
        cudaGraph_t graph = nullptr;
        const cudaError_t e = cudaStreamEndCapture(cs, &graph);      // always ends the capture
        pl->graph = graph;
        if (st == SIKV_OK && (e != cudaSuccess || !graph)) st = SIKV_ERR_CUDA;
    }
    cudaStreamDestroy(cs);
    cudaGetLastError();
    // the two copy nodes: the one writing the q slot and the one reading the output slot
    if (st == SIKV_OK) {
        size_t n = 0;
        if (cudaGraphGetNodes(pl->graph, nullptr, &n) != cudaSuccess) st = SIKV_ERR_CUDA;
        std::vector<cudaGraphNode_t> nodes(n);
        if (st == SIKV_OK && n && cudaGraphGetNodes(pl->graph, nodes.data(), &n) != cudaSuccess) st = SIKV_ERR_CUDA;
        for (size_t i = 0; st == SIKV_OK && i < n; ++i) {
            cudaGraphNodeType type;
            if (cudaGraphNodeGetType(nodes[i], &type) != cudaSuccess || type != cudaGraphNodeTypeKernel) continue;
            cudaKernelNodeParams kp;
            if (cudaGraphKernelNodeGetParams(nodes[i], &kp) != cudaSuccess) continue;
            if (kp.func != reinterpret_cast<void *>(sikv::copy16_kernel) || !kp.kernelParams) continue;
            const uint4 *src = *static_cast<const uint4 *const *>(kp.kernelParams[0]);
            uint4 *dst = *static_cast<uint4 *const *>(kp.kernelParams[1]);
            if (dst == pl->q_slot && src == pl->q_slot) {
                pl->up = nodes[i];
                pl->up_kp = kp;
            } else if (src == pl->out_slot) {
                pl->down = nodes[i];
                pl->down_kp = kp;
            }
        }
        if (st == SIKV_OK && (!pl->up || !pl->down)) st = SIKV_ERR_CUDA;
    }
    if (st == SIKV_OK && cudaGraphInstantiate(&pl->exec, pl->graph, 0) != cudaSuccess) st = SIKV_ERR_CUDA;
    cudaGetLastError();
    if (st != SIKV_OK) {
        sikv_decode_host_plan_destroy(pl);
        return st;
    }
    *plan = pl;
    return SIKV_OK;
}

sikv_status sikv_decode_host_plan_run(sikv_host_plan *plan, const void *q_host, void *out_host,
                                      sikv_stream_t stream) {
    if (!plan || !q_host || !out_host) return SIKV_ERR_INVALID_ARG;
    const void *qv = sikv::device_view(q_host);
    void *ov = sikv::device_view(out_host);
    const bool graphed = qv && ov && (reinterpret_cast<uintptr_t>(qv) & 15u) == 0 &&
                         (reinterpret_cast<uintptr_t>(ov) & 15u) == 0;
    if (!graphed)
        return sikv_decode_host(&plan->p, q_host, plan->K, plan->V, plan->codes, plan->codebook, plan->mu,
                                plan->seq_lens, plan->k_per_seq, out_host, plan->ws, plan->ws_bytes, stream);
    int n16 = plan->n16;
    const uint4 *up_src = static_cast<const uint4 *>(qv);
    uint4 *up_dst = plan->q_slot;
    void *up_args[] = {&up_src, &up_dst, &n16};
    cudaKernelNodeParams kp = plan->up_kp;
    kp.kernelParams = up_args;
    kp.extra = nullptr;
    if (cudaGraphExecKernelNodeSetParams(plan->exec, plan->up, &kp) != cudaSuccess) return SIKV_ERR_CUDA;
    const uint4 *down_src = plan->out_slot;
    uint4 *down_dst = static_cast<uint4 *>(ov);
    void *down_args[] = {&down_src, &down_dst, &n16};
    kp = plan->down_kp;
    kp.kernelParams = down_args;
    kp.extra = nullptr;
    if (cudaGraphExecKernelNodeSetParams(plan->exec, plan->down, &kp) != cudaSuccess) return SIKV_ERR_CUDA;
    if (cudaGraphLaunch(plan->exec, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SIKV_ERR_CUDA;
    return SIKV_OK;
}

}  // extern "C"
