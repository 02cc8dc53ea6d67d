// sikv_score: compressed-domain LUT-GEMV scores of every cached token.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 2 (LUT-GEMV retrieval) and item 3 (sinks are
// not scored).  Grid: (token chunk, segment); each CTA builds the segment's
// tables in shared memory and streams its chunk of 16-byte code rows.  The
// chunk length is chosen per shape and device: long enough that building
// the 64 KB table is a small part of a CTA's time, short enough that the
// chunk CTAs fill whole waves (3 per SM).
#include <algorithm>

#include "score_device.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kScoreCtasPerSm = 3;     // the byte table (64 KB) allows three
constexpr int kScoreUnroll = 8;        // code rows in flight per thread

template <int DT>
__global__ void __launch_bounds__(kScoreThreads, kScoreCtasPerSm)
score_kernel(const void *__restrict__ q, const uint8_t *__restrict__ codes,
             const float *__restrict__ codebook, const float *__restrict__ mu,
             const int32_t *__restrict__ seq_lens, int hq, int hkv, int nmax, int num_sinks, int chunk,
             float *__restrict__ scores, int32_t *status) {
    extern __shared__ __align__(16) unsigned char score_smem[];
    ScoreTables &sh = *reinterpret_cast<ScoreTables *>(score_smem);
    // staged table inputs live in the byte table's space: they are last read
    // before the barrier that precedes the table's first write
    float4 *cbs = reinterpret_cast<float4 *>(sh.t2);                       // 2048 floats
    float *qs = sh.t2 + kSubspaces * kClusters * 4;                          // <= 8 x 128 floats
    float *mus = qs + kMaxGroup * kHeadDim;                                  // 128 floats
    const int seg = blockIdx.y, b = seg / hkv, h = seg % hkv, group = hq / hkv;
    const int n_tok = load_seq_len(seq_lens, b, nmax, status);
    if (n_tok < 0) return;
    const int t_begin = blockIdx.x * chunk;
    if (t_begin >= n_tok) return;
    const int t_end = min(t_begin + chunk, n_tok);
    {
        TableInputs<DT> in;
        in.load(q, codebook, mu, b, h, hq, group, seg);
        in.store(qs, cbs, mus, group);
    }
    __syncthreads();
    build_score_tables(sh, qs, cbs, mus, group);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float qmu = sh.qmu;
    float *srow = scores + static_cast<size_t>(seg) * nmax;
    const uint4 *crow = reinterpret_cast<const uint4 *>(codes + static_cast<size_t>(seg) * nmax * kCodeBytes);
    constexpr int kStride = kScoreWarps * 32;
    for (int g0 = t_begin + warp * 32; g0 < t_end; g0 += kStride * kScoreUnroll) {
        uint4 rows[kScoreUnroll];
#pragma unroll
        for (int u = 0; u < kScoreUnroll; ++u) {
            const int t = g0 + u * kStride + lane;
            rows[u] = (t >= num_sinks && t < t_end) ? __ldcs(crow + t) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kScoreUnroll; u += 2) {
            const float2 v = lut2_score2(sh.t2, rows[u], rows[u + 1], lane, qmu);
            const int ta = g0 + u * kStride + lane, tb = ta + kStride;
            if (ta < t_end) srow[ta] = (ta >= num_sinks) ? v.x : -INFINITY;
            if (tb < t_end) srow[tb] = (tb >= num_sinks) ? v.y : -INFINITY;
        }
    }
}

// Tokens per CTA: a multiple of 256 (each warp's 32 tokens start at a
// multiple of 32, which the lane rotation of the tables needs), chosen to
// minimize (waves of chunk CTAs) x (chunk + 2048), the second term the table
// build's cost in tokens.  4096 without a device.
int score_chunk(int nmax, int segs) {
    const int sms = device_sm_count();
    nmax = std::max(nmax, 1);
    if (sms < 1 || segs < 1) return 4096;
    const long long slots = static_cast<long long>(kScoreCtasPerSm) * sms;
    long long best = -1;
    int chunk = 4096;
    for (int n = 1; n <= (nmax + 255) / 256; ++n) {
        const int ch = ((nmax + n - 1) / n + 255) / 256 * 256;
        const long long nn = (nmax + ch - 1) / ch;
        const long long cost = (static_cast<long long>(segs) * nn + slots - 1) / slots * (ch + 2048);
        if (best < 0 || cost < best) {
            best = cost;
            chunk = ch;
        }
    }
    return chunk;
}

}  // namespace

sikv_status launch_score(const sikv_params &p, const void *q, const uint8_t *codes,
                         const float *codebook, const float *mu, const int32_t *seq_lens,
                         float *scores, int32_t *status, cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    const int chunk = score_chunk(p.max_seq_len, segs);
    const dim3 grid((p.max_seq_len + chunk - 1) / chunk, segs);
    const size_t smem = sizeof(ScoreTables);
    if (p.dtype == SIKV_DTYPE_BF16) {
        auto kern = score_kernel<SIKV_DTYPE_BF16>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return SIKV_ERR_CUDA;
        kern<<<grid, kScoreThreads, smem, stream>>>(q, codes, codebook, mu, seq_lens, p.num_q_heads,
                                                    p.num_kv_heads, p.max_seq_len, p.num_sinks, chunk, scores, status);
    } else {
        auto kern = score_kernel<SIKV_DTYPE_F32>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return SIKV_ERR_CUDA;
        kern<<<grid, kScoreThreads, smem, stream>>>(q, codes, codebook, mu, seq_lens, p.num_q_heads,
                                                    p.num_kv_heads, p.max_seq_len, p.num_sinks, chunk, scores, status);
    }
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
