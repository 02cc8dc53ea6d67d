// Prefill encoder: channel mean, sign-pattern codes and the one-pass codebook.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 1 (sign-based 1-bit VQ: channel-mean
// normalization, 4-dim sub-vectors -> 16 sign-pattern clusters, codebook
// without iterations) and item 3 (token-wise codes, 64 sink tokens).
//
// Three passes per (sequence, KV head) segment, each split into token chunks:
//   enc_mean_partial   K -> per-chunk exact channel sums (double-double)
//   enc_mean_final     partial sums -> mu, the correctly rounded fp32 mean
//   enc_codes_partial  K, mu -> packed codes + per-chunk cluster sums/counts
//   enc_codebook_final partial sums -> centroids (fp32) and counts
// K is read twice (the mean must be known before any sign is taken).
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / 32;
constexpr int kEncUnroll = 4;      // rows in flight per thread, mean pass
constexpr int kEncUnrollCodes = 16; // rows in flight per thread, codes pass (2 CTAs/SM by shared memory)

template <int DT>
__global__ void __launch_bounds__(kEncThreads)
enc_mean_partial(const void *__restrict__ K, const int32_t *__restrict__ seq_lens, int hkv,
                 int nmax, int num_sinks, int chunk, int nchunks, double2 *__restrict__ part,
                 int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    const int seg = blockIdx.y, c = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = max(c * chunk, num_sinks), t1 = min((c + 1) * chunk, n_tok);
    const char *base = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;

    dd acc[4] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
    int t = t0 + warp;
    for (; t + (kEncUnroll - 1) * kEncWarps < t1; t += kEncUnroll * kEncWarps) {
        float4 v[kEncUnroll];
#pragma unroll
        for (int u = 0; u < kEncUnroll; ++u)
            v[u] = load4<DT>(base + static_cast<size_t>(t + u * kEncWarps) * kHeadDim * EB, lane * 4);
#pragma unroll
        for (int u = 0; u < kEncUnroll; ++u) {
            dd_add_double(acc[0], v[u].x);
            dd_add_double(acc[1], v[u].y);
            dd_add_double(acc[2], v[u].z);
            dd_add_double(acc[3], v[u].w);
        }
    }
    for (; t < t1; t += kEncWarps) {
        float4 v = load4<DT>(base + static_cast<size_t>(t) * kHeadDim * EB, lane * 4);
        dd_add_double(acc[0], v.x);
        dd_add_double(acc[1], v.y);
        dd_add_double(acc[2], v.z);
        dd_add_double(acc[3], v.w);
    }

    __shared__ dd red[kEncWarps][kHeadDim];
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane * 4 + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < kHeadDim) {
        dd s = red[0][threadIdx.x];
#pragma unroll
        for (int w = 1; w < kEncWarps; ++w) s = dd_add(s, red[w][threadIdx.x]);
        part[(static_cast<size_t>(seg) * nchunks + c) * kHeadDim + threadIdx.x] = make_double2(s.hi, s.lo);
    }
}

__global__ void __launch_bounds__(kHeadDim)
enc_mean_final(const double2 *__restrict__ part, const int32_t *__restrict__ seq_lens, int hkv,
               int nmax, int num_sinks, int chunk, int nchunks, float *__restrict__ mu,
               int32_t *status) {
    const int seg = blockIdx.x, ch = threadIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int n = max(n_tok - num_sinks, 0);
    float m = 0.0f;
    if (n > 0) {
        const int used = min((n_tok + chunk - 1) / chunk, nchunks);
        dd s = {0.0, 0.0};
        for (int c = 0; c < used; ++c) {
            double2 p = part[(static_cast<size_t>(seg) * nchunks + c) * kHeadDim + ch];
            s = dd_add(s, dd{p.x, p.y});
        }
        m = dd_div_to_float_rn(s, static_cast<double>(n));
    }
    mu[static_cast<size_t>(seg) * kHeadDim + ch] = m;
}

// Thread (warp w, lane s) owns subspace s: channels 4s..4s+3 of every row the
// warp visits.  Its cluster sums live in shared memory, private to the thread:
// bins[j][thread] (float4) and cnt[j][thread], laid out so that a warp's
// accesses hit distinct banks whatever the codes are.
template <int DT>
__global__ void __launch_bounds__(kEncThreads)
enc_codes_partial(const void *__restrict__ K, const int32_t *__restrict__ seq_lens,
                  const float *__restrict__ mu, int hkv, int nmax, int num_sinks, int chunk,
                  int nchunks, uint8_t *__restrict__ codes, double *__restrict__ cb_part,
                  int32_t *__restrict__ cnt_part, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    extern __shared__ float4 enc_smem[];
    float4 *bins = enc_smem;                                             // [16][256]
    uint32_t *cnt = reinterpret_cast<uint32_t *>(enc_smem + kClusters * kEncThreads);   // [16][256]

    const int seg = blockIdx.y, c = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = c * chunk, t1 = min((c + 1) * chunk, n_tok);
    const char *base = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    uint8_t *crow = codes + static_cast<size_t>(seg) * nmax * kCodeBytes;
    const float4 m = __ldg(reinterpret_cast<const float4 *>(mu + static_cast<size_t>(seg) * kHeadDim) + lane);

#pragma unroll
    for (int j = 0; j < kClusters; ++j) {
        bins[j * kEncThreads + tid] = make_float4(0.f, 0.f, 0.f, 0.f);
        cnt[j * kEncThreads + tid] = 0u;
    }

    auto consume = [&](int t, float4 v) {
        const int j = (v.x >= m.x ? 1 : 0) | (v.y >= m.y ? 2 : 0) | (v.z >= m.z ? 4 : 0) |
                      (v.w >= m.w ? 8 : 0);
        const int jn = __shfl_down_sync(0xffffffffu, j, 1);
        if (!(lane & 1)) crow[static_cast<size_t>(t) * kCodeBytes + (lane >> 1)] = static_cast<uint8_t>(j | (jn << 4));
        if (t >= num_sinks) {
            float4 *bp = bins + j * kEncThreads + tid;
            float4 a = *bp;
            a.x += v.x - m.x;
            a.y += v.y - m.y;
            a.z += v.z - m.z;
            a.w += v.w - m.w;
            *bp = a;
            cnt[j * kEncThreads + tid] += 1u;
        }
    };

    int t = t0 + warp;
    for (; t + (kEncUnrollCodes - 1) * kEncWarps < t1; t += kEncUnrollCodes * kEncWarps) {
        float4 v[kEncUnrollCodes];
#pragma unroll
        for (int u = 0; u < kEncUnrollCodes; ++u)
            v[u] = load4<DT>(base + static_cast<size_t>(t + u * kEncWarps) * kHeadDim * EB, lane * 4);
#pragma unroll
        for (int u = 0; u < kEncUnrollCodes; ++u) consume(t + u * kEncWarps, v[u]);
    }
    for (; t < t1; t += kEncWarps)
        consume(t, load4<DT>(base + static_cast<size_t>(t) * kHeadDim * EB, lane * 4));
    __syncthreads();

    // Reduce the 8 warps' bins of each (subspace, cluster) in a fixed order.
    for (int pr = tid; pr < kSubspaces * kClusters; pr += kEncThreads) {
        const int j = pr >> 5, s = pr & 31;
        double sx = 0.0, sy = 0.0, sz = 0.0, sw = 0.0;
        uint32_t n = 0;
#pragma unroll
        for (int w = 0; w < kEncWarps; ++w) {
            const float4 a = bins[j * kEncThreads + w * 32 + s];
            sx += a.x;
            sy += a.y;
            sz += a.z;
            sw += a.w;
            n += cnt[j * kEncThreads + w * 32 + s];
        }
        const size_t o = ((static_cast<size_t>(seg) * nchunks + c) * kSubspaces + s) * kClusters + j;
        reinterpret_cast<double4 *>(cb_part)[o] = make_double4(sx, sy, sz, sw);
        cnt_part[o] = static_cast<int32_t>(n);
    }
}

__global__ void __launch_bounds__(kSubspaces * kClusters)
enc_codebook_final(const double *__restrict__ cb_part, const int32_t *__restrict__ cnt_part,
                   const int32_t *__restrict__ seq_lens, int hkv, int nmax, int chunk,
                   int nchunks, float *__restrict__ codebook, int32_t *__restrict__ counts,
                   int32_t *status) {
    const int seg = blockIdx.x, pr = threadIdx.x;       // pr = s * 16 + j
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int used = min((n_tok + chunk - 1) / chunk, nchunks);
    double sx = 0.0, sy = 0.0, sz = 0.0, sw = 0.0;
    long long n = 0;
    for (int c = 0; c < used; ++c) {
        const size_t o = (static_cast<size_t>(seg) * nchunks + c) * kSubspaces * kClusters + pr;
        const double4 a = reinterpret_cast<const double4 *>(cb_part)[o];
        sx += a.x;
        sy += a.y;
        sz += a.z;
        sw += a.w;
        n += cnt_part[o];
    }
    float4 cv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n > 0) {
        const double dn = static_cast<double>(n);
        cv = make_float4(__double2float_rn(sx / dn), __double2float_rn(sy / dn),
                         __double2float_rn(sz / dn), __double2float_rn(sw / dn));
    }
    reinterpret_cast<float4 *>(codebook)[static_cast<size_t>(seg) * kSubspaces * kClusters + pr] = cv;
    if (counts) counts[static_cast<size_t>(seg) * kSubspaces * kClusters + pr] = static_cast<int32_t>(n);
}

}  // namespace

EncodeLayout encode_layout(const sikv_params &p) {
    EncodeLayout L;
    const int nmax = p.max_seq_len;
    int chunk = (nmax + 15) / 16;
    chunk = (chunk + 255) / 256 * 256;
    chunk = chunk < 256 ? 256 : (chunk > 4096 ? 4096 : chunk);
    L.chunk = chunk;
    L.nchunks = (nmax + chunk - 1) / chunk;
    const size_t segs = static_cast<size_t>(p.batch) * p.num_kv_heads;
    size_t off = kHeaderBytes;
    L.mean_part = off;
    off = align_up(off + segs * L.nchunks * kHeadDim * sizeof(double2), 256);
    L.cb_part = off;
    off = align_up(off + segs * L.nchunks * kSubspaces * kClusters * 4 * sizeof(double), 256);
    L.cnt_part = off;
    off = align_up(off + segs * L.nchunks * kSubspaces * kClusters * sizeof(int32_t), 256);
    L.total = off;
    return L;
}

sikv_status launch_encode(const sikv_params &p, const void *K, const int32_t *seq_lens, float *mu,
                          uint8_t *codes, float *codebook, int32_t *counts, char *ws,
                          cudaStream_t stream) {
    const EncodeLayout L = encode_layout(p);
    const int segs = p.batch * p.num_kv_heads;
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    double2 *mean_part = reinterpret_cast<double2 *>(ws + L.mean_part);
    double *cb_part = reinterpret_cast<double *>(ws + L.cb_part);
    int32_t *cnt_part = reinterpret_cast<int32_t *>(ws + L.cnt_part);
    const dim3 grid(L.nchunks, segs);
    const size_t codes_smem = kClusters * kEncThreads * (sizeof(float4) + sizeof(uint32_t));

    if (p.dtype == SIKV_DTYPE_BF16) {
        enc_mean_partial<SIKV_DTYPE_BF16><<<grid, kEncThreads, 0, stream>>>(
            K, seq_lens, p.num_kv_heads, p.max_seq_len, p.num_sinks, L.chunk, L.nchunks, mean_part, status);
    } else {
        enc_mean_partial<SIKV_DTYPE_F32><<<grid, kEncThreads, 0, stream>>>(
            K, seq_lens, p.num_kv_heads, p.max_seq_len, p.num_sinks, L.chunk, L.nchunks, mean_part, status);
    }
    enc_mean_final<<<segs, kHeadDim, 0, stream>>>(mean_part, seq_lens, p.num_kv_heads, p.max_seq_len,
                                                  p.num_sinks, L.chunk, L.nchunks, mu, status);
    if (p.dtype == SIKV_DTYPE_BF16) {
        auto kern = enc_codes_partial<SIKV_DTYPE_BF16>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)codes_smem) != cudaSuccess)
            return SIKV_ERR_CUDA;
        kern<<<grid, kEncThreads, codes_smem, stream>>>(K, seq_lens, mu, p.num_kv_heads, p.max_seq_len,
                                                        p.num_sinks, L.chunk, L.nchunks, codes, cb_part,
                                                        cnt_part, status);
    } else {
        auto kern = enc_codes_partial<SIKV_DTYPE_F32>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)codes_smem) != cudaSuccess)
            return SIKV_ERR_CUDA;
        kern<<<grid, kEncThreads, codes_smem, stream>>>(K, seq_lens, mu, p.num_kv_heads, p.max_seq_len,
                                                        p.num_sinks, L.chunk, L.nchunks, codes, cb_part,
                                                        cnt_part, status);
    }
    enc_codebook_final<<<segs, kSubspaces * kClusters, 0, stream>>>(
        cb_part, cnt_part, seq_lens, p.num_kv_heads, p.max_seq_len, L.chunk, L.nchunks, codebook, counts, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
