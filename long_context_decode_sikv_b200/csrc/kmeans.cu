// K-means codebook: the iterative clustering that the one-pass sign-pattern
// codebook replaces.  A comparison baseline, not the method.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 1 (the one-pass clustering of the normalized
// 4-dim sub-vectors into 16 clusters is offered in place of iterative
// K-means) and §4 (efficiency: clustering 20x faster than K-means with 20
// iterations).  The pages give no K-means details; this is Lloyd's algorithm
// on the same points and codebook shape:
//   points    x = fl32(k - mu) of the non-sink tokens, sub-vector s = dims 4s..4s+3;
//   start     centroid j of every subspace = sub-vector of the given token j;
//   assign    nearest centroid by ((d0*d0 + d1*d1) + d2*d2) + d3*d3, d_i = x_i - c_i,
//             each operation rounded to fp32 in that order, ties to the lower cluster;
//   update    a non-empty cluster moves to the exact mean of its points, rounded once
//             to fp32; an empty cluster keeps its centroid.
// The codes are the last assignment, packed like the sign codes (two per
// byte, even subspace in the low nibble), so the LUT scorer reads them as is.
//
// Per iteration: kmeans_assign_kernel, kmeans_accum_kernel, kmeans_update_kernel.
//   assign  lane l of a warp owns subspace l: the warp reads one key row per
//           token (coalesced), each lane finds its sub-vector's nearest of 16
//           centroids held in registers (differences and squares of two
//           clusters per f32x2 instruction, then a tree argmin) and the 8
//           lanes of each 32-bit word store the packed codes.
//   accum   thread d owns channel d: for each token of its chunk it adds
//           fl32(k_d - mu_d) exactly (double-double) to the sum of the token's
//           cluster in its own shared-memory column (16 clusters x 16 bytes),
//           so accesses never conflict and many CTAs share an SM; one partial
//           per chunk.
//   update  per (segment, subspace, cluster, dim): the chunk partials in chunk
//           order, then the correctly rounded quotient by the count.
// The sums are exact while a cluster's points span fewer than about 40
// binades, so the result does not depend on how tokens fall into chunks.
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kKmWarps = 4;                    // assign: 4 warps per CTA, several CTAs per SM
constexpr int kKmThreads = kKmWarps * 32;
constexpr int kKmUnroll = 4;                   // key rows per group; two groups in flight per warp
constexpr int kKmClusters = 16;
constexpr int kKmSub = kHeadDim / 4;           // 32 subspaces: one per lane
constexpr int kKmEntries = kKmClusters * 4 * kKmSub;   // (cluster, dim, subspace) sums
constexpr int kKmUpdateThreads = 256;
constexpr int kKaThreads = kHeadDim;           // accum: one thread per channel
constexpr int kKaUnroll = 8;                   // keys loaded ahead per thread
constexpr int kKmCtasPerSm = 6;                // accum CTAs per SM the chunking aims for

// One accumulation CTA's exact sums: column d (channel d) belongs to thread
// d, so a warp's 16-byte accesses are conflict-free whatever the clusters.
struct KmAccSmem {
    double2 sum[kKmClusters][kKaThreads];      // (hi, lo) double-double, 32 KB
    int32_t cnt[kKmClusters][kKmSub];          // 2 KB (threads of dimension 0 count)
};

__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
    return static_cast<unsigned long long>(__float_as_uint(lo)) |
           (static_cast<unsigned long long>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float lo_of(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_of(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

// Lane-wise fp32 arithmetic on pairs, each lane rounded to nearest.  The
// squared terms are summed with scalar __fadd_rn, not add.f32x2: ptxas fuses
// a paired multiply and a paired add into a fused multiply-add even when both
// carry .rn (measured: an exact distance tie then went to the higher
// cluster), while a scalar add.rn is never fused.
__device__ __forceinline__ unsigned long long sub_x2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long mul_x2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Index of the nearest centroid; cp[p][i] holds dimension i of clusters 2p
// (low) and 2p+1 (high).  The tree keeps the left (lower-index) side unless
// the right is strictly nearer, so of equal distances the lowest index wins.
__device__ __forceinline__ int nearest(const unsigned long long (&cp)[kKmClusters / 2][4], float x0, float x1,
                                       float x2, float x3) {
    const unsigned long long xx0 = pack2(x0, x0), xx1 = pack2(x1, x1), xx2 = pack2(x2, x2), xx3 = pack2(x3, x3);
    float d[kKmClusters];
#pragma unroll
    for (int p = 0; p < kKmClusters / 2; ++p) {
        const unsigned long long e0 = sub_x2(xx0, cp[p][0]), e1 = sub_x2(xx1, cp[p][1]);
        const unsigned long long e2 = sub_x2(xx2, cp[p][2]), e3 = sub_x2(xx3, cp[p][3]);
        const unsigned long long q0 = mul_x2(e0, e0), q1 = mul_x2(e1, e1), q2 = mul_x2(e2, e2), q3 = mul_x2(e3, e3);
        d[2 * p] = __fadd_rn(__fadd_rn(__fadd_rn(lo_of(q0), lo_of(q1)), lo_of(q2)), lo_of(q3));
        d[2 * p + 1] = __fadd_rn(__fadd_rn(__fadd_rn(hi_of(q0), hi_of(q1)), hi_of(q2)), hi_of(q3));
    }
    int idx[kKmClusters];
#pragma unroll
    for (int j = 0; j < kKmClusters; ++j) idx[j] = j;
#pragma unroll
    for (int w = 1; w < kKmClusters; w <<= 1) {
#pragma unroll
        for (int j = 0; j < kKmClusters; j += 2 * w) {
            const bool right = d[j + w] < d[j];
            d[j] = right ? d[j + w] : d[j];
            idx[j] = right ? idx[j + w] : idx[j];
        }
    }
    return idx[0];
}

// Sum of two double-double values, both sides by two_sum (no ordering
// precondition): exact while the result fits the pair.
__device__ __forceinline__ dd dd_merge(dd a, dd b) {
    const dd s = two_sum(a.hi, b.hi), t = two_sum(a.lo, b.lo);
    dd r = two_sum(s.hi, s.lo + t.hi);
    r.lo += t.lo;
    return two_sum(r.hi, r.lo);
}

// Starting centroids: c[s][j][i] = fl32(K[init_j][4s+i] - mu[4s+i]).  A
// segment with no non-sink token, an invalid length or an invalid start
// token gets 0 for the affected centroids (the latter two flagged).
template <int DT>
__global__ void __launch_bounds__(256)
kmeans_init_kernel(const void *__restrict__ K, const int32_t *__restrict__ seq_lens, const float *__restrict__ mu,
                   const int32_t *__restrict__ init_idx, float *__restrict__ cent, int hkv, int nmax, int num_sinks,
                   int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    const int seg = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    float *c = cent + static_cast<size_t>(seg) * kKmSub * kKmClusters * 4;
    const char *krows = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    for (int e = threadIdx.x; e < kKmSub * kKmClusters * 4; e += blockDim.x) {
        const int s = e / (kKmClusters * 4), j = (e / 4) % kKmClusters, i = e % 4;
        float v = 0.f;
        if (n_tok > num_sinks) {
            const int t = __ldg(init_idx + static_cast<size_t>(seg) * kKmClusters + j);
            if (t >= num_sinks && t < n_tok) {
                const int dim = 4 * s + i;
                v = __fsub_rn(load1<DT>(krows + static_cast<size_t>(t) * kHeadDim * EB, dim),
                              __ldg(mu + static_cast<size_t>(seg) * kHeadDim + dim));
            } else if (s == 0 && i == 0) {
                flag_error(status, SIKV_DEVERR_INDEX);
            }
        }
        c[e] = v;
    }
}

// Assignment of the tokens of chunk blockIdx.x of segment blockIdx.y: the
// packed nearest-centroid codes of every token into codes.
template <int DT>
__global__ void __launch_bounds__(kKmThreads)
kmeans_assign_kernel(const void *__restrict__ K, const int32_t *__restrict__ seq_lens, const float *__restrict__ mu,
                     const float *__restrict__ cent, int hkv, int nmax, int num_sinks, int chunk,
                     uint8_t *__restrict__ codes, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    const int seg = blockIdx.y, c = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    const int t0 = num_sinks + c * chunk;
    if (n_tok < 0 || t0 >= n_tok) return;
    const int t1 = min(n_tok, t0 + chunk);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // this lane's subspace: its 16 centroids (as pairs) and 4 mean entries
    unsigned long long cp[kKmClusters / 2][4];
    const float4 *cs = reinterpret_cast<const float4 *>(cent + (static_cast<size_t>(seg) * kKmSub + lane) * kKmClusters * 4);
#pragma unroll
    for (int p = 0; p < kKmClusters / 2; ++p) {
        const float4 a = __ldg(cs + 2 * p), b = __ldg(cs + 2 * p + 1);
        cp[p][0] = pack2(a.x, b.x);
        cp[p][1] = pack2(a.y, b.y);
        cp[p][2] = pack2(a.z, b.z);
        cp[p][3] = pack2(a.w, b.w);
    }
    const float4 m4 = __ldg(reinterpret_cast<const float4 *>(mu + static_cast<size_t>(seg) * kHeadDim) + lane);
    const char *krows = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    uint32_t *crow = reinterpret_cast<uint32_t *>(codes) + static_cast<size_t>(seg) * nmax * 4;

    // rows t, t + W, ..., t + (U-1) W of this warp; the next group is loaded
    // before the current one is processed, so its latency overlaps the work
    float4 cur[kKmUnroll];
    int t = t0 + warp;
#pragma unroll
    for (int u = 0; u < kKmUnroll; ++u)
        cur[u] = t + u * kKmWarps < t1 ? load4<DT>(krows + static_cast<size_t>(t + u * kKmWarps) * kHeadDim * EB, 4 * lane)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
    while (t < t1) {                                    // warp-uniform
        const int tn = t + kKmUnroll * kKmWarps;
        float4 nxt[kKmUnroll];
#pragma unroll
        for (int u = 0; u < kKmUnroll; ++u)
            nxt[u] = tn + u * kKmWarps < t1
                         ? load4<DT>(krows + static_cast<size_t>(tn + u * kKmWarps) * kHeadDim * EB, 4 * lane)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kKmUnroll; ++u) {
            const int tu = t + u * kKmWarps;
            if (tu < t1) {                              // warp-uniform
                const int a = nearest(cp, __fsub_rn(cur[u].x, m4.x), __fsub_rn(cur[u].y, m4.y),
                                      __fsub_rn(cur[u].z, m4.z), __fsub_rn(cur[u].w, m4.w));
                uint32_t word = static_cast<uint32_t>(a) << (4 * (lane & 7));
#pragma unroll
                for (int off = 1; off < 8; off <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, off);
                if ((lane & 7) == 0) crow[static_cast<size_t>(tu) * 4 + (lane >> 3)] = word;
            }
        }
#pragma unroll
        for (int u = 0; u < kKmUnroll; ++u) cur[u] = nxt[u];
        t = tn;
    }
}

// Exact per-cluster sums and counts of chunk blockIdx.x of segment
// blockIdx.y under the codes of this iteration, into part_sum / part_cnt
// (entry (cluster, dim, subspace) = (a * 4 + i) * 32 + s).
template <int DT>
__global__ void __launch_bounds__(kKaThreads)
kmeans_accum_kernel(const void *__restrict__ K, const int32_t *__restrict__ seq_lens, const float *__restrict__ mu,
                    const uint8_t *__restrict__ codes, int hkv, int nmax, int num_sinks, int chunk, int nchunks,
                    double2 *__restrict__ part_sum, int32_t *__restrict__ part_cnt, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    extern __shared__ __align__(16) unsigned char km_smem[];
    KmAccSmem &A = *reinterpret_cast<KmAccSmem *>(km_smem);
    const int seg = blockIdx.y, c = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    const int t0 = num_sinks + c * chunk;
    if (n_tok < 0 || t0 >= n_tok) return;               // block-uniform
    const int t1 = min(n_tok, t0 + chunk);
    const int d = threadIdx.x, s = d >> 2, i = d & 3;
#pragma unroll
    for (int a = 0; a < kKmClusters; ++a) A.sum[a][d] = make_double2(0.0, 0.0);
    if (i == 0) {
#pragma unroll
        for (int a = 0; a < kKmClusters; ++a) A.cnt[a][s] = 0;
    }
    const float m = __ldg(mu + static_cast<size_t>(seg) * kHeadDim + d);
    const char *krows = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    const uint8_t *cbytes = codes + static_cast<size_t>(seg) * nmax * kCodeBytes + (s >> 1);
    const int shift = 4 * (s & 1);
#pragma unroll 1
    for (int t = t0; t < t1; t += kKaUnroll) {
        float v[kKaUnroll];
        uint32_t cb[kKaUnroll];
#pragma unroll
        for (int u = 0; u < kKaUnroll; ++u) {
            const bool ok = t + u < t1;
            v[u] = ok ? load1<DT>(krows + static_cast<size_t>(t + u) * kHeadDim * EB, d) : 0.f;
            cb[u] = ok ? __ldg(cbytes + static_cast<size_t>(t + u) * kCodeBytes) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kKaUnroll; ++u) {
            if (t + u >= t1) break;
            const int a = static_cast<int>((cb[u] >> shift) & 15u);
            double2 acc = A.sum[a][d];
            const dd r = two_sum(acc.x, static_cast<double>(__fsub_rn(v[u], m)));
            acc.x = r.hi;
            acc.y += r.lo;
            A.sum[a][d] = acc;
            if (i == 0) A.cnt[a][s] += 1;
        }
    }
    // this thread's sums (its own column) and counts -> the chunk's partial
    const size_t pbase = static_cast<size_t>(seg) * nchunks + c;
    double2 *ps = part_sum + pbase * kKmEntries;
#pragma unroll
    for (int a = 0; a < kKmClusters; ++a) {
        const double2 acc = A.sum[a][d];
        const dd r = two_sum(acc.x, acc.y);
        ps[(a * 4 + i) * kKmSub + s] = make_double2(r.hi, r.lo);
    }
    if (i == 0) {
        int32_t *pc = part_cnt + pbase * kKmClusters * kKmSub;
#pragma unroll
        for (int a = 0; a < kKmClusters; ++a) pc[a * kKmSub + s] = A.cnt[a][s];
    }
}

// New centroids of segment blockIdx.x from its chunk partials (chunk order);
// counts (may be null) are written on the last iteration.
__global__ void __launch_bounds__(kKmUpdateThreads)
kmeans_update_kernel(const int32_t *__restrict__ seq_lens, int hkv, int nmax, int num_sinks, int chunk, int nchunks,
                     const double2 *__restrict__ part_sum, const int32_t *__restrict__ part_cnt,
                     float *__restrict__ cent, int32_t *__restrict__ counts, int32_t *status) {
    const int seg = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    const int n_pts = n_tok < 0 ? 0 : max(n_tok - num_sinks, 0);
    const int nch = min(nchunks, (n_pts + chunk - 1) / chunk);
    const double2 *ps = part_sum + static_cast<size_t>(seg) * nchunks * kKmEntries;
    const int32_t *pc = part_cnt + static_cast<size_t>(seg) * nchunks * kKmClusters * kKmSub;
    float *c = cent + static_cast<size_t>(seg) * kKmSub * kKmClusters * 4;
    for (int e = threadIdx.x; e < kKmEntries; e += kKmUpdateThreads) {
        const int a = e / (4 * kKmSub), i = (e / kKmSub) % 4, s = e % kKmSub;
        dd sum = {0.0, 0.0};
        int n = 0;
        for (int ch = 0; ch < nch; ++ch) {
            const double2 v = ps[static_cast<size_t>(ch) * kKmEntries + e];
            sum = dd_merge(sum, dd{v.x, v.y});
            n += pc[static_cast<size_t>(ch) * kKmClusters * kKmSub + a * kKmSub + s];
        }
        if (n > 0) c[(s * kKmClusters + a) * 4 + i] = dd_div_to_float_rn(sum, static_cast<double>(n));
        if (counts && i == 0)
            counts[static_cast<size_t>(seg) * kKmSub * kKmClusters + s * kKmClusters + a] = n;
    }
}

}  // namespace

KmeansLayout kmeans_layout(const sikv_params &p, int num_sms) {
    KmeansLayout L;
    const int segs = p.batch * p.num_kv_heads;
    const int pts = std::max(p.max_seq_len - p.num_sinks, 1);
    // about kKmCtasPerSm accumulation CTAs per SM, chunks of at least 256 tokens
    const int per_seg = std::max(1, std::min(kKmCtasPerSm * num_sms / segs, (pts + 255) / 256));
    L.chunk = (pts + per_seg - 1) / per_seg;
    L.nchunks = (pts + L.chunk - 1) / L.chunk;
    size_t off = kHeaderBytes;
    L.part_sum = off;
    off = align_up(off + static_cast<size_t>(segs) * L.nchunks * kKmEntries * sizeof(double2), 256);
    L.part_cnt = off;
    off = align_up(off + static_cast<size_t>(segs) * L.nchunks * kKmClusters * kKmSub * sizeof(int32_t), 256);
    L.total = off;
    return L;
}

sikv_status launch_kmeans(const sikv_params &p, const KmeansLayout &L, const void *K, const int32_t *seq_lens,
                          const float *mu, const int32_t *init_idx, int iters, uint8_t *codes, float *codebook,
                          int32_t *counts, char *ws, cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    double2 *psum = reinterpret_cast<double2 *>(ws + L.part_sum);
    int32_t *pcnt = reinterpret_cast<int32_t *>(ws + L.part_cnt);
    const bool bf16 = p.dtype == SIKV_DTYPE_BF16;
    auto accum = bf16 ? kmeans_accum_kernel<SIKV_DTYPE_BF16> : kmeans_accum_kernel<SIKV_DTYPE_F32>;
    auto assign = bf16 ? kmeans_assign_kernel<SIKV_DTYPE_BF16> : kmeans_assign_kernel<SIKV_DTYPE_F32>;
    const size_t smem = sizeof(KmAccSmem);
    if (cudaFuncSetAttribute(accum, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return SIKV_ERR_CUDA;
    if (bf16)
        kmeans_init_kernel<SIKV_DTYPE_BF16><<<segs, 256, 0, stream>>>(K, seq_lens, mu, init_idx, codebook,
                                                                      p.num_kv_heads, p.max_seq_len, p.num_sinks,
                                                                      status);
    else
        kmeans_init_kernel<SIKV_DTYPE_F32><<<segs, 256, 0, stream>>>(K, seq_lens, mu, init_idx, codebook,
                                                                     p.num_kv_heads, p.max_seq_len, p.num_sinks,
                                                                     status);
    const dim3 grid(L.nchunks, segs);
    for (int it = 0; it < iters; ++it) {
        const bool last = it == iters - 1;
        assign<<<grid, kKmThreads, 0, stream>>>(K, seq_lens, mu, codebook, p.num_kv_heads, p.max_seq_len,
                                                p.num_sinks, L.chunk, codes, status);
        accum<<<grid, kKaThreads, smem, stream>>>(K, seq_lens, mu, codes, p.num_kv_heads, p.max_seq_len, p.num_sinks,
                                                  L.chunk, L.nchunks, psum, pcnt, status);
        kmeans_update_kernel<<<segs, kKmUpdateThreads, 0, stream>>>(seq_lens, p.num_kv_heads, p.max_seq_len,
                                                                   p.num_sinks, L.chunk, L.nchunks, psum, pcnt,
                                                                   codebook, last ? counts : nullptr, status);
    }
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
