// sikv_sparse_attn: dequantization fused with sparse attention over the sink
// tokens plus the selected tokens.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 3 (64 full-precision sink tokens, token-wise
// codes) and item 4 (dequantization and sparse attention in one pass).
//
// The attended list of a segment is [sinks 0..min(S,N)-1, idx[0..k)].  It is
// split into runs of kSplit positions, one CTA each (split-k):
//   - logits: a sink uses its stored key; a selected token never leaves the
//     compressed domain: q_h . (mu + c[code]) = q_h . mu + sum_s LUT_h[s][code_s]
//     with one 512-entry table per query head of the group;
//   - online-softmax partials (m, l, o) per query head, V read in its storage
//     dtype and accumulated in fp32;
//   - attn_combine merges the partials with log-sum-exp weights.
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kSplit = 128;            // list positions per CTA (== threads)

template <int G>
struct AttnSmem {
    alignas(16) float qs[G][kHeadDim];
    alignas(16) float lut[G][kSubspaces * kClusters];
    alignas(16) float qmu[G];
    alignas(16) float logit[G][kSplit];
    alignas(16) int32_t tok[kSplit];
    alignas(16) float ml[G][2];
    alignas(16) float red[kAttnWarps][G][kHeadDim];   // written with float4 stores
};

template <int DT, int G, bool VQ>
__global__ void __launch_bounds__(kAttnThreads)
attn_partial_kernel(const void *__restrict__ q, const void *__restrict__ K, const void *__restrict__ V,
                    const uint8_t *__restrict__ vq, const uint8_t *__restrict__ codes, const float *__restrict__ codebook,
                    const float *__restrict__ mu, const int32_t *__restrict__ idx,
                    const int32_t *__restrict__ k_per_seq, const int32_t *__restrict__ seq_lens,
                    int hq, int hkv, int nmax, int num_sinks, int kmax, int nsplit, float scale,
                    float *__restrict__ part_o, float2 *__restrict__ part_ml, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    extern __shared__ __align__(16) unsigned char attn_smem[];
    AttnSmem<G> &sh = *reinterpret_cast<AttnSmem<G> *>(attn_smem);
    const int seg = blockIdx.y, split = blockIdx.x, b = seg / hkv, h = seg % hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_tok = load_seq_len(seq_lens, b, nmax, status);
    if (n_tok < 0) return;
    const int ns = min(num_sinks, n_tok);
    const int k = load_topk(k_per_seq, b, kmax, max(n_tok - num_sinks, 0), status);
    if (k < 0) return;
    const int n_list = ns + k, p0 = split * kSplit;
    if (p0 >= n_list) return;

    // query rows of the group, per-head LUTs and q . mu
    const char *qrow = static_cast<const char *>(q) +
                       (static_cast<size_t>(b) * hq + static_cast<size_t>(h) * G) * kHeadDim * EB;
    for (int e = tid; e < G * kHeadDim; e += kAttnThreads)
        sh.qs[e / kHeadDim][e % kHeadDim] = load1<DT>(qrow, e);
    __syncthreads();
    // each codebook row is loaded once (all loads of a thread in flight
    // together) and serves every head of the group
    const float4 *cb = reinterpret_cast<const float4 *>(codebook) + static_cast<size_t>(seg) * kSubspaces * kClusters;
    {
        constexpr int kRows = kSubspaces * kClusters / kAttnThreads;   // 4
        float4 c4[kRows];
#pragma unroll
        for (int i = 0; i < kRows; ++i) c4[i] = __ldg(cb + tid + i * kAttnThreads);
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            const int r = tid + i * kAttnThreads, s = r >> 4;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float v = sh.qs[g][4 * s] * c4[i].x;
                v = fmaf(sh.qs[g][4 * s + 1], c4[i].y, v);
                v = fmaf(sh.qs[g][4 * s + 2], c4[i].z, v);
                v = fmaf(sh.qs[g][4 * s + 3], c4[i].w, v);
                sh.lut[g][r] = v;
            }
        }
    }
    const float4 m4 = __ldg(reinterpret_cast<const float4 *>(mu + static_cast<size_t>(seg) * kHeadDim) + lane);
    for (int g = warp; g < G; g += kAttnWarps) {
        double a = static_cast<double>(sh.qs[g][4 * lane]) * m4.x;
        a = fma(static_cast<double>(sh.qs[g][4 * lane + 1]), static_cast<double>(m4.y), a);
        a = fma(static_cast<double>(sh.qs[g][4 * lane + 2]), static_cast<double>(m4.z), a);
        a = fma(static_cast<double>(sh.qs[g][4 * lane + 3]), static_cast<double>(m4.w), a);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (lane == 0) sh.qmu[g] = static_cast<float>(a);
    }
    __syncthreads();

    // logits: one list position per thread
    const size_t kv_seg = static_cast<size_t>(seg) * nmax;
    {
        const int pos = p0 + tid;
        int t = -1;
        float lg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) lg[g] = -INFINITY;
        if (pos < n_list) {
            if (pos < ns) {
                t = pos;
                const char *krow = static_cast<const char *>(K) + (kv_seg + t) * kHeadDim * EB;
                float acc[G];
#pragma unroll
                for (int g = 0; g < G; ++g) acc[g] = 0.f;
                for (int c = 0; c < kHeadDim; c += 4) {
                    const float4 kv = load4<DT>(krow, c);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        acc[g] = fmaf(sh.qs[g][c], kv.x, acc[g]);
                        acc[g] = fmaf(sh.qs[g][c + 1], kv.y, acc[g]);
                        acc[g] = fmaf(sh.qs[g][c + 2], kv.z, acc[g]);
                        acc[g] = fmaf(sh.qs[g][c + 3], kv.w, acc[g]);
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) lg[g] = acc[g] * scale;
            } else {
                t = __ldg(idx + static_cast<size_t>(seg) * kmax + (pos - ns));
                if (t < num_sinks || t >= n_tok) {
                    flag_error(status, SIKV_DEVERR_INDEX);
                    t = -1;
                } else {
                    const uint4 row = __ldg(reinterpret_cast<const uint4 *>(codes) + kv_seg + t);
                    const uint32_t w[4] = {row.x, row.y, row.z, row.w};
                    float acc[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) acc[g] = 0.f;
#pragma unroll
                    for (int s = 0; s < kSubspaces; ++s) {
                        const int j = (w[s >> 3] >> (4 * (s & 7))) & 15;
#pragma unroll
                        for (int g = 0; g < G; ++g) acc[g] += sh.lut[g][s * kClusters + j];
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) lg[g] = (acc[g] + sh.qmu[g]) * scale;
                }
            }
        }
        sh.tok[tid] = t;
#pragma unroll
        for (int g = 0; g < G; ++g) sh.logit[g][tid] = (t >= 0) ? lg[g] : -INFINITY;
    }
    __syncthreads();

    // softmax statistics of this run (fixed reduction order)
    for (int g = warp; g < G; g += kAttnWarps) {
        float mx = -INFINITY;
        for (int i = lane; i < kSplit; i += 32) mx = fmaxf(mx, sh.logit[g][i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float l = 0.f;
        for (int i = lane; i < kSplit; i += 32) {
            const float lv = sh.logit[g][i];
            const float pv = (lv == -INFINITY) ? 0.f : expf(lv - mx);
            sh.logit[g][i] = pv;
            l += pv;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            sh.ml[g][0] = mx;
            sh.ml[g][1] = l;
        }
    }
    __syncthreads();

    // o_h = sum_i p_h[i] V[t_i]; warp w takes rows w, w+4, ...; lane owns dims 4l..4l+3
    float o[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) o[g][0] = o[g][1] = o[g][2] = o[g][3] = 0.f;
    // 8 value rows in flight per warp
    constexpr int kVRows = 8;
    const int n_here = min(kSplit, n_list - p0);
#pragma unroll 1
    for (int i0 = warp; i0 < n_here; i0 += kAttnWarps * kVRows) {
        float4 v[kVRows];
#pragma unroll
        for (int u = 0; u < kVRows; ++u) {
            const int i = i0 + u * kAttnWarps;
            const int t = (i < n_here) ? sh.tok[i] : -1;
            if (t < 0)
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            else if (VQ && t >= num_sinks)   // a selected token's 2-bit row (sinks read V)
                v[u] = vq_decode4(vq + (kv_seg + t) * kVqRowBytes, lane);
            else
                v[u] = load4<DT>(static_cast<const char *>(V) + (kv_seg + t) * kHeadDim * EB, lane * 4);
        }
#pragma unroll
        for (int u = 0; u < kVRows; ++u) {
            const int i = i0 + u * kAttnWarps;
            if (i >= n_here) break;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float pv = sh.logit[g][i];     // 0 for a skipped entry
                o[g][0] = fmaf(pv, v[u].x, o[g][0]);
                o[g][1] = fmaf(pv, v[u].y, o[g][1]);
                o[g][2] = fmaf(pv, v[u].z, o[g][2]);
                o[g][3] = fmaf(pv, v[u].w, o[g][3]);
            }
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
        *reinterpret_cast<float4 *>(&sh.red[warp][g][lane * 4]) = make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
    __syncthreads();
    const size_t pbase = (static_cast<size_t>(seg) * nsplit + split) * G;
    for (int e = tid; e < G * kHeadDim; e += kAttnThreads) {
        const int g = e / kHeadDim, c = e % kHeadDim;
        float acc = sh.red[0][g][c];
#pragma unroll
        for (int w = 1; w < kAttnWarps; ++w) acc += sh.red[w][g][c];
        part_o[(pbase + g) * kHeadDim + c] = acc;
    }
    if (tid < G) part_ml[pbase + tid] = make_float2(sh.ml[tid][0], sh.ml[tid][1]);
}

template <int DT>
__global__ void __launch_bounds__(kHeadDim)
attn_combine_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml,
                    const int32_t *__restrict__ k_per_seq, const int32_t *__restrict__ seq_lens,
                    int hq, int hkv, int nmax, int num_sinks, int kmax, int nsplit, void *out) {
    const int g = blockIdx.x, seg = blockIdx.y, b = seg / hkv, h = seg % hkv, c = threadIdx.x;
    const int group = hq / hkv;
    const int n_tok = __ldg(seq_lens + b);
    if (n_tok < 0 || n_tok > nmax) return;
    const int k = __ldg(k_per_seq + b);
    if (k < 0 || k > kmax || k > max(n_tok - num_sinks, 0)) return;
    const int n_list = min(num_sinks, n_tok) + k;
    const int used = (n_list + kSplit - 1) / kSplit;
    float mx = -INFINITY;
    for (int sp = 0; sp < used; ++sp) mx = fmaxf(mx, part_ml[(static_cast<size_t>(seg) * nsplit + sp) * group + g].x);
    float l = 0.f, acc = 0.f;
    if (mx != -INFINITY) {
        for (int sp = 0; sp < used; ++sp) {
            const size_t pb = (static_cast<size_t>(seg) * nsplit + sp) * group + g;
            const float2 ml = part_ml[pb];
            const float wgt = (ml.x == -INFINITY) ? 0.f : expf(ml.x - mx);
            l = fmaf(ml.y, wgt, l);
            acc = fmaf(part_o[pb * kHeadDim + c], wgt, acc);
        }
    }
    const float r = (l > 0.f) ? acc / l : 0.f;
    const size_t orow = (static_cast<size_t>(b) * hq + static_cast<size_t>(h) * group + g) * kHeadDim + c;
    if (DT == SIKV_DTYPE_F32)
        static_cast<float *>(out)[orow] = r;
    else
        static_cast<unsigned short *>(out)[orow] = static_cast<unsigned short>(f32_to_bf16_bits(r));
}

template <int DT, int G, bool VQ>
sikv_status launch_partial(const sikv_params &p, const void *q, const void *K, const void *V, const uint8_t *vq,
                           const uint8_t *codes, const float *codebook, const float *mu,
                           const int32_t *idx, const int32_t *k_per_seq, const int32_t *seq_lens,
                           const AttnLayout &L, char *ws, float scale, int32_t *status,
                           cudaStream_t stream) {
    const size_t smem = sizeof(AttnSmem<G>);
    auto kern = attn_partial_kernel<DT, G, VQ>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SIKV_ERR_CUDA;
    const dim3 grid(L.nsplit, p.batch * p.num_kv_heads);
    kern<<<grid, kAttnThreads, smem, stream>>>(q, K, V, vq, codes, codebook, mu, idx, k_per_seq, seq_lens,
                                               p.num_q_heads, p.num_kv_heads, p.max_seq_len, p.num_sinks,
                                               p.max_topk, L.nsplit, scale,
                                               reinterpret_cast<float *>(ws + L.part_o),
                                               reinterpret_cast<float2 *>(ws + L.part_ml), status);
    return SIKV_OK;
}

template <int DT, bool VQ>
sikv_status dispatch_group(int group, const sikv_params &p, const void *q, const void *K, const void *V,
                           const uint8_t *vq, const uint8_t *codes, const float *codebook, const float *mu,
                           const int32_t *idx, const int32_t *k_per_seq, const int32_t *seq_lens,
                           const AttnLayout &L, char *ws, float scale, int32_t *status,
                           cudaStream_t stream) {
#define SIKV_G(NG) \
    case NG:       \
        return launch_partial<DT, NG, VQ>(p, q, K, V, vq, codes, codebook, mu, idx, k_per_seq, seq_lens, L, ws, scale, status, stream)
    switch (group) {
        SIKV_G(1);
        SIKV_G(2);
        SIKV_G(3);
        SIKV_G(4);
        SIKV_G(5);
        SIKV_G(6);
        SIKV_G(7);
        SIKV_G(8);
        default:
            return SIKV_ERR_UNSUPPORTED;
    }
#undef SIKV_G
}

}  // namespace

AttnLayout attn_layout(const sikv_params &p, size_t base) {
    AttnLayout L;
    const int group = p.num_q_heads / p.num_kv_heads;
    const size_t segs = static_cast<size_t>(p.batch) * p.num_kv_heads;
    L.split = kSplit;
    L.nsplit = (p.num_sinks + p.max_topk + kSplit - 1) / kSplit;
    if (L.nsplit < 1) L.nsplit = 1;
    size_t off = align_up(base, 256);
    L.part_o = off;
    off = align_up(off + segs * L.nsplit * group * kHeadDim * sizeof(float), 256);
    L.part_ml = off;
    off = align_up(off + segs * L.nsplit * group * sizeof(float2), 256);
    L.total = off;
    return L;
}

sikv_status launch_sparse_attn(const sikv_params &p, const void *q, const void *K, const void *V,
                               const uint8_t *vq, const uint8_t *codes, const float *codebook, const float *mu,
                               const int32_t *idx, const int32_t *k_per_seq,
                               const int32_t *seq_lens, void *out, char *ws, size_t attn_base,
                               int32_t *status, cudaStream_t stream) {
    const AttnLayout L = attn_layout(p, attn_base);
    const int group = p.num_q_heads / p.num_kv_heads;
    const float scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf(static_cast<float>(p.head_dim));
    sikv_status st;
    if (p.dtype == SIKV_DTYPE_BF16)
        st = vq ? dispatch_group<SIKV_DTYPE_BF16, true>(group, p, q, K, V, vq, codes, codebook, mu, idx, k_per_seq,
                                                        seq_lens, L, ws, scale, status, stream)
                : dispatch_group<SIKV_DTYPE_BF16, false>(group, p, q, K, V, vq, codes, codebook, mu, idx, k_per_seq,
                                                         seq_lens, L, ws, scale, status, stream);
    else
        st = vq ? dispatch_group<SIKV_DTYPE_F32, true>(group, p, q, K, V, vq, codes, codebook, mu, idx, k_per_seq,
                                                       seq_lens, L, ws, scale, status, stream)
                : dispatch_group<SIKV_DTYPE_F32, false>(group, p, q, K, V, vq, codes, codebook, mu, idx, k_per_seq,
                                                        seq_lens, L, ws, scale, status, stream);
    if (st != SIKV_OK) return st;
    const dim3 grid(group, p.batch * p.num_kv_heads);
    const float *po = reinterpret_cast<const float *>(ws + L.part_o);
    const float2 *pml = reinterpret_cast<const float2 *>(ws + L.part_ml);
    if (p.dtype == SIKV_DTYPE_BF16)
        attn_combine_kernel<SIKV_DTYPE_BF16><<<grid, kHeadDim, 0, stream>>>(
            po, pml, k_per_seq, seq_lens, p.num_q_heads, p.num_kv_heads, p.max_seq_len, p.num_sinks,
            p.max_topk, L.nsplit, out);
    else
        attn_combine_kernel<SIKV_DTYPE_F32><<<grid, kHeadDim, 0, stream>>>(
            po, pml, k_per_seq, seq_lens, p.num_q_heads, p.num_kv_heads, p.max_seq_len, p.num_sinks,
            p.max_topk, L.nsplit, out);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
