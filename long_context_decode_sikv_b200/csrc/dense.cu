// Dense comparison baselines: full-precision scoring (q_bar . K[t] for every
// token) and dense decode attention over every token.  Not the method: they
// are what "Self-Indexing KVCache: Predicting Sparse Attention from
// Compressed Keys" compares its compressed-domain retrieval (technical
// summary §2.1 item 2) and its sparse attention (item 4) against, written
// here so that both sides are measured on the same GPU with kernels of the
// same library.
//
// Both kernels stream K (and V) once.  Scoring: a warp takes 8 consecutive
// tokens per iteration; lane l loads columns 4l..4l+3 of each row (one
// coalesced row per warp instruction) and a shuffle reduction completes each
// dot product.  Attention: one token per lane for the logits (below), one
// online softmax per warp, the warps merged once per CTA into (m, l, o)
// partials, and a second kernel merging the partials of each segment.
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kDenseThreads = 256;
constexpr int kDenseWarps = kDenseThreads / 32;
constexpr int kDenseRows = 8;                 // tokens per warp iteration
constexpr int kDenseScoreChunk = 4096;        // tokens per CTA (scoring)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int DT>
__global__ void __launch_bounds__(kDenseThreads)
dense_score_kernel(const void *__restrict__ q, const void *__restrict__ K, const int32_t *__restrict__ seq_lens,
                   int hq, int hkv, int nmax, int num_sinks, float *__restrict__ scores, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    const int seg = blockIdx.y, b = seg / hkv, h = seg % hkv, group = hq / hkv;
    const int n_tok = load_seq_len(seq_lens, b, nmax, status);
    if (n_tok < 0) return;
    const int t_begin = blockIdx.x * kDenseScoreChunk;
    if (t_begin >= n_tok) return;
    const int t_end = min(t_begin + kDenseScoreChunk, n_tok);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // lane l keeps q_bar[4l..4l+3] (the summed group query, fp32)
    const char *qrow = static_cast<const char *>(q) + (static_cast<size_t>(b) * hq + static_cast<size_t>(h) * group) * kHeadDim * EB;
    float4 qb = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < group; ++g) {
        const float4 v = load4<DT>(qrow + static_cast<size_t>(g) * kHeadDim * EB, 4 * lane);
        qb.x += v.x;
        qb.y += v.y;
        qb.z += v.z;
        qb.w += v.w;
    }
    const char *krows = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    float *srow = scores + static_cast<size_t>(seg) * nmax;
#pragma unroll 1
    for (int t0 = t_begin + warp * kDenseRows; t0 < t_end; t0 += kDenseWarps * kDenseRows) {
        float4 kv[kDenseRows];
#pragma unroll
        for (int u = 0; u < kDenseRows; ++u)
            kv[u] = (t0 + u < t_end) ? load4<DT>(krows + static_cast<size_t>(t0 + u) * kHeadDim * EB, 4 * lane)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kDenseRows; ++u) {
            float d = qb.x * kv[u].x;
            d = fmaf(qb.y, kv[u].y, d);
            d = fmaf(qb.z, kv[u].z, d);
            d = fmaf(qb.w, kv[u].w, d);
            d = warp_sum(d);
            const int t = t0 + u;
            if (lane == u && t < t_end) srow[t] = (t >= num_sinks) ? d : -INFINITY;
        }
    }
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

constexpr int kDenseStage = 8192;     // bytes of key rows (and of value rows) a warp stages per batch

// Dense attention partials.  Warp w takes batches of consecutive tokens (32
// bf16 rows or 16 fp32 rows: 8 KB of keys and 8 KB of values), staged into
// its shared-memory slots with cp.async, so that a whole batch is in flight
// at once without holding registers.  Logits: one token per lane, reading
// its key row piece by piece (the piece index is XOR-swizzled with the row,
// so the 8 lanes of each shared-memory phase hit distinct banks) against the
// group's queries (broadcast reads).  Then the warp folds the batch into its
// online softmax and accumulates the value rows, lane l owning columns
// 4l..4l+3.
template <int DT, int GM>
__global__ void __launch_bounds__(kDenseThreads, 1)
dense_attn_partial_kernel(const void *__restrict__ q, const void *__restrict__ K, const void *__restrict__ V,
                          const int32_t *__restrict__ seq_lens, int hq, int hkv, int nmax, int chunk, float scale,
                          float *__restrict__ part_o, float2 *__restrict__ part_ml, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    constexpr int kRowBytes = kHeadDim * EB;
    constexpr int kPieces = kRowBytes / 16;               // 16 (bf16) or 32 (fp32)
    constexpr int kPer = 16 / EB;                          // columns per piece: 8 or 4
    constexpr int kTok = kDenseStage / kRowBytes;          // tokens per batch: 32 or 16
    extern __shared__ __align__(16) unsigned char dense_smem[];
    float (*qs)[kHeadDim] = reinterpret_cast<float (*)[kHeadDim]>(dense_smem);                    // [GM][128]
    float (*red_o)[GM][kHeadDim] = reinterpret_cast<float (*)[GM][kHeadDim]>(dense_smem + GM * kHeadDim * 4);
    float *red_m = reinterpret_cast<float *>(dense_smem + (1 + kDenseWarps) * GM * kHeadDim * 4);  // [kFW][GM]
    float *red_l = red_m + kDenseWarps * GM;
    unsigned char *stage = dense_smem + (1 + kDenseWarps) * GM * kHeadDim * 4 + 2 * kDenseWarps * GM * 4;
    stage = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(stage) + 127) & ~uintptr_t(127));
    const int seg = blockIdx.y, b = seg / hkv, h = seg % hkv, group = hq / hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char *ks = stage + static_cast<size_t>(warp) * 2 * kDenseStage, *vs = ks + kDenseStage;
    int n_tok = load_seq_len(seq_lens, b, nmax, status);
    if (n_tok < 0) n_tok = 0;
    const int t_begin = blockIdx.x * chunk, t_end = min(t_begin + chunk, n_tok);
    const char *qrow = static_cast<const char *>(q) + (static_cast<size_t>(b) * hq + static_cast<size_t>(h) * group) * kHeadDim * EB;
    for (int e = threadIdx.x; e < GM * kHeadDim; e += kDenseThreads) {
        const int g = e / kHeadDim, d = e % kHeadDim;
        qs[g][d] = (g < group) ? load1<DT>(qrow + static_cast<size_t>(g) * kHeadDim * EB, d) : 0.f;
    }
    __syncthreads();
    float m[GM], l[GM], o[GM][4];
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
        o[g][0] = o[g][1] = o[g][2] = o[g][3] = 0.f;
    }
    const char *krows = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kRowBytes;
    const char *vrows = static_cast<const char *>(V) + static_cast<size_t>(seg) * nmax * kRowBytes;
#pragma unroll 1
    for (int t0 = t_begin + kTok * warp; t0 < t_end; t0 += kTok * kDenseWarps) {
        const int nb = min(kTok, t_end - t0);
        // stage the batch: piece c of key row j at slot c ^ (j mod kPieces)
#pragma unroll 1
        for (int i = lane; i < nb * kPieces; i += 32) {
            const int j = i / kPieces, c = i % kPieces;
            const size_t src = static_cast<size_t>(t0 + j) * kRowBytes + 16 * c;
            cp_async16(ks + j * kRowBytes + 16 * (c ^ (j & (kPieces - 1))), krows + src);
            cp_async16(vs + j * kRowBytes + 16 * c, vrows + src);
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
        __syncwarp();
        const bool valid = lane < nb;
        float acc[GM];
#pragma unroll
        for (int g = 0; g < GM; ++g) acc[g] = 0.f;
        if (lane < kTok) {
            const unsigned char *kr = ks + lane * kRowBytes;
#pragma unroll 4
            for (int c = 0; c < kPieces; ++c) {
                const uint4 w = *reinterpret_cast<const uint4 *>(kr + 16 * (c ^ (lane & (kPieces - 1))));
                float kf[kPer];
                if (DT == SIKV_DTYPE_BF16) {
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        kf[2 * i] = bf16_lo(ww[i]);
                        kf[2 * i + 1] = bf16_hi(ww[i]);
                    }
                } else {
                    kf[0] = __uint_as_float(w.x);
                    kf[1] = __uint_as_float(w.y);
                    kf[2] = __uint_as_float(w.z);
                    kf[3] = __uint_as_float(w.w);
                }
#pragma unroll
                for (int g = 0; g < GM; ++g) {
#pragma unroll
                    for (int i = 0; i < kPer; i += 4) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(&qs[g][kPer * c + i]);
                        acc[g] = fmaf(q4.x, kf[i], acc[g]);
                        acc[g] = fmaf(q4.y, kf[i + 1], acc[g]);
                        acc[g] = fmaf(q4.z, kf[i + 2], acc[g]);
                        acc[g] = fmaf(q4.w, kf[i + 3], acc[g]);
                    }
                }
            }
        }
        float pr[GM];
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            const float lg = (valid && g < group) ? acc[g] * scale : -INFINITY;
            float mx = lg;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mn = fmaxf(m[g], mx);
            const float alpha = (m[g] == -INFINITY) ? 0.f : __expf(m[g] - mn);
            pr[g] = (lg == -INFINITY) ? 0.f : __expf(lg - mn);
            l[g] = fmaf(l[g], alpha, warp_sum(pr[g]));
            m[g] = mn;
#pragma unroll
            for (int i = 0; i < 4; ++i) o[g][i] *= alpha;
        }
#pragma unroll 4
        for (int j = 0; j < nb; ++j) {
            float4 vv;
            if (DT == SIKV_DTYPE_BF16) {
                const uint2 w = *reinterpret_cast<const uint2 *>(vs + j * kRowBytes + 8 * lane);
                vv = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
            } else {
                vv = *reinterpret_cast<const float4 *>(vs + j * kRowBytes + 16 * lane);
            }
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                const float w = __shfl_sync(0xffffffffu, pr[g], j);
                o[g][0] = fmaf(w, vv.x, o[g][0]);
                o[g][1] = fmaf(w, vv.y, o[g][1]);
                o[g][2] = fmaf(w, vv.z, o[g][2]);
                o[g][3] = fmaf(w, vv.w, o[g][3]);
            }
        }
        __syncwarp();                      // the slots are refilled by the next batch
    }
    // merge the warps (fixed order), write this CTA's partial
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        *reinterpret_cast<float4 *>(&red_o[warp][g][4 * lane]) = make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
        if (lane == 0) {
            red_m[warp * GM + g] = m[g];
            red_l[warp * GM + g] = l[g];
        }
    }
    __syncthreads();
    const size_t pb = (static_cast<size_t>(seg) * gridDim.x + blockIdx.x) * GM;
    for (int e = threadIdx.x; e < GM * kHeadDim; e += kDenseThreads) {
        const int g = e / kHeadDim, d = e % kHeadDim;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDenseWarps; ++w) mx = fmaxf(mx, red_m[w * GM + g]);
        float acc = 0.f, ls = 0.f;
        if (mx != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDenseWarps; ++w) {
                const float f = (red_m[w * GM + g] == -INFINITY) ? 0.f : __expf(red_m[w * GM + g] - mx);
                acc = fmaf(f, red_o[w][g][d], acc);
                ls = fmaf(f, red_l[w * GM + g], ls);
            }
        }
        part_o[(pb + g) * kHeadDim + d] = acc;
        if (d == 0) part_ml[pb + g] = make_float2(mx, ls);
    }
}

template <int GM>
constexpr size_t dense_attn_smem() {
    return ((1 + kDenseWarps) * GM * kHeadDim * 4 + 2 * kDenseWarps * GM * 4 + 127) / 128 * 128 + 127 +
           static_cast<size_t>(kDenseWarps) * 2 * kDenseStage;
}

template <int DT, int GM>
__global__ void __launch_bounds__(kHeadDim)
dense_attn_combine_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int hq, int hkv,
                          int nchunks, void *__restrict__ out) {
    // block (segment, head g); thread d.  The chunks' (m, l) pairs are read
    // once into shared memory, their weights formed, then each thread sums
    // its column over the chunks with the loads unrolled.
    __shared__ float wts[1024];
    __shared__ float inv_l;
    const int seg = blockIdx.x, g = blockIdx.y, b = seg / hkv, h = seg % hkv, group = hq / hkv, d = threadIdx.x;
    if (g >= group) return;
    const size_t base = static_cast<size_t>(seg) * nchunks;
    __shared__ float mx_s;
    if (d < 32) {
        float mx = -INFINITY;
        for (int c = d; c < nchunks; c += 32) mx = fmaxf(mx, part_ml[(base + c) * GM + g].x);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float l = 0.f;
        for (int c = d; c < nchunks; c += 32) {
            const float2 ml = part_ml[(base + c) * GM + g];
            const float f = (ml.x == -INFINITY || mx == -INFINITY) ? 0.f : __expf(ml.x - mx);
            wts[c] = f;
            l = fmaf(ml.y, f, l);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (d == 0) {
            inv_l = (l > 0.f) ? __fdividef(1.f, l) : 0.f;
            mx_s = mx;
        }
    }
    __syncthreads();
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < nchunks; ++c) acc = fmaf(wts[c], part_o[((base + c) * GM + g) * kHeadDim + d], acc);
    const float r = acc * inv_l;
    const size_t orow = (static_cast<size_t>(b) * hq + static_cast<size_t>(h) * group + g) * kHeadDim + d;
    if (DT == SIKV_DTYPE_F32)
        static_cast<float *>(out)[orow] = r;
    else
        static_cast<unsigned short *>(out)[orow] = static_cast<unsigned short>(f32_to_bf16_bits(r));
}

template <int DT, int GM>
sikv_status launch_dense_attn_t(const sikv_params &p, const void *q, const void *K, const void *V,
                                const int32_t *seq_lens, void *out, const DenseAttnLayout &L, char *ws,
                                int32_t *status, cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    const float scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf(static_cast<float>(p.head_dim));
    float *po = reinterpret_cast<float *>(ws + L.part_o);
    float2 *pml = reinterpret_cast<float2 *>(ws + L.part_ml);
    auto kern = dense_attn_partial_kernel<DT, GM>;
    const size_t smem = dense_attn_smem<GM>();
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return SIKV_ERR_CUDA;
    kern<<<dim3(L.nchunks, segs), kDenseThreads, smem, stream>>>(q, K, V, seq_lens, p.num_q_heads, p.num_kv_heads,
                                                                 p.max_seq_len, L.chunk, scale, po, pml, status);
    dense_attn_combine_kernel<DT, GM><<<dim3(segs, GM), kHeadDim, 0, stream>>>(po, pml, p.num_q_heads,
                                                                               p.num_kv_heads, L.nchunks, out);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace

DenseAttnLayout dense_attn_layout(const sikv_params &p, size_t base) {
    DenseAttnLayout L;
    const size_t segs = static_cast<size_t>(p.batch) * p.num_kv_heads;
    const int gm = (p.num_q_heads / p.num_kv_heads) <= 4 ? 4 : 8;
    // enough CTAs to fill the device a few times over, each a multiple of
    // the warps' 8-token steps
    L.chunk = 2048;
    if ((p.max_seq_len + L.chunk - 1) / L.chunk > 1024)          // the combine holds at most 1024 weights
        L.chunk = ((p.max_seq_len + 1023) / 1024 + 255) / 256 * 256;
    L.nchunks = (p.max_seq_len + L.chunk - 1) / L.chunk;
    size_t off = align_up(base, 256);
    L.part_o = off;
    off = align_up(off + segs * L.nchunks * gm * kHeadDim * sizeof(float), 256);
    L.part_ml = off;
    off = align_up(off + segs * L.nchunks * gm * sizeof(float2), 256);
    L.total = off;
    return L;
}

sikv_status launch_dense_score(const sikv_params &p, const void *q, const void *K, const int32_t *seq_lens,
                               float *scores, int32_t *status, cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    const dim3 grid((p.max_seq_len + kDenseScoreChunk - 1) / kDenseScoreChunk, segs);
    if (p.dtype == SIKV_DTYPE_BF16)
        dense_score_kernel<SIKV_DTYPE_BF16><<<grid, kDenseThreads, 0, stream>>>(
            q, K, seq_lens, p.num_q_heads, p.num_kv_heads, p.max_seq_len, p.num_sinks, scores, status);
    else
        dense_score_kernel<SIKV_DTYPE_F32><<<grid, kDenseThreads, 0, stream>>>(
            q, K, seq_lens, p.num_q_heads, p.num_kv_heads, p.max_seq_len, p.num_sinks, scores, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

sikv_status launch_dense_attn(const sikv_params &p, const void *q, const void *K, const void *V,
                              const int32_t *seq_lens, void *out, char *ws, size_t base, int32_t *status,
                              cudaStream_t stream) {
    const DenseAttnLayout L = dense_attn_layout(p, base);
    const int gm = (p.num_q_heads / p.num_kv_heads) <= 4 ? 4 : 8;
    if (p.dtype == SIKV_DTYPE_BF16)
        return gm == 4 ? launch_dense_attn_t<SIKV_DTYPE_BF16, 4>(p, q, K, V, seq_lens, out, L, ws, status, stream)
                       : launch_dense_attn_t<SIKV_DTYPE_BF16, 8>(p, q, K, V, seq_lens, out, L, ws, status, stream);
    return gm == 4 ? launch_dense_attn_t<SIKV_DTYPE_F32, 4>(p, q, K, V, seq_lens, out, L, ws, status, stream)
                   : launch_dense_attn_t<SIKV_DTYPE_F32, 8>(p, q, K, V, seq_lens, out, L, ws, status, stream);
}

}  // namespace sikv
