// sikv_topk: exact top-k of the compressed-domain scores, without a full sort.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 2 (top-k selection on the LUT-GEMV scores).
// Order: score descending, then token index ascending (-0.0 == +0.0).
//
// One CTA of 1024 threads per segment:
//   1. min / max of the scores;
//   2. 4096-bin histogram linear in the score over [min, max] (a monotone
//      map, so every token in a higher bin has a strictly higher score);
//      the bin b* holding the k-th score is found by a top-down scan;
//   3. the tokens of bin b* are compacted into shared memory and an 8-bit
//      radix select on their order-preserving keys finds the exact k-th key T
//      and how many tokens equal to T are needed (falls back to radix passes
//      over global memory when bin b* does not fit);
//   4. every key > T and the lowest-index keys == T are emitted in ascending
//      token order: each warp owns a contiguous run of 32-token groups
//      (coalesced reads, ballot counts), one scan over the warps places the
//      runs (no atomics).
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBins = 4096;
constexpr int kCap = 12288;

struct TopkSmem {
    uint32_t hist[kBins];
    uint32_t ckey[kCap];
    int32_t cidx[kCap];
    uint32_t wtot[kTopkWarps + 1];
    float rmin[kTopkWarps], rmax[kTopkWarps];
    uint32_t sc[8];
};

struct Binner {
    float lo, inv;
    bool flat;
    __device__ __forceinline__ int operator()(float s) const {
        if (flat) return 0;
        const int b = __float2int_rz((s - lo) * inv);
        return min(max(b, 0), kBins - 1);
    }
};

// Exclusive prefix sum of one value per thread over the whole CTA (1024
// threads, thread order); *total receives the sum.  Contains __syncthreads.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *wtot, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = wtot[lane];
        uint32_t wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        wtot[lane] = wi - w;
        if (lane == 31) wtot[kTopkWarps] = wi;
    }
    __syncthreads();
    const uint32_t res = wtot[warp] + incl - v;
    *total = wtot[kTopkWarps];
    __syncthreads();
    return res;
}

// Finds, in a 256-bin digit histogram scanned from digit 255 down, the digit
// where the running count first reaches `need`; returns it in sc[0] and the
// count above it in sc[1].  Executed by warp 0; caller synchronizes.
__device__ __forceinline__ void find_digit(const uint32_t *hist, uint32_t need, uint32_t *sc) {
    const int lane = threadIdx.x & 31;
    uint32_t loc = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) loc += hist[255 - (lane * 8 + i)];
    uint32_t incl = loc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    uint32_t above = incl - loc;
    if (above < need && need <= incl) {
        for (int i = 0; i < 8; ++i) {
            const int d = 255 - (lane * 8 + i);
            if (above + hist[d] >= need) {
                sc[0] = static_cast<uint32_t>(d);
                sc[1] = above;
                break;
            }
            above += hist[d];
        }
    }
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
            const int32_t *__restrict__ k_per_seq, int hkv, int nmax, int num_sinks, int kmax,
            int32_t *__restrict__ idx, int32_t *status) {
    extern __shared__ __align__(16) unsigned char topk_smem[];
    TopkSmem &sh = *reinterpret_cast<TopkSmem *>(topk_smem);
    const int seg = blockIdx.x, b = seg / hkv, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t *out = idx + static_cast<size_t>(seg) * kmax;
    const int n_tok = load_seq_len(seq_lens, b, nmax, status);
    if (n_tok < 0) return;
    const int n = max(n_tok - num_sinks, 0);
    const int k = load_topk(k_per_seq, b, kmax, n, status);
    if (k < 0) return;
    const float *srow = scores + static_cast<size_t>(seg) * nmax;

    if (k > 0) {
        // 1. range of the scores
        float lo = INFINITY, hi = -INFINITY;
        for (int t = num_sinks + tid; t < n_tok; t += kTopkThreads) {
            const float s = srow[t];
            lo = fminf(lo, s);
            hi = fmaxf(hi, s);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        if (lane == 0) {
            sh.rmin[warp] = lo;
            sh.rmax[warp] = hi;
        }
        for (int i = tid; i < kBins; i += kTopkThreads) sh.hist[i] = 0;
        __syncthreads();
        lo = sh.rmin[0];
        hi = sh.rmax[0];
        for (int w = 1; w < kTopkWarps; ++w) {
            lo = fminf(lo, sh.rmin[w]);
            hi = fmaxf(hi, sh.rmax[w]);
        }
        Binner bin;
        const float width = hi - lo;
        bin.lo = lo;
        bin.inv = static_cast<float>(kBins) / width;
        bin.flat = !(isfinite(width) && width > 0.0f && isfinite(bin.inv));

        // 2. histogram and the threshold bin
        for (int t = num_sinks + tid; t < n_tok; t += kTopkThreads) atomicAdd(&sh.hist[bin(srow[t])], 1u);
        __syncthreads();
        uint32_t loc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) loc += sh.hist[kBins - 1 - (tid * 4 + i)];
        uint32_t tot;
        uint32_t above = block_excl_scan(loc, sh.wtot, &tot);
        if (above < static_cast<uint32_t>(k) && static_cast<uint32_t>(k) <= above + loc) {
            for (int i = 0; i < 4; ++i) {
                const int bb = kBins - 1 - (tid * 4 + i);
                if (above + sh.hist[bb] >= static_cast<uint32_t>(k)) {
                    sh.sc[2] = static_cast<uint32_t>(bb);
                    sh.sc[3] = above;
                    sh.sc[4] = sh.hist[bb];
                    break;
                }
                above += sh.hist[bb];
            }
        }
        if (tid == 0) sh.sc[5] = 0;
        __syncthreads();
        const int bstar = static_cast<int>(sh.sc[2]);
        const uint32_t in_above = sh.sc[3], in_bin = sh.sc[4];

        // 3. exact key of the k-th element among bin b*
        const bool fits = in_bin <= static_cast<uint32_t>(kCap);
        if (fits) {
            for (int t = num_sinks + tid; t < n_tok; t += kTopkThreads) {
                const float s = srow[t];
                if (bin(s) == bstar) {
                    const uint32_t slot = atomicAdd(&sh.sc[5], 1u);
                    if (slot < static_cast<uint32_t>(kCap)) {
                        sh.ckey[slot] = score_key(s);
                        sh.cidx[slot] = t;
                    }
                }
            }
            __syncthreads();
        }
        uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(k) - in_above;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += kTopkThreads) sh.hist[i] = 0;
            __syncthreads();
            if (fits) {
                for (uint32_t e = tid; e < in_bin; e += kTopkThreads) {
                    const uint32_t key = sh.ckey[e];
                    if (((key ^ prefix) & mask) == 0) atomicAdd(&sh.hist[(key >> shift) & 255u], 1u);
                }
            } else {
                for (int t = num_sinks + tid; t < n_tok; t += kTopkThreads) {
                    const float s = srow[t];
                    const uint32_t key = score_key(s);
                    if (bin(s) == bstar && ((key ^ prefix) & mask) == 0)
                        atomicAdd(&sh.hist[(key >> shift) & 255u], 1u);
                }
            }
            __syncthreads();
            if (warp == 0) find_digit(sh.hist, need, sh.sc);
            __syncthreads();
            prefix |= sh.sc[0] << shift;
            mask |= 255u << shift;
            need -= sh.sc[1];
            __syncthreads();
        }
        const uint32_t T = prefix, ties_needed = need;

        // 4. emission in ascending token order.  Warp w owns a contiguous run
        // of whole 32-token groups, read with coalesced loads; ballots count
        // its keys above T and equal to T, one block scan over the warps'
        // counts places the run, and a second pass over the run writes the
        // selections in order (a tie is selected while its rank among the
        // ties, in token order, is below ties_needed).
        const int groups = (n + 31) / 32;
        const int gpw = (groups + kTopkWarps - 1) / kTopkWarps;
        const int t_lo = num_sinks + 32 * min(warp * gpw, groups), t_hi = min(num_sinks + 32 * min((warp + 1) * gpw, groups), n_tok);
        const uint32_t below = (1u << lane) - 1u;
        uint32_t c_gt = 0, c_eq = 0;
#pragma unroll 4
        for (int t0 = t_lo; t0 < t_hi; t0 += 32) {
            const int t = t0 + lane;
            const uint32_t key = t < t_hi ? score_key(srow[t]) : 0u;
            c_gt += __popc(__ballot_sync(0xffffffffu, t < t_hi && key > T));
            c_eq += __popc(__ballot_sync(0xffffffffu, t < t_hi && key == T));
        }
        // exclusive prefix over the warps of (c_gt, c_eq), packed into one
        // 64-bit scan done by warp 0
        if (lane == 0) {
            sh.hist[2 * warp] = c_gt;
            sh.hist[2 * warp + 1] = c_eq;
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t g = sh.hist[2 * lane], e = sh.hist[2 * lane + 1];
            uint32_t gi = g, ei = e;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t og = __shfl_up_sync(0xffffffffu, gi, off), oe = __shfl_up_sync(0xffffffffu, ei, off);
                if (lane >= off) {
                    gi += og;
                    ei += oe;
                }
            }
            sh.hist[2 * lane] = gi - g;
            sh.hist[2 * lane + 1] = ei - e;
        }
        __syncthreads();
        uint32_t tie_rank = sh.hist[2 * warp + 1];
        uint32_t pos = sh.hist[2 * warp] + min(tie_rank, ties_needed);
#pragma unroll 1
        for (int t0 = t_lo; t0 < t_hi; t0 += 32) {
            const int t = t0 + lane;
            const uint32_t key = t < t_hi ? score_key(srow[t]) : 0u;
            const bool gt = t < t_hi && key > T, eq = t < t_hi && key == T;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const bool tie_sel = eq && tie_rank + __popc(eqm & below) < ties_needed;
            const uint32_t selm = __ballot_sync(0xffffffffu, gt || tie_sel);
            if ((gt || tie_sel) && pos + __popc(selm & below) < static_cast<uint32_t>(k)) out[pos + __popc(selm & below)] = t;
            pos += __popc(selm);
            tie_rank += __popc(eqm);
        }
    }
    for (int i = k + tid; i < kmax; i += kTopkThreads) out[i] = -1;
}

}  // namespace

TopkLayout topk_layout(const sikv_params &) {
    TopkLayout L;
    L.total = kHeaderBytes;
    return L;
}

sikv_status launch_topk(const sikv_params &p, const float *scores, const int32_t *seq_lens,
                        const int32_t *k_per_seq, int32_t *idx, int32_t *status,
                        cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    const size_t smem = sizeof(TopkSmem);
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SIKV_ERR_CUDA;
    topk_kernel<<<segs, kTopkThreads, smem, stream>>>(scores, seq_lens, k_per_seq, p.num_kv_heads,
                                                      p.max_seq_len, p.num_sinks, p.max_topk, idx, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
