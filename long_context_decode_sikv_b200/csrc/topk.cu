// sikv_topk: exact top-k of the compressed-domain scores, without a full sort.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 2 (top-k selection on the LUT-GEMV scores).
// Order: score descending, then token index ascending (-0.0 == +0.0).
//
// Two kernels.  The cluster kernel (below) splits each segment's scores over
// a thread-block cluster; the single-CTA kernel (one CTA of 1024 threads per
// segment) serves segments longer than a cluster holds and shapes whose
// cluster would hold one CTA:
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
#include <atomic>

#include "cluster_common.cuh"
#include "decode_common.cuh"
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

// ---------------------------------------------------------------------------
// Cluster top-k.  Segment s is cut into C chunks of `chunk` scores, one CTA
// of 512 threads per chunk, the C CTAs forming one thread-block cluster.
// Each CTA keeps its chunk's order-preserving keys in shared memory.  The k-th
// largest key T is found digit by digit: every CTA histograms the top 12 bits
// of its keys and adds the counts at or above its own need-th largest into
// the leader's histogram (distributed shared memory); the leader finds the
// digit where the running count from the top reaches k and hands every CTA
// the digit, the count above it and how many keys share it.  When at most
// kKCandCap keys share it, every CTA copies its keys of that digit into the
// leader, which finds T among them alone (bits 19-10, then 9-0).  Otherwise
// two more cluster-wide levels follow (bits 19-8, then 7-0).  Then every CTA
// counts its keys above T and equal to T (one ballot pass that also keeps
// per-group masks), reads the other CTAs' counts, and writes its selected
// tokens in ascending token order at its place from the masks: the ties
// (keys equal to T) are taken lowest token first.
// ---------------------------------------------------------------------------

constexpr int kKT = 512;                  // threads per CTA (two CTAs per SM at 64 registers)
constexpr int kKW = kKT / 32;
constexpr int kKMaxChunk = 32768;         // keys per CTA at most
constexpr int kKMaxCluster = 16;
constexpr int kKDigits = 4096;            // 12-bit digits of the first two levels
constexpr uint32_t kKCandCap = kKDigits;  // threshold-digit keys the leader can take (its mhist)
static_assert(2 * (kKT / 32) <= kKDigits, "the warps' emission counts fit mhist");

struct TopkClusterSmem {
    uint32_t hist[kKDigits];              // this CTA's digit histogram
    uint32_t mhist[kKDigits];             // leader: the cluster's
    uint32_t wtot[kKW + 1];
    uint32_t sc[8];
    uint32_t bsd[3];                      // (digit, count above it, keys in it), from the leader
    uint32_t ccount;                      // leader: threshold-digit keys gathered so far
    uint32_t cnt[2];                      // this CTA's (keys > T, keys == T)
    uint32_t allcnt[2 * kKMaxCluster];
    uint32_t gmask[2 * (kKMaxChunk / 32)];// per 32-key group: keys above T, keys equal to T
    uint32_t key[1];                      // `chunk` keys (dynamic size)
};

constexpr size_t topk_cluster_smem(int chunk) {
    return sizeof(TopkClusterSmem) + sizeof(uint32_t) * (static_cast<size_t>(chunk) - 1);
}

__global__ void __launch_bounds__(kKT, 2)
topk_cluster_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_lens,
                    const int32_t *__restrict__ k_per_seq, int hkv, int nmax, int num_sinks, int kmax, int csize,
                    int chunk, int32_t *__restrict__ idx, int32_t *status) {
    extern __shared__ __align__(16) unsigned char topk_cluster_smem_raw[];
    TopkClusterSmem &sh = *reinterpret_cast<TopkClusterSmem *>(topk_cluster_smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = csize;
    const int c = static_cast<int>(cluster_ctarank());
    const int seg = blockIdx.x / C, b = seg / hkv;
    int32_t *out = idx + static_cast<size_t>(seg) * kmax;

    // lengths (an invalid segment selects nothing but still takes part)
    int n_tok = __ldg(seq_lens + b);
    if (n_tok < 0 || n_tok > nmax) {
        if (tid == 0 && c == 0) flag_error(status, SIKV_DEVERR_SEQ_LEN);
        n_tok = 0;
    }
    const int n = max(n_tok - num_sinks, 0);
    int k = __ldg(k_per_seq + b);
    if (k < 0 || k > kmax || k > n) {
        if (tid == 0 && c == 0) flag_error(status, SIKV_DEVERR_TOPK);
        k = 0;
    }
    // this CTA's scored tokens: positions [p_lo, p_hi) of its chunk
    const int t0 = c * chunk;
    const int p_lo = min(max(num_sinks - t0, 0), chunk), p_hi = max(min(n_tok - t0, chunk), p_lo);
    const float *srow = scores + static_cast<size_t>(seg) * nmax;
    // emission layout: warp w owns 32-key groups [g_lo, g_hi) of [p_lo, p_hi)
    const int groups = (p_hi - p_lo + 31) / 32;
    const int gpw = (groups + kKW - 1) / kKW;
    const int g_lo = min(warp * gpw, groups), g_hi = min((warp + 1) * gpw, groups);
    {
        // eight independent loads in flight per thread
        int p = p_lo + tid;
        for (; p + 7 * kKT < p_hi; p += 8 * kKT) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(srow + t0 + p + u * kKT);
#pragma unroll
            for (int u = 0; u < 8; ++u) sh.key[p + u * kKT] = score_key(v[u]);
        }
        for (; p < p_hi; p += kKT) sh.key[p] = score_key(__ldg(srow + t0 + p));
    }
    for (int i = tid; i < kKDigits; i += kKT) sh.mhist[i] = 0;
    if (tid == 0) sh.ccount = 0;
    cluster_arrive_cta();                                    // the leader's histogram is zero
    const uint32_t mh_leader = dsmem_map(&sh.mhist[0], 0);

    // the k-th key, digit by digit (bits 31-20, then 19-8 and 7-0 unless the
    // leader finishes from the first digit's keys)
    uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(k);
    bool fast = false;
#pragma unroll 1
    for (int level = 0; level < 3; ++level) {
        const int shift = level == 0 ? 20 : (level == 1 ? 8 : 0);
        const uint32_t nd = level == 2 ? 256u : static_cast<uint32_t>(kKDigits);
        for (int i = tid; i < static_cast<int>(nd); i += kKT) sh.hist[i] = 0;
        __syncthreads();
        if (k > 0)
            for (int p = p_lo + tid; p < p_hi; p += kKT) {
                const uint32_t key = sh.key[p];
                if (((key ^ prefix) & mask) == 0) atomicAdd(&sh.hist[(key >> shift) & (nd - 1u)], 1u);
            }
        __syncthreads();
        if (level == 0) cluster_wait();                      // the leader's histogram is zero
        if (k > 0) {
            // only the digits at or above this CTA's own need-th largest: the
            // cluster's is never below it (0 when the CTA holds fewer keys)
            if (tid == 0) {
                sh.sc[2] = 0;
                sh.sc[3] = 0;
            }
            __syncthreads();
            if (level < 2)
                cta_find_bin<kKDigits / kKT, kKT>([&](int i) { return sh.hist[i]; }, need, sh.wtot, sh.sc + 2);
            else
                cta_find_bin<1, kKT>([&](int i) { return i < 256 ? sh.hist[i] : 0u; }, need, sh.wtot, sh.sc + 2);
            for (int i = static_cast<int>(sh.sc[2]) + tid; i < static_cast<int>(nd); i += kKT) {
                const uint32_t v = sh.hist[i];
                if (v) dsmem_red_add(mh_leader + 4u * static_cast<uint32_t>(i), v);
            }
        }
        cluster_arrive_cta();                                // every count is in the leader's histogram
        cluster_wait();
        if (c == 0 && k > 0) {
            if (tid == 0) {
                sh.sc[0] = 0;
                sh.sc[1] = 0;
            }
            __syncthreads();
            if (level < 2)
                cta_find_bin<kKDigits / kKT, kKT>([&](int i) { return sh.mhist[i]; }, need, sh.wtot, sh.sc);
            else
                cta_find_bin<1, kKT>([&](int i) { return i < 256 ? sh.mhist[i] : 0u; }, need, sh.wtot, sh.sc);
            if (tid < C) {
                dsmem_st_u32(dsmem_map(&sh.bsd[0], static_cast<uint32_t>(tid)), sh.sc[0]);
                dsmem_st_u32(dsmem_map(&sh.bsd[1], static_cast<uint32_t>(tid)), sh.sc[1]);
                dsmem_st_u32(dsmem_map(&sh.bsd[2], static_cast<uint32_t>(tid)), sh.mhist[sh.sc[0]]);
            }
            __syncthreads();
            for (int i = tid; i < kKDigits; i += kKT) sh.mhist[i] = 0;   // for the next level
        }
        cluster_arrive_cta();                                // the digit is in every CTA
        cluster_wait();
        if (k > 0) {
            prefix |= sh.bsd[0] << shift;
            mask |= (nd - 1u) << shift;
            need -= sh.bsd[1];
        }
        // few keys share the first digit of the k-th: the leader finishes alone
        if (level == 0 && k > 0 && sh.bsd[2] <= kKCandCap) {
            fast = true;
            break;
        }
    }
    if (fast) {
        // every key of the threshold digit into the leader's mhist (it holds
        // bsd[2] <= kKCandCap of them): gathered in this CTA's hist first, then
        // one range of the leader's list reserved for the CTA
        // This CTA's candidates are its level-0 count of the threshold digit:
        // their range of the leader's list is reserved before the scan, which
        // hides the round trip.
        const uint32_t below = (1u << lane) - 1u;
        uint32_t at0 = 0;
        if (tid == 0) {
            const uint32_t mine = min(sh.hist[prefix >> 20], kKCandCap);
            at0 = mine ? dsmem_atom_add(dsmem_map(&sh.ccount, 0), mine) : 0u;
            sh.cnt[0] = 0;
        }
        __syncthreads();
        for (int base = p_lo; base < p_hi; base += kKT) {
            const int p = base + tid;
            const uint32_t key = p < p_hi ? sh.key[p] : 0u;
            const bool cand = p < p_hi && ((key ^ prefix) & mask) == 0;
            const uint32_t m = __ballot_sync(0xffffffffu, cand);
            if (m) {
                uint32_t slot = 0;
                if (lane == 0) slot = atomicAdd(&sh.cnt[0], static_cast<uint32_t>(__popc(m)));
                slot = __shfl_sync(0xffffffffu, slot, 0) + static_cast<uint32_t>(__popc(m & below));
                if (cand && slot < kKCandCap) sh.hist[slot] = key;
            }
        }
        __syncthreads();
        const uint32_t nmine = min(sh.cnt[0], kKCandCap);
        if (tid == 0) sh.sc[4] = at0;
        __syncthreads();
        {
            const uint32_t cbuf = dsmem_map(&sh.mhist[0], 0), at = sh.sc[4];
            for (uint32_t i = tid; i < nmine; i += kKT)
                if (at + i < kKCandCap) dsmem_st_u32(cbuf + 4u * (at + i), sh.hist[i]);
        }
        cluster_arrive_cta();                                // the leader holds every candidate
        cluster_wait();
        if (c == 0) {
            // the need-th largest candidate: bits 19-10, then bits 9-0
            constexpr uint32_t kSub = 1024;
            const int nc = static_cast<int>(min(sh.ccount, kKCandCap));
            for (int i = tid; i < static_cast<int>(kSub); i += kKT) sh.hist[i] = 0;
            if (tid == 0) {
                sh.sc[0] = 0;
                sh.sc[1] = 0;
            }
            __syncthreads();
            for (int i = tid; i < nc; i += kKT) atomicAdd(&sh.hist[(sh.mhist[i] >> 10) & (kSub - 1u)], 1u);
            __syncthreads();
            cta_find_bin<kSub / kKT, kKT>([&](int i) { return sh.hist[i]; }, need, sh.wtot, sh.sc);
            const uint32_t d1 = sh.sc[0], above1 = sh.sc[1];
            for (int i = tid; i < static_cast<int>(kSub); i += kKT) sh.hist[i] = 0;
            if (tid == 0) {
                sh.sc[0] = 0;
                sh.sc[1] = 0;
            }
            __syncthreads();
            for (int i = tid; i < nc; i += kKT) {
                const uint32_t key = sh.mhist[i];
                if (((key >> 10) & (kSub - 1u)) == d1) atomicAdd(&sh.hist[key & (kSub - 1u)], 1u);
            }
            __syncthreads();
            cta_find_bin<kSub / kKT, kKT>([&](int i) { return sh.hist[i]; }, need - above1, sh.wtot, sh.sc);
            if (tid < C) {
                dsmem_st_u32(dsmem_map(&sh.bsd[0], static_cast<uint32_t>(tid)), prefix | (d1 << 10) | sh.sc[0]);
                dsmem_st_u32(dsmem_map(&sh.bsd[1], static_cast<uint32_t>(tid)), need - above1 - sh.sc[1]);
            }
        }
        cluster_arrive_cta();                                // the k-th key is in every CTA
        cluster_wait();
        prefix = sh.bsd[0];
        need = sh.bsd[1];
    }
    const uint32_t T = prefix, ties_needed = need;           // the k-th key; how many keys == T are selected

    // Keys above T and equal to T, in ascending token order: warp w owns a
    // contiguous run of 32-position groups; one ballot pass records each
    // group's two masks (above at gmask[2 g], equal at gmask[2 g + 1]) and the
    // warp's counts (in mhist[2 w], mhist[2 w + 1]); the CTA's totals go to
    // the cluster; then the selections are written from the masks.
    if (k > 0) {
        uint32_t c_gt = 0, c_eq = 0;
        for (int g = g_lo; g < g_hi; ++g) {
            const int q = p_lo + 32 * g + lane;
            const uint32_t key = q < p_hi ? sh.key[q] : 0u;
            const uint32_t gm = __ballot_sync(0xffffffffu, q < p_hi && key > T);
            const uint32_t em = __ballot_sync(0xffffffffu, q < p_hi && key == T);
            if (lane == 0) {
                sh.gmask[2 * g] = gm;
                sh.gmask[2 * g + 1] = em;
            }
            c_gt += __popc(gm);
            c_eq += __popc(em);
        }
        if (lane == 0) {
            sh.mhist[2 * warp] = c_gt;
            sh.mhist[2 * warp + 1] = c_eq;
        }
    }
    __syncthreads();
    if (k > 0 && warp == 0) {
        // exclusive scans of the warps' counts; lane 0 also writes the totals
        const uint32_t g = lane < kKW ? sh.mhist[2 * lane] : 0u, e = lane < kKW ? sh.mhist[2 * lane + 1] : 0u;
        uint32_t gi = g, ei = e;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t og = __shfl_up_sync(0xffffffffu, gi, off), oe = __shfl_up_sync(0xffffffffu, ei, off);
            if (lane >= off) {
                gi += og;
                ei += oe;
            }
        }
        if (lane < kKW) {
            sh.mhist[2 * lane] = gi - g;
            sh.mhist[2 * lane + 1] = ei - e;
        }
        if (lane == 31) {
            sh.cnt[0] = gi;
            sh.cnt[1] = ei;
        }
    }
    cluster_arrive_cta();                                    // every CTA's counts are published
    cluster_wait();
    if (k > 0) {
        if (tid < 2 * C) sh.allcnt[tid] = dsmem_ld_u32(dsmem_map(&sh.cnt[tid & 1], static_cast<uint32_t>(tid >> 1)));
        __syncthreads();
        uint32_t gt_before = 0, eq_before = 0;
        for (int r = 0; r < c; ++r) {
            gt_before += sh.allcnt[2 * r];
            eq_before += sh.allcnt[2 * r + 1];
        }
        // this CTA's first output position, and how many of its ties are taken
        const uint32_t base = gt_before + min(eq_before, ties_needed);
        const uint32_t my_ties = ties_needed > eq_before ? ties_needed - eq_before : 0u;
        const uint32_t below = (1u << lane) - 1u;
        uint32_t tie_rank = sh.mhist[2 * warp + 1];
        uint32_t pos = base + sh.mhist[2 * warp] + min(tie_rank, my_ties);
        for (int g = g_lo; g < g_hi; ++g) {
            const uint32_t gm = sh.gmask[2 * g], em = sh.gmask[2 * g + 1];
            if ((gm | em) == 0u) continue;
            // ties are taken while this CTA's share lasts, lowest positions first
            const bool tie_sel = ((em >> lane) & 1u) && tie_rank + static_cast<uint32_t>(__popc(em & below)) < my_ties;
            const uint32_t selm = gm | __ballot_sync(0xffffffffu, tie_sel);
            if ((selm >> lane) & 1u) {
                const uint32_t at = pos + static_cast<uint32_t>(__popc(selm & below));
                if (at < static_cast<uint32_t>(k)) out[at] = t0 + p_lo + 32 * g + lane;
            }
            pos += static_cast<uint32_t>(__popc(selm));
            tie_rank += static_cast<uint32_t>(__popc(em));
        }
    }
    if (c == 0)
        for (int i = k + tid; i < kmax; i += kKT) out[i] = -1;
    cluster_arrive_relaxed();                                // no CTA leaves while its counts are read
    cluster_wait();
}

}  // namespace

TopkLayout topk_layout(const sikv_params &) {
    TopkLayout L;
    L.total = kHeaderBytes;
    return L;
}

namespace {

// Cluster size and chunk of the cluster kernel for these parameters (0: the
// segments are longer than a cluster holds).  The largest cluster whose whole
// batch fits on the device at once (with a margin for how clusters pack into
// GPCs) and whose chunks are not tiny; else the smallest cluster, whose
// waves carry the most keys per CTA.
int topk_cluster_plan(const sikv_params &p, int *chunk_out) {
    const int nmax = p.max_seq_len, segs = p.batch * p.num_kv_heads;
    const int cmin = std::max(1, (nmax + kKMaxChunk - 1) / kKMaxChunk);
    if (cmin > kKMaxCluster) return 0;
    const int sms = device_sm_count();
    auto chunk_of = [&](int cs) { return ((nmax + cs - 1) / cs + 31) / 32 * 32; };
    int csize = cmin;
    for (int cs = kKMaxCluster; cs > std::max(cmin, 1); --cs) {
        const int ch = chunk_of(cs);
        if (ch < 2048 || (nmax + ch - 1) / ch != cs) continue;
        // CTAs per SM: two by registers (64 per thread), fewer when the keys need more shared memory
        const int bps = std::min<int>(2, static_cast<int>(233472 / (topk_cluster_smem(ch) + 1024)));
        if (10 * segs * cs <= 9 * sms * bps) {
            csize = cs;
            break;
        }
    }
    *chunk_out = chunk_of(csize);
    // one CTA per segment: the single-CTA kernel (1024 threads) does that better
    if (csize == 1) return 0;
    return *chunk_out <= kKMaxChunk ? csize : 0;
}

}  // namespace

sikv_status launch_topk(const sikv_params &p, const float *scores, const int32_t *seq_lens,
                        const int32_t *k_per_seq, int32_t *idx, int32_t *status,
                        cudaStream_t stream) {
    // per device: 0 unknown, 1 the cluster kernel launches, 2 it does not
    // (then the single-CTA kernel serves every call)
    static std::atomic<int> usable[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
    const int segs = p.batch * p.num_kv_heads;
    int chunk = 0;
    const int csize = (dev >= 0 && usable[dev].load(std::memory_order_relaxed) != 2) ? topk_cluster_plan(p, &chunk) : 0;
    if (csize > 0) {
        const size_t smem = topk_cluster_smem(chunk);
        if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(topk_cluster_smem(kKMaxChunk))) == cudaSuccess &&
            cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(segs * csize));
            cfg.blockDim = dim3(kKT);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = stream;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = static_cast<unsigned>(csize);
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, seq_lens, k_per_seq, p.num_kv_heads,
                                   p.max_seq_len, p.num_sinks, p.max_topk, csize, chunk, idx, status) == cudaSuccess) {
                usable[dev].store(1, std::memory_order_relaxed);
                return SIKV_OK;
            }
        }
        cudaGetLastError();                  // a configuration the device refuses: the single-CTA kernel
        usable[dev].store(2, std::memory_order_relaxed);
    }
    const size_t smem = sizeof(TopkSmem);
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SIKV_ERR_CUDA;
    topk_kernel<<<segs, kTopkThreads, smem, stream>>>(scores, seq_lens, k_per_seq, p.num_kv_heads,
                                                      p.max_seq_len, p.num_sinks, p.max_topk, idx, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
