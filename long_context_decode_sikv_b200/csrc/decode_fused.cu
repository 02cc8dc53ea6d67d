// sikv_decode, single-launch form: scoring, exact top-k and fused sparse
// attention of a whole decode step in one cooperative kernel.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 items 2-4: LUT-GEMV scores in the compressed domain,
// top-k on them, dequantization fused with sparse attention over the 64 sink
// tokens plus the selected tokens.
//
// Work split.  Each (sequence, KV head) segment is cut into `cps` chunks of
// `chunk` tokens, one CTA per chunk, all CTAs co-resident (cooperative
// launch).  A CTA never writes its scores to memory (unless asked to): it
// keeps each token's histogram bin in shared memory.  The CTAs of a segment
// agree on the selection through three counters in the workspace:
//   1. every CTA builds a 1024-bin histogram of its scores (bins linear in the
//      score between the bounds the LUT implies, so a higher bin means a
//      strictly higher score), finds its own local k-th bin b_c and adds its
//      counts for bins >= b_c into the segment histogram (the segment's k-th
//      bin b* is >= every b_c, so the lower bins are never needed);  arrive #1;
//   2. after all arrivals every CTA scans the segment histogram from the top
//      and finds b*; tokens in higher bins are selected outright, tokens in
//      b* are re-scored and appended with their exact keys to a candidate
//      list;  arrive #2;
//   3. every CTA ranks the candidates (order: key descending, token
//      ascending) and marks the winners of its own chunk — the same answer in
//      every CTA — then attends over its selected tokens and its share of the
//      sinks with an online softmax and writes (m, l, o) partials;  arrive #3 —
//      the last CTA to arrive merges the partials into the output and zeroes
//      the segment's coordination state for the next launch.
// Waits are bounded: a wait that runs out sets SIKV_DEVERR_TIMEOUT and the
// CTA carries on, so a kernel always ends.
//
// Code size matters here: every phase but the scoring loop runs once per CTA
// with a cold instruction cache, so loops over a thread's tokens stay rolled
// (their state lives in shared memory, not in registers).
#include "score_device.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kFT = 256;                 // threads per CTA
constexpr int kFW = kFT / 32;            // warps per CTA
constexpr int kFBins = 1024;             // histogram bins per segment
constexpr int kFTile = 256;              // list entries attended per pass
constexpr int kFListCap = 2048;          // attended tokens staged per window
constexpr int kFMaxNpt = 64;             // token slots per thread at most
constexpr int kFMaxChunk = kFMaxNpt * kFT;
constexpr int kFCandSmem = 1024;         // candidates staged in shared memory
constexpr int kFRankMax = 512;           // up to this many candidates: rank directly
constexpr int kFUnroll = 8;              // code rows in flight per thread
constexpr int kFPrefetchRows = 16;       // code rows per thread kept ahead in L2
constexpr int kFVRows = 8;               // value rows in flight per warp
constexpr int kSpinLimit = 1 << 23;      // ~1 s of __nanosleep(128) polls
constexpr int kFRow = 256;               // tokens per row scan of a warp (32 lanes x 8)

struct FusedArgs {
    const void *q, *K, *V;
    const uint8_t *codes;
    const float *codebook, *mu;
    const int32_t *seq_lens, *k_per_seq;
    void *out;
    int32_t *idx_out;
    float *scores_out;
    int hq, hkv, nmax, num_sinks, kmax, cps, chunk, npt, cand_cap;
    float scale;
    uint32_t *ghist;      // [segs][kFBins]
    uint2 *cand;          // [segs][cand_cap] (key, token)
    FusedCtl *ctl;        // [segs]
    int32_t *selcnt;      // [segs][cps]
    float *part_o;        // [segs][cps][GM][D]
    float2 *part_ml;      // [segs][cps][GM]
    int32_t *status;
};

// Shared memory.  The union is reused in time: scoring tables (until the
// candidates are written), then the candidate ranking buffers, then the
// attention buffers.
template <int GM>
struct FusedSmem {
    union {
        ScoreTables tab;
        struct {
            uint32_t ckey[kFCandSmem];
            int32_t cidx[kFCandSmem];
            uint32_t winbits[kFMaxChunk / 32];
        } sel;
        struct {
            int32_t list[kFListCap];
            alignas(16) float logit[GM][kFTile];
            alignas(16) float red[kFW][GM][kHeadDim];
            alignas(16) float luth[kSubspaces * kClusters][GM];   // per-head LUT, [s*16+j][g]
        } at;
    } u;
    alignas(16) float qs[GM][kHeadDim];
    alignas(16) float mus[kHeadDim];
    alignas(16) float qmu_h[GM];
    alignas(16) float run_m[GM];
    alignas(16) float run_l[GM];
    alignas(16) float tile_stat[kFW][GM];
    uint32_t hist[kFBins];
    // one entry per token of the chunk, in token order (entry p: token t0 + p,
    // scored by thread p mod 256): its bin + 1 (0: no token), bit 15 set once
    // the token is selected.  Holds the codebook before scoring.
    alignas(16) uint16_t bins[kFMaxChunk];
    uint32_t rowcnt[kFMaxChunk / 256];        // selected tokens per row of 256, then their prefix
    uint32_t wtot[kFW + 1];
    uint32_t sc[16];
    float bin_lo, bin_inv;
    int bin_flat, last;
};

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Thread 0 waits until *ctr >= target (bounded); the CTA then synchronizes.
__device__ __forceinline__ void cta_wait(const int *ctr, int target, int32_t *status) {
    if (threadIdx.x == 0) {
        int it = 0;
        while (ld_acquire(ctr) < target) {
            if (++it > kSpinLimit) {
                flag_error(status, SIKV_DEVERR_TIMEOUT);
                break;
            }
            __nanosleep(128);
        }
    }
    __syncthreads();
    __threadfence();
}

// Every thread's prior global writes become visible, then thread 0 arrives.
// Returns the counter's previous value to thread 0 (others get 0).
__device__ __forceinline__ int cta_arrive(int *ctr) {
    __threadfence();
    __syncthreads();
    int old = 0;
    if (threadIdx.x == 0) old = atomicAdd(ctr, 1);
    return old;
}

// Exclusive scan over the CTA (256 threads) of one value per thread.
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t *wtot, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t run = 0;
        for (int w = 0; w < kFW; ++w) {
            const uint32_t t = wtot[w];
            wtot[w] = run;
            run += t;
        }
        wtot[kFW] = run;
    }
    __syncthreads();
    const uint32_t r = wtot[warp] + incl - v;
    *total = wtot[kFW];
    __syncthreads();
    return r;
}

// In a histogram of PER * 256 bins scanned from the top bin down, finds the
// bin where the running count first reaches `need` (1 <= need <= total).
// Each thread loads its PER consecutive bins once.  Writes (bin, count above)
// to out[0..1]; out is left untouched when the total is below need.  Ends
// synchronized.
template <int PER, typename Load>
__device__ __forceinline__ void cta_find_bin(Load load, uint32_t need, uint32_t *wtot, uint32_t *out) {
    const int top = PER * kFT - 1 - static_cast<int>(threadIdx.x) * PER;
    uint32_t h[PER];
    uint32_t loc = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        h[i] = load(top - i);
        loc += h[i];
    }
    uint32_t total;
    uint32_t above = cta_excl_scan(loc, wtot, &total);
    if (above < need && need <= above + loc) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if (above < need && above + h[i] >= need) {
                out[0] = static_cast<uint32_t>(top - i);
                out[1] = above;
            }
            above += h[i];
        }
    }
    __syncthreads();
}

// Radix select over `n` elements (element e has key key(e) and passes
// keep(e)): returns the key of rank `need` counted from the largest and, in
// *need_left, how many elements equal to it are still needed.  Uses hist[0..255].
template <typename KeyF, typename KeepF>
__device__ __noinline__ uint32_t cta_radix_select(KeyF key, KeepF keep, int n, uint32_t need, uint32_t *hist,
                                                  uint32_t *wtot, uint32_t *sc, uint32_t *need_left) {
    uint32_t prefix = 0, mask = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kFT) hist[i] = 0;
        __syncthreads();
        for (int e = threadIdx.x; e < n; e += kFT) {
            if (!keep(e)) continue;
            const uint32_t k = key(e);
            if (((k ^ prefix) & mask) == 0) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        cta_find_bin<1>([&](int i) { return hist[i]; }, need, wtot, sc);
        prefix |= sc[0] << shift;
        mask |= 255u << shift;
        need -= sc[1];
        __syncthreads();
    }
    *need_left = need;
    return prefix;
}

// Appends token t of the threshold bin to the segment's candidate list with
// its exact key: re-scored by the lane that scored it (same table, same
// rotation, same order of additions, so bit-identical).
__device__ __noinline__ void emit_candidate(const float *t2, const uint4 *crow, int t, int lane, float qmu,
                                            int *ncand, uint2 *cand, int cap) {
    const float sv = lut2_score(t2, __ldg(crow + t), lane, qmu);
    const int slot = atomicAdd(ncand, 1);
    if (slot < cap) cand[slot] = make_uint2(score_key(sv), static_cast<uint32_t>(t));
}

// bins[] holds one 16-bit entry per token of the chunk in token order (entry
// p is token t0 + p).  A lane scans 8 consecutive entries with one 16-byte
// load; these give, per 16-bit half of each word, an all-ones mask where the
// entry's bin is above / equal to a threshold (entries hold bin + 1).
__device__ __forceinline__ uint32_t half_gt(uint32_t w, uint32_t thr2) { return __vcmpgtu2(w & 0x7FFF7FFFu, thr2); }
__device__ __forceinline__ uint32_t half_eq(uint32_t w, uint32_t thr2) { return __vcmpeq2(w & 0x7FFF7FFFu, thr2); }
// 8-bit mask (bit j = entry j of the lane's 8) from four per-half masks
__device__ __forceinline__ uint32_t mask8(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
    return (m0 & 1u) | ((m0 >> 15) & 2u) | ((m1 & 1u) << 2) | ((m1 >> 13) & 8u) | ((m2 & 1u) << 4) |
           ((m2 >> 11) & 32u) | ((m3 & 1u) << 6) | ((m3 >> 9) & 128u);
}

// Winners among many candidates (more than the rank path takes): radix
// select of the need-th key and of the lowest tied token indices, then one
// marking pass.  Returns this thread's count of winners before the chunk.
// Kept out of line: it only runs for heavily tied or flat score tables.
__device__ __noinline__ uint32_t refine_by_radix(const uint2 *cand, int ncand, uint32_t need, int t0, int chunk,
                                                 uint32_t *winbits, uint32_t *hist, uint32_t *wtot, uint32_t *sc) {
    uint32_t ties_needed, left, before = 0;
    const uint32_t T = cta_radix_select([&](int e) { return __ldcg(cand + e).x; }, [&](int) { return true; }, ncand,
                                        need, hist, wtot, sc, &ties_needed);
    // the ties_needed lowest token indices among keys equal to T
    const uint32_t tie_idx = ~cta_radix_select([&](int e) { return ~__ldcg(cand + e).y; },
                                               [&](int e) { return __ldcg(cand + e).x == T; }, ncand, ties_needed,
                                               hist, wtot, sc, &left);
    for (int e = threadIdx.x; e < ncand; e += kFT) {
        const uint2 v = __ldcg(cand + e);
        if (v.x > T || (v.x == T && v.y <= tie_idx)) {
            const int rel = static_cast<int>(v.y) - t0;
            if (rel >= 0 && rel < chunk) atomicOr(&winbits[rel >> 5], 1u << (rel & 31));
            else if (rel < 0) ++before;
        }
    }
    return before;
}

template <int DT, int GM>
__global__ void __launch_bounds__(kFT, 2) decode_fused_kernel(FusedArgs a) {
    constexpr int EB = ElemBytes<DT>::value;
    extern __shared__ __align__(16) unsigned char fused_smem[];
    FusedSmem<GM> &sh = *reinterpret_cast<FusedSmem<GM> *>(fused_smem);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seg = blockIdx.x / a.cps, c = blockIdx.x % a.cps;
    const int b = seg / a.hkv, h = seg % a.hkv, group = a.hq / a.hkv;
    const int npt = a.npt;
    FusedCtl *ctl = a.ctl + seg;

    // ---- lengths (an invalid segment decodes as empty but still takes part)
    int n_tok = __ldg(a.seq_lens + b);
    if (n_tok < 0 || n_tok > a.nmax) {
        if (tid == 0 && c == 0) flag_error(a.status, SIKV_DEVERR_SEQ_LEN);
        n_tok = 0;
    }
    const int n_scored = max(n_tok - a.num_sinks, 0);
    int k = __ldg(a.k_per_seq + b);
    if (k < 0 || k > a.kmax || k > n_scored) {
        if (tid == 0 && c == 0) flag_error(a.status, SIKV_DEVERR_TOPK);
        k = 0;
    }
    const int t0 = c * a.chunk;
    const int t1 = min(t0 + a.chunk, n_tok);
    const int tstart = max(t0, a.num_sinks);
    const size_t kv_seg = static_cast<size_t>(seg) * a.nmax;
    const uint4 *crow = reinterpret_cast<const uint4 *>(a.codes) + kv_seg;
    const int my = 32 * warp + lane;                         // slot i of this thread: token t0 + 256 i + my

    // ---- tables.  The prologue leaves HBM idle, so the first code rows and
    // this CTA's share of the sink rows go to L2 meanwhile.
#pragma unroll 1
    for (int i = 0; i < kFPrefetchRows && i < npt; ++i) {
        const int t = t0 + kFT * i + my;
        if (t >= tstart && t < t1) prefetch_l2(crow + t);
    }
    {
        const int n_sinks0 = min(a.num_sinks, n_tok);
        for (int sk = c + a.cps * tid; sk < n_sinks0; sk += a.cps * kFT) {
            prefetch_l2(static_cast<const char *>(a.K) + (kv_seg + sk) * kHeadDim * EB);
            prefetch_l2(static_cast<const char *>(a.V) + (kv_seg + sk) * kHeadDim * EB);
        }
    }
    float4 *cbs = reinterpret_cast<float4 *>(sh.bins);     // 8 KB, free until scoring
    for (int e = tid; e < GM * kHeadDim; e += kFT) sh.qs[e / kHeadDim][e % kHeadDim] = 0.f;
    __syncthreads();
    stage_table_inputs<DT>(&sh.qs[0][0], cbs, sh.mus, a.q, a.codebook, a.mu, b, h, a.hq, group, seg);
    for (int i = tid; i < kFBins; i += kFT) sh.hist[i] = 0;
    __syncthreads();
    build_score_tables(sh.u.tab, &sh.qs[0][0], cbs, sh.mus, group);
    for (int g = warp; g < GM; g += kFW) {
        double s = static_cast<double>(sh.qs[g][4 * lane]) * sh.mus[4 * lane];
        s = fma(static_cast<double>(sh.qs[g][4 * lane + 1]), static_cast<double>(sh.mus[4 * lane + 1]), s);
        s = fma(static_cast<double>(sh.qs[g][4 * lane + 2]), static_cast<double>(sh.mus[4 * lane + 2]), s);
        s = fma(static_cast<double>(sh.qs[g][4 * lane + 3]), static_cast<double>(sh.mus[4 * lane + 3]), s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) sh.qmu_h[g] = static_cast<float>(s);
    }
    if (warp == kFW - 1) {
        // score bounds: q_bar.mu + sum over subspaces of the min / max LUT entry
        float lo = INFINITY, hi = -INFINITY;
        for (int j = 0; j < kClusters; ++j) {
            const float v = sh.u.tab.lutT[j * kSubspaces + lane];
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo += __shfl_xor_sync(0xffffffffu, lo, off);
            hi += __shfl_xor_sync(0xffffffffu, hi, off);
        }
        if (lane == 0) {
            lo += sh.u.tab.qmu;
            hi += sh.u.tab.qmu;
            const float width = hi - lo;
            const float inv = static_cast<float>(kFBins) / width;
            sh.bin_lo = lo;
            sh.bin_inv = inv;
            sh.bin_flat = !(isfinite(width) && width > 0.f && isfinite(inv));
        }
    }
    __syncthreads();
    const float bin_lo = sh.bin_lo, bin_inv = sh.bin_inv;
    const bool bin_flat = sh.bin_flat != 0;
    const float qmu = sh.u.tab.qmu;

    // ---- scores of this chunk -> histogram and per-slot bins
    {
        float *so = a.scores_out ? a.scores_out + kv_seg : nullptr;
#pragma unroll 1
        for (int i0 = 0; i0 < npt; i0 += kFUnroll) {
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u) {
                const int t = t0 + kFT * (i0 + kFPrefetchRows + u) + my;
                if (i0 + kFPrefetchRows + u < npt && t >= tstart && t < t1) prefetch_l2(crow + t);
            }
            uint4 rows[kFUnroll];
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u) {
                const int t = t0 + kFT * (i0 + u) + my;
                rows[u] = (i0 + u < npt && t >= tstart && t < t1) ? __ldcs(crow + t) : make_uint4(0, 0, 0, 0);
            }
            float sc2[kFUnroll];
#pragma unroll
            for (int u = 0; u < kFUnroll; u += 2) {
                const float2 v = lut2_score2(sh.u.tab.t2, rows[u], rows[u + 1], lane, qmu);
                sc2[u] = v.x;
                sc2[u + 1] = v.y;
            }
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u) {
                const int i = i0 + u;
                if (i >= npt) break;
                const int t = t0 + kFT * i + my;
                uint16_t e = 0;
                if (t >= tstart && t < t1) {
                    const float sv = sc2[u];
                    int bi = 0;
                    if (!bin_flat) bi = min(max(__float2int_rz((sv - bin_lo) * bin_inv), 0), kFBins - 1);
                    atomicAdd(&sh.hist[bi], 1u);
                    e = static_cast<uint16_t>(bi + 1);
                    if (so) so[t] = sv;
                } else if (so && t < t1) {
                    so[t] = -INFINITY;
                }
                sh.bins[i * kFT + tid] = e;
            }
        }
    }
    __syncthreads();

    // ---- 1. local k-th bin, publish the bins at or above it
    if (k > 0) {
        if (tid == 0) {
            sh.sc[0] = 0;
            sh.sc[1] = 0;
        }
        __syncthreads();
        cta_find_bin<kFBins / kFT>([&](int i) { return sh.hist[i]; }, static_cast<uint32_t>(k), sh.wtot, sh.sc);
        const int bc = static_cast<int>(sh.sc[0]);    // 0 when the chunk holds fewer than k tokens
        uint32_t *gh = a.ghist + static_cast<size_t>(seg) * kFBins;
        for (int i = bc + tid; i < kFBins; i += kFT) {
            const uint32_t v = sh.hist[i];
            if (v) atomicAdd(gh + i, v);
        }
    }
    cta_arrive(&ctl->arrive1);
    cta_wait(&ctl->arrive1, a.cps, a.status);

    // ---- 2. segment k-th bin b*; count higher bins, list the tokens of b*
    int bstar = kFBins;              // nothing selected when k == 0
    uint32_t above_bstar = 0;
    if (k > 0) {
        const uint32_t *gh = a.ghist + static_cast<size_t>(seg) * kFBins;
        cta_find_bin<kFBins / kFT>([&](int i) { return __ldcg(gh + i); }, static_cast<uint32_t>(k), sh.wtot, sh.sc);
        bstar = static_cast<int>(sh.sc[0]);
        above_bstar = sh.sc[1];
        uint32_t mine = 0;
        uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
        const uint32_t b2 = static_cast<uint32_t>(bstar + 1) * 0x10001u;
#pragma unroll 1
        for (int row = warp; row * kFRow < a.chunk; row += kFW) {
            const int p0 = row * kFRow + 8 * lane;
            const uint4 w = *reinterpret_cast<const uint4 *>(sh.bins + p0);
            const uint32_t gt = mask8(half_gt(w.x, b2), half_gt(w.y, b2), half_gt(w.z, b2), half_gt(w.w, b2));
            const uint32_t eq = mask8(half_eq(w.x, b2), half_eq(w.y, b2), half_eq(w.z, b2), half_eq(w.w, b2));
            mine += __popc(gt);
            // selected for sure: the code and value rows are needed by the
            // attention pass, so they go to L2 now
            for (uint32_t mm = gt; mm; mm &= mm - 1) {
                const int t = t0 + p0 + __ffs(mm) - 1;
                prefetch_l2(crow + t);
                prefetch_l2(static_cast<const char *>(a.V) + (kv_seg + t) * kHeadDim * EB);
                if (EB * kHeadDim > 128) prefetch_l2(static_cast<const char *>(a.V) + (kv_seg + t) * kHeadDim * EB + 128);
            }
            // tokens of the threshold bin: exact key needed.  The lane that
            // scored token t0 + p is p mod 32 (the table's bank rotation), so
            // the warp hands each one to that lane.
            uint32_t todo = __ballot_sync(0xffffffffu, eq != 0);
            while (todo) {
                const int src = __ffs(todo) - 1;
                todo &= todo - 1;
                const uint32_t em = __shfl_sync(0xffffffffu, eq, src);
                for (uint32_t mm = em; mm; mm &= mm - 1) {
                    const int p = row * kFRow + 8 * src + __ffs(mm) - 1;
                    if (lane == (p & 31))
                        emit_candidate(sh.u.tab.t2, crow, t0 + p, lane, qmu, &ctl->ncand, cand, a.cand_cap);
                }
            }
        }
        uint32_t tot;
        cta_excl_scan(mine, sh.wtot, &tot);
        if (tid == 0) a.selcnt[static_cast<size_t>(seg) * a.cps + c] = static_cast<int32_t>(tot);
    }
    cta_arrive(&ctl->arrive2);

    // Tokens above b* are selected whatever the candidates decide, so they
    // (and this CTA's share of the sinks) are attended first, while the
    // other CTAs finish the candidate list; the winners of the threshold bin
    // follow in a second pass over the same code, continuing the same online
    // softmax.  Entry bit 15 marks a token of the first pass, bit 14 one of
    // the second.
    const int nrows = (a.chunk + kFRow - 1) / kFRow;           // <= 64
    const uint32_t b2 = static_cast<uint32_t>(bstar + 1) * 0x10001u;
    auto row_mask = [&](int row, uint32_t bit2) -> uint32_t {
        const uint4 w = *reinterpret_cast<const uint4 *>(sh.bins + row * kFRow + 8 * lane);
        return mask8(__vcmpne2(w.x & bit2, 0u), __vcmpne2(w.y & bit2, 0u), __vcmpne2(w.z & bit2, 0u),
                     __vcmpne2(w.w & bit2, 0u));
    };
    // sets bit2 on the entries picked by pick(row, words) and counts them per row;
    // returns the total, with sh.rowcnt turned into each row's ordinal base
    auto mark_rows = [&](uint32_t bit2, auto pick) -> uint32_t {
#pragma unroll 1
        for (int row = warp; row < nrows; row += kFW) {
            const int p0 = row * kFRow + 8 * lane;
            uint4 w = *reinterpret_cast<const uint4 *>(sh.bins + p0);
            const uint32_t m = pick(p0, w);
            if (m) {
                const uint32_t lo = bit2 & 0xFFFFu, hi = bit2 & 0xFFFF0000u;
                w.x |= ((m & 1u) ? lo : 0u) | ((m & 2u) ? hi : 0u);
                w.y |= ((m & 4u) ? lo : 0u) | ((m & 8u) ? hi : 0u);
                w.z |= ((m & 16u) ? lo : 0u) | ((m & 32u) ? hi : 0u);
                w.w |= ((m & 64u) ? lo : 0u) | ((m & 128u) ? hi : 0u);
                *reinterpret_cast<uint4 *>(sh.bins + p0) = w;
            }
            uint32_t cnt = __popc(m);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
            if (lane == 0) sh.rowcnt[row] = cnt;
        }
        __syncthreads();
        uint32_t total;
        const uint32_t v = tid < nrows ? sh.rowcnt[tid] : 0u;
        const uint32_t run = cta_excl_scan(v, sh.wtot, &total);
        if (tid < nrows) sh.rowcnt[tid] = run;
        __syncthreads();
        return total;
    };
    const uint32_t kSure = 0x80008000u, kWin = 0x40004000u;
    const uint32_t n_sure = k > 0 ? mark_rows(kSure, [&](int, uint4 w) -> uint32_t {
        return mask8(half_gt(w.x, b2), half_gt(w.y, b2), half_gt(w.z, b2), half_gt(w.w, b2));
    }) : 0u;

    // per-head LUTs: q_h[4s:4s+4] . c[s][j] (the codebook again, from L2)
    {
        const float4 *cb = reinterpret_cast<const float4 *>(a.codebook) + static_cast<size_t>(seg) * kSubspaces * kClusters;
#pragma unroll 1
        for (int r = tid; r < kSubspaces * kClusters; r += kFT) {
            const int s = r >> 4;
            const float4 c4 = __ldg(cb + r);
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                float v = sh.qs[g][4 * s] * c4.x;
                v = fmaf(sh.qs[g][4 * s + 1], c4.y, v);
                v = fmaf(sh.qs[g][4 * s + 2], c4.z, v);
                v = fmaf(sh.qs[g][4 * s + 3], c4.w, v);
                sh.u.at.luth[r][g] = v;
            }
        }
    }
    const int n_sinks = min(a.num_sinks, n_tok);
    const int my_sinks = (n_sinks > c) ? (n_sinks - c + a.cps - 1) / a.cps : 0;   // sinks t = c (mod cps)
    if (tid < GM) {
        sh.run_m[tid] = -INFINITY;
        sh.run_l[tid] = 0.f;
    }
    float o[GM][4];
#pragma unroll
    for (int g = 0; g < GM; ++g) o[g][0] = o[g][1] = o[g][2] = o[g][3] = 0.f;
    uint32_t win_before = 0;           // this thread's share of winners with token < t0
    uint32_t n_win = 0;

#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        uint32_t n_sel = n_sure, bit2 = kSure, n_list = n_sure + static_cast<uint32_t>(my_sinks);
        if (pass == 1) {
            // ---- exact winners among the threshold-bin candidates (the same
            // answer in every CTA): a candidate wins when fewer than `need`
            // candidates come before it (key descending, token ascending)
            cta_wait(&ctl->arrive2, a.cps, a.status);
            for (int i = tid; i < kFMaxChunk / 32; i += kFT) sh.u.sel.winbits[i] = 0;
            __syncthreads();
            if (k > 0) {
                const int ncand = min(__ldcg(&ctl->ncand), a.cand_cap);
                const uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
                const uint32_t need = static_cast<uint32_t>(k) - above_bstar;   // >= 1
                if (ncand <= kFRankMax) {
                    for (int e = tid; e < ncand; e += kFT) {
                        const uint2 v = __ldcg(cand + e);
                        sh.u.sel.ckey[e] = v.x;
                        sh.u.sel.cidx[e] = static_cast<int32_t>(v.y);
                    }
                    __syncthreads();
                    for (int e = tid; e < ncand; e += kFT) {
                        const uint32_t ke = sh.u.sel.ckey[e], ie = static_cast<uint32_t>(sh.u.sel.cidx[e]);
                        uint32_t rank = 0;
                        for (int f = 0; f < ncand; ++f) {
                            const uint32_t kf = sh.u.sel.ckey[f];
                            rank += (kf > ke) || (kf == ke && static_cast<uint32_t>(sh.u.sel.cidx[f]) < ie);
                        }
                        if (rank < need) {
                            const int rel = static_cast<int>(ie) - t0;
                            if (rel >= 0 && rel < a.chunk) atomicOr(&sh.u.sel.winbits[rel >> 5], 1u << (rel & 31));
                            else if (rel < 0) ++win_before;
                        }
                    }
                } else {
                    win_before += refine_by_radix(cand, ncand, need, t0, a.chunk, sh.u.sel.winbits, sh.hist, sh.wtot,
                                                  sh.sc);
                }
                __syncthreads();
                n_win = mark_rows(kWin, [&](int p0, uint4 w) -> uint32_t {
                    const uint32_t eq = mask8(half_eq(w.x, b2), half_eq(w.y, b2), half_eq(w.z, b2), half_eq(w.w, b2));
                    return eq ? (eq & ((sh.u.sel.winbits[p0 >> 5] >> (p0 & 31)) & 0xFFu)) : 0u;
                });
            }
            n_sel = n_win;
            bit2 = kWin;
            n_list = n_win;
        }
#pragma unroll 1
        for (uint32_t wbase = 0; wbase < n_list; wbase += kFListCap) {
            // stage the window [wbase, wbase + kFListCap) of this pass's list:
            // selected tokens in ascending order, then (first pass) the sinks
            const uint32_t wn = min(static_cast<uint32_t>(kFListCap), n_list - wbase);
#pragma unroll 1
            for (int row = warp; row < nrows; row += kFW) {
                const uint32_t m = row_mask(row, bit2);
                uint32_t incl = __popc(m);
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t o2 = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += o2;
                }
                uint32_t ord = sh.rowcnt[row] + incl - __popc(m);
                for (uint32_t mm = m; mm; mm &= mm - 1, ++ord) {
                    const int t = t0 + row * kFRow + 8 * lane + __ffs(mm) - 1;
                    if (ord >= wbase && ord < wbase + kFListCap) sh.u.at.list[ord - wbase] = t;
                }
            }
            for (uint32_t e = tid; e < wn; e += kFT) {
                const uint32_t ord = wbase + e;
                if (ord >= n_sel) sh.u.at.list[e] = -1 - static_cast<int32_t>(c + (ord - n_sel) * a.cps);   // a sink
            }
            __syncthreads();
#pragma unroll 1
            for (uint32_t tbase = 0; tbase < wn; tbase += kFTile) {
                const uint32_t tile_n = min(static_cast<uint32_t>(kFTile), wn - tbase);
                // logits, one list entry per thread
                {
                    float lg[GM];
#pragma unroll
                    for (int g = 0; g < GM; ++g) lg[g] = -INFINITY;
                    if (static_cast<uint32_t>(tid) < tile_n) {
                        const int32_t ent = sh.u.at.list[tbase + tid];
                        float acc[GM];
#pragma unroll
                        for (int g = 0; g < GM; ++g) acc[g] = 0.f;
                        if (ent >= 0) {
                            const uint4 row = __ldg(crow + ent);
                            const uint32_t w[4] = {row.x, row.y, row.z, row.w};
#pragma unroll 8
                            for (int s = 0; s < kSubspaces; ++s) {
                                const int j = (w[s >> 3] >> (4 * (s & 7))) & 15;
                                const float *lp = sh.u.at.luth[s * kClusters + j];
#pragma unroll
                                for (int g = 0; g < GM; g += 4) {
                                    const float4 v4 = *reinterpret_cast<const float4 *>(lp + g);
                                    acc[g] += v4.x;
                                    acc[g + 1] += v4.y;
                                    acc[g + 2] += v4.z;
                                    acc[g + 3] += v4.w;
                                }
                            }
#pragma unroll
                            for (int g = 0; g < GM; ++g) lg[g] = (acc[g] + sh.qmu_h[g]) * a.scale;
                        } else {
                            const char *krow = static_cast<const char *>(a.K) + (kv_seg + (-1 - ent)) * kHeadDim * EB;
#pragma unroll 2
                            for (int d = 0; d < kHeadDim; d += 4) {
                                const float4 kv = load4<DT>(krow, d);
#pragma unroll
                                for (int g = 0; g < GM; ++g) {
                                    acc[g] = fmaf(sh.qs[g][d], kv.x, acc[g]);
                                    acc[g] = fmaf(sh.qs[g][d + 1], kv.y, acc[g]);
                                    acc[g] = fmaf(sh.qs[g][d + 2], kv.z, acc[g]);
                                    acc[g] = fmaf(sh.qs[g][d + 3], kv.w, acc[g]);
                                }
                            }
#pragma unroll
                            for (int g = 0; g < GM; ++g) lg[g] = acc[g] * a.scale;
                        }
                    }
#pragma unroll
                    for (int g = 0; g < GM; ++g) {
                        const float v = (g < group) ? lg[g] : -INFINITY;
                        sh.u.at.logit[g][tid] = v;
                        float mx = v;
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                        if (lane == 0) sh.tile_stat[warp][g] = mx;
                    }
                }
                __syncthreads();
                // new running max per head and the rescale factor of what came before
                float alpha[GM], mnew[GM];
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    float mx = sh.run_m[g];
                    for (int w = 0; w < kFW; ++w) mx = fmaxf(mx, sh.tile_stat[w][g]);
                    mnew[g] = mx;
                    alpha[g] = (sh.run_m[g] == -INFINITY) ? 0.f : __expf(sh.run_m[g] - mx);
                }
                __syncthreads();
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    const float lv = sh.u.at.logit[g][tid];
                    const float pr = (lv == -INFINITY) ? 0.f : __expf(lv - mnew[g]);
                    sh.u.at.logit[g][tid] = pr;
                    float sm = pr;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
                    if (lane == 0) sh.tile_stat[warp][g] = sm;
                }
                __syncthreads();
                if (tid < GM) {
                    float sm = 0.f;
                    for (int w = 0; w < kFW; ++w) sm += sh.tile_stat[w][tid];
                    sh.run_l[tid] = sh.run_l[tid] * alpha[tid] + sm;
                    sh.run_m[tid] = mnew[tid];
                }
                // o = alpha o + sum_e p_e V[t_e]; warp w takes entries w, w + 8, ...
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    o[g][0] *= alpha[g];
                    o[g][1] *= alpha[g];
                    o[g][2] *= alpha[g];
                    o[g][3] *= alpha[g];
                }
#pragma unroll 1
                for (uint32_t e0 = warp; e0 < tile_n; e0 += kFVRows * kFW) {
                    float4 v[kFVRows];
#pragma unroll
                    for (int u = 0; u < kFVRows; ++u) {
                        const uint32_t e = e0 + u * kFW;
                        if (e < tile_n) {
                            const int32_t ent = sh.u.at.list[tbase + e];
                            const int t = ent >= 0 ? ent : -1 - ent;
                            v[u] = load4<DT>(static_cast<const char *>(a.V) + (kv_seg + t) * kHeadDim * EB, lane * 4);
                        } else {
                            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kFVRows; ++u) {
                        const uint32_t e = e0 + u * kFW;
                        const float4 vv = v[u];
#pragma unroll
                        for (int g = 0; g < GM; ++g) {
                            const float pr = e < tile_n ? sh.u.at.logit[g][e] : 0.f;
                            o[g][0] = fmaf(pr, vv.x, o[g][0]);
                            o[g][1] = fmaf(pr, vv.y, o[g][1]);
                            o[g][2] = fmaf(pr, vv.z, o[g][2]);
                            o[g][3] = fmaf(pr, vv.w, o[g][3]);
                        }
                    }
                }
                __syncthreads();
            }
        }
    }

    // selected tokens in ascending order into idx_out, after the selected
    // tokens of the earlier chunks (their higher-bin counts plus their winners)
    if (a.idx_out && k > 0) {
        uint32_t before = win_before;
        for (int cc = tid; cc < c; cc += kFT)
            before += static_cast<uint32_t>(__ldcg(a.selcnt + static_cast<size_t>(seg) * a.cps + cc));
        uint32_t out_base;
        cta_excl_scan(before, sh.wtot, &out_base);
#pragma unroll 1
        for (int row = warp; row < nrows; row += kFW) {
            const uint32_t m = row_mask(row, kSure | kWin);
            uint32_t cnt = __popc(m);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
            if (lane == 0) sh.rowcnt[row] = cnt;
        }
        __syncthreads();
        {
            uint32_t total;
            const uint32_t v = tid < nrows ? sh.rowcnt[tid] : 0u;
            const uint32_t run = cta_excl_scan(v, sh.wtot, &total);
            if (tid < nrows) sh.rowcnt[tid] = run;
            __syncthreads();
        }
        int32_t *io = a.idx_out + static_cast<size_t>(seg) * a.kmax;
#pragma unroll 1
        for (int row = warp; row < nrows; row += kFW) {
            const uint32_t m = row_mask(row, kSure | kWin);
            uint32_t incl = __popc(m);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t o2 = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o2;
            }
            uint32_t ord = out_base + sh.rowcnt[row] + incl - __popc(m);
            for (uint32_t mm = m; mm; mm &= mm - 1, ++ord)
                if (ord < static_cast<uint32_t>(k)) io[ord] = t0 + row * kFRow + 8 * lane + __ffs(mm) - 1;
        }
    }

    // reduce o over the warps and write this CTA's partial
#pragma unroll
    for (int g = 0; g < GM; ++g)
        *reinterpret_cast<float4 *>(&sh.u.at.red[warp][g][lane * 4]) = make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
    __syncthreads();
    {
        const size_t pb = (static_cast<size_t>(seg) * a.cps + c) * GM;
        for (int e = tid; e < GM * kHeadDim; e += kFT) {
            const int g = e / kHeadDim, d = e % kHeadDim;
            float s = sh.u.at.red[0][g][d];
#pragma unroll
            for (int w = 1; w < kFW; ++w) s += sh.u.at.red[w][g][d];
            a.part_o[(pb + g) * kHeadDim + d] = s;
        }
        if (tid < GM) a.part_ml[pb + tid] = make_float2(sh.run_m[tid], sh.run_l[tid]);
    }

    // ---- last CTA of the segment: merge partials, reset coordination state
    const int old = cta_arrive(&ctl->arrive3);
    if (tid == 0) sh.last = (old == a.cps - 1);
    __syncthreads();
    if (!sh.last) return;
    __threadfence();
#pragma unroll 1
    for (int e = tid; e < group * kHeadDim; e += kFT) {
        const int g = e / kHeadDim, d = e % kHeadDim;
        float mx = -INFINITY;
        for (int cc = 0; cc < a.cps; ++cc)
            mx = fmaxf(mx, __ldcg(a.part_ml + (static_cast<size_t>(seg) * a.cps + cc) * GM + g).x);
        float l = 0.f, acc = 0.f;
        if (mx != -INFINITY) {
            for (int cc = 0; cc < a.cps; ++cc) {
                const size_t pb = (static_cast<size_t>(seg) * a.cps + cc) * GM + g;
                const float2 ml = __ldcg(a.part_ml + pb);
                const float wgt = (ml.x == -INFINITY) ? 0.f : __expf(ml.x - mx);
                l = fmaf(ml.y, wgt, l);
                acc = fmaf(__ldcg(a.part_o + pb * kHeadDim + d), wgt, acc);
            }
        }
        const float r = (l > 0.f) ? __fdividef(acc, l) : 0.f;
        const size_t orow = (static_cast<size_t>(b) * a.hq + static_cast<size_t>(h) * group + g) * kHeadDim + d;
        if (DT == SIKV_DTYPE_F32)
            static_cast<float *>(a.out)[orow] = r;
        else
            static_cast<unsigned short *>(a.out)[orow] = static_cast<unsigned short>(f32_to_bf16_bits(r));
    }
    if (a.idx_out) {
        int32_t *io = a.idx_out + static_cast<size_t>(seg) * a.kmax;
        for (int i = k + tid; i < a.kmax; i += kFT) io[i] = -1;
    }
    uint32_t *gh = a.ghist + static_cast<size_t>(seg) * kFBins;
    for (int i = tid; i < kFBins; i += kFT) gh[i] = 0;
    if (tid == 0) {
        ctl->arrive1 = 0;
        ctl->arrive2 = 0;
        ctl->arrive3 = 0;
        ctl->ncand = 0;
    }
}

template <int DT, int GM>
sikv_status launch_fused_t(const FusedArgs &args, const FusedPlan &plan, cudaStream_t stream) {
    auto kern = decode_fused_kernel<DT, GM>;
    const size_t smem = sizeof(FusedSmem<GM>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SIKV_ERR_CUDA;
    FusedArgs a = args;
    void *params[] = {&a};
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(plan.grid),
                                                      dim3(kFT), params, smem, stream);
    return e == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

template <int DT, int GM>
int occupancy_of() {
    // the occupancy calculator honours the kernel's dynamic shared-memory
    // limit, which must be raised above the 48 KB default first
    auto kern = decode_fused_kernel<DT, GM>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FusedSmem<GM>)) !=
        cudaSuccess)
        return 0;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kFT, sizeof(FusedSmem<GM>)) != cudaSuccess)
        return 0;
    return blocks;
}

}  // namespace

size_t fused_cand_cap(const sikv_params &p) { return static_cast<size_t>(p.max_seq_len); }

FusedLayout fused_layout(const sikv_params &p, size_t base) {
    FusedLayout L;
    const size_t segs = static_cast<size_t>(p.batch) * p.num_kv_heads;
    const int gm = (p.num_q_heads / p.num_kv_heads) <= 4 ? 4 : 8;
    size_t off = align_up(base, 256);
    L.ghist = off;
    off = align_up(off + segs * kFBins * sizeof(uint32_t), 256);
    L.ctl = off;
    off = align_up(off + segs * sizeof(FusedCtl), 256);
    L.cand = off;
    off = align_up(off + segs * fused_cand_cap(p) * sizeof(uint2), 256);
    L.selcnt = off;
    off = align_up(off + segs * kFusedMaxCps * sizeof(int32_t), 256);
    L.part_o = off;
    off = align_up(off + segs * kFusedMaxCps * gm * kHeadDim * sizeof(float), 256);
    L.part_ml = off;
    off = align_up(off + segs * kFusedMaxCps * gm * sizeof(float2), 256);
    L.total = off;
    return L;
}

FusedPlan fused_plan(const sikv_params &p) {
    FusedPlan plan;
    const int group = p.num_q_heads / p.num_kv_heads;
    const int gm = group <= 4 ? 4 : 8;
    const int segs = p.batch * p.num_kv_heads;
    const int sms = device_sm_count();
    if (sms <= 0) return plan;
    int occ = 0;
    if (p.dtype == SIKV_DTYPE_BF16)
        occ = gm == 4 ? occupancy_of<SIKV_DTYPE_BF16, 4>() : occupancy_of<SIKV_DTYPE_BF16, 8>();
    else
        occ = gm == 4 ? occupancy_of<SIKV_DTYPE_F32, 4>() : occupancy_of<SIKV_DTYPE_F32, 8>();
    if (occ < 1) return plan;
    int cps = (sms * occ) / segs;
    const int min_chunk = 2048;
    cps = std::min(cps, (p.max_seq_len + min_chunk - 1) / min_chunk);
    cps = std::min(cps, kFusedMaxCps);
    if (cps < 1) return plan;                     // more segments than co-resident CTAs
    int chunk = (p.max_seq_len + cps - 1) / cps;
    chunk = (chunk + kFT - 1) / kFT * kFT;
    cps = (p.max_seq_len + chunk - 1) / chunk;
    if (chunk > kFMaxChunk) return plan;
    plan.ok = true;
    plan.cps = cps;
    plan.chunk = chunk;
    plan.npt = chunk / kFT;
    plan.gm = gm;
    plan.grid = segs * cps;
    return plan;
}

sikv_status launch_decode_fused(const sikv_params &p, const FusedPlan &plan, const void *q, const void *K,
                                const void *V, const uint8_t *codes, const float *codebook, const float *mu,
                                const int32_t *seq_lens, const int32_t *k_per_seq, void *out, int32_t *idx_out,
                                float *scores_out, char *ws, size_t base, int32_t *status, cudaStream_t stream) {
    const FusedLayout L = fused_layout(p, base);
    FusedArgs a;
    a.q = q;
    a.K = K;
    a.V = V;
    a.codes = codes;
    a.codebook = codebook;
    a.mu = mu;
    a.seq_lens = seq_lens;
    a.k_per_seq = k_per_seq;
    a.out = out;
    a.idx_out = idx_out;
    a.scores_out = scores_out;
    a.hq = p.num_q_heads;
    a.hkv = p.num_kv_heads;
    a.nmax = p.max_seq_len;
    a.num_sinks = p.num_sinks;
    a.kmax = p.max_topk;
    a.cps = plan.cps;
    a.chunk = plan.chunk;
    a.npt = plan.npt;
    a.cand_cap = static_cast<int>(fused_cand_cap(p));
    a.scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf(static_cast<float>(p.head_dim));
    a.ghist = reinterpret_cast<uint32_t *>(ws + L.ghist);
    a.cand = reinterpret_cast<uint2 *>(ws + L.cand);
    a.ctl = reinterpret_cast<FusedCtl *>(ws + L.ctl);
    a.selcnt = reinterpret_cast<int32_t *>(ws + L.selcnt);
    a.part_o = reinterpret_cast<float *>(ws + L.part_o);
    a.part_ml = reinterpret_cast<float2 *>(ws + L.part_ml);
    a.status = status;
    if (p.dtype == SIKV_DTYPE_BF16)
        return plan.gm == 4 ? launch_fused_t<SIKV_DTYPE_BF16, 4>(a, plan, stream)
                            : launch_fused_t<SIKV_DTYPE_BF16, 8>(a, plan, stream);
    return plan.gm == 4 ? launch_fused_t<SIKV_DTYPE_F32, 4>(a, plan, stream)
                        : launch_fused_t<SIKV_DTYPE_F32, 8>(a, plan, stream);
}

}  // namespace sikv
