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
#include <atomic>

#include "decode_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kSpinLimit = 1 << 23;      // polls of a wait: seconds, far above any real wait

struct FusedArgs {
    const void *q, *K, *V;
    const uint8_t *vq;    // 2-bit value rows of the selected tokens (VQ kernels only)
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
            // candidate (key, token) as one 64-bit value: key above the
            // inverted token, so a larger value ranks first (ties: lower token)
            unsigned long long ck[kFRankMax];
            uint32_t winbits[kFMaxChunk / 32];
        } sel;
        struct {
            int32_t list[kFListCap];
            union {
                alignas(16) float red[kFW][GM][kHeadDim];     // the warps' outputs at the end
                alignas(16) char vbuf[kFW][kFVBytes];         // each warp's staged value rows
            };
            alignas(16) float luth[kSubspaces * kClusters][GM];   // per-head LUT, [s*16+j][g]
            int32_t tok[kFW][32];                                 // each warp's batch tokens
        } at;
    } u;
    alignas(16) float qs[GM][kHeadDim];
    alignas(16) float mus[kHeadDim];
    alignas(16) float qmu_h[GM];
    alignas(16) float wm[kFW][GM];            // per-warp softmax state at the end
    alignas(16) float wl[kFW][GM];
    // the scoring histogram; from phase 2 on the threshold-bin tokens (offsets
    // in [0, kFPend), their keys in [kFPend, 2 kFPend)) and the direct list of
    // attended tokens in [2 kFPend, kFBins)
    uint32_t hist[kFBins];
    // one entry per token of the chunk, in token order (entry p: token t0 + p,
    // scored by thread p mod 256): its bin + 1 (0: no token) in bits 0-13,
    // bit 15 set once the token is above the segment's threshold bin, bit 14
    // once it wins in the threshold bin.  Holds the codebook before scoring.
    alignas(16) uint16_t bins[kFMaxChunk];
    uint32_t rowcnt[kFMaxChunk / 256];        // selected tokens per row of 256, then their prefix
    uint32_t wtot[kFW + 1];
    uint32_t wcnt[kFW];                       // tokens in each warp's direct list
    uint32_t sc[16];
    float bin_lo, bin_inv;
    int bin_flat, last;
};

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Thread 0 waits until *ctr >= target (bounded); the CTA then synchronizes.
// The acquire load orders every later read of the CTA after the arrivals.
__device__ __forceinline__ void cta_wait(const int *ctr, int target, int32_t *status) {
    if (threadIdx.x == 0) {
        int it = 0;
        while (ld_acquire(ctr) < target) {
            if (++it > kSpinLimit) {
                flag_error(status, SIKV_DEVERR_TIMEOUT);
                break;
            }
            __nanosleep(64);
        }
    }
    __syncthreads();
}

// After the CTA barrier thread 0 fences (cumulative over the writes of the
// CTA that the barrier ordered before it) and arrives.  Returns the
// counter's previous value to thread 0 (others get 0).
__device__ __forceinline__ int cta_arrive(int *ctr) {
    __syncthreads();
    int old = 0;
    if (threadIdx.x == 0) {
        __threadfence();
        old = atomicAdd(ctr, 1);
    }
    return old;
}


template <int DT, int GM, bool VQ>
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

    // ---- tables.  Their inputs are requested first; while they travel, the
    // first code rows and this CTA's share of the sink rows go to L2 (the
    // prologue would otherwise leave HBM idle).
    TableInputs<DT> tin;
    tin.load(a.q, a.codebook, a.mu, b, h, a.hq, group, seg);
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
    for (int i = tid; i < kFBins; i += kFT) sh.hist[i] = 0;
    __syncthreads();
    tin.store(&sh.qs[0][0], cbs, sh.mus, group);
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
    const float bin_mul = sh.bin_flat ? 0.f : sh.bin_inv;
    const float bin_add = sh.bin_flat ? 0.f : -sh.bin_lo * sh.bin_inv;
    const float qmu = sh.u.tab.qmu;

    // ---- scores of this chunk -> histogram and per-slot bins
    {
        float *so = a.scores_out ? a.scores_out + kv_seg : nullptr;
        // Two register groups of kFUnroll rows per thread, ping-ponged: one is
        // scored while the other is in flight.  Loads are guarded only by the
        // warp-uniform slot count; their token index is clamped into the cache
        // (rows of sinks or past the sequence are loaded and discarded).
        const int tmax = a.nmax - 1;
        const uint32_t span = static_cast<uint32_t>(max(t1 - tstart, 0));   // scored tokens of the chunk
        uint4 ra[kFUnroll], rb[kFUnroll];
#pragma unroll
        for (int u = 0; u < kFUnroll; ++u) ra[u] = rb[u] = make_uint4(0u, 0u, 0u, 0u);
        auto load_group = [&](uint4 (&r)[kFUnroll], int i0) {
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u)
                if (i0 + u < npt) r[u] = __ldcs(crow + min(t0 + kFT * (i0 + u) + my, tmax));
        };
        auto score_group = [&](const uint4 (&r)[kFUnroll], int i0) {
            float sc2[kFUnroll];
#pragma unroll
            for (int u = 0; u < kFUnroll; u += 2) {
                const float2 v = lut2_score2(sh.u.tab.t2, r[u], r[u + 1], lane, qmu);
                sc2[u] = v.x;
                sc2[u + 1] = v.y;
            }
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u) {
                const int i = i0 + u;
                if (i >= npt) break;
                const int t = t0 + kFT * i + my;
                uint32_t e = 0;
                if (static_cast<uint32_t>(t - tstart) < span) {
                    const float sv = sc2[u];
                    // sv >= the lowest possible score up to rounding; a negative
                    // value converts to 0
                    const uint32_t bi = min(__float2uint_rz(fmaf(sv, bin_mul, bin_add)), static_cast<uint32_t>(kFBins - 1));
                    atomicAdd(&sh.hist[bi], 1u);
                    e = bi + 1u;
                    if (so) so[t] = sv;
                } else if (so && t < t1) {
                    so[t] = -INFINITY;
                }
                sh.bins[i * kFT + tid] = static_cast<uint16_t>(e);
            }
        };
        load_group(ra, 0);
#pragma unroll 1
        for (int i0 = 0; i0 < npt; i0 += 2 * kFUnroll) {
            load_group(rb, i0 + kFUnroll);
            score_group(ra, i0);
            if (i0 + kFUnroll >= npt) break;
            load_group(ra, i0 + 2 * kFUnroll);
            score_group(rb, i0 + kFUnroll);
        }
    }
    __syncthreads();

    // ---- 1. local k-th bin, publish the bins at or above it
    if (k > 0) {
        if (tid == 0) {
            sh.sc[0] = 0;
            sh.sc[1] = 0;
            sh.sc[8] = 0;     // threshold-bin tokens listed
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
    // this thread's codebook rows for the per-head LUTs, fetched during the wait
    constexpr int kCbPer = kSubspaces * kClusters / kFT;
    float4 cbr[kCbPer];
    {
        const float4 *cb = reinterpret_cast<const float4 *>(a.codebook) + static_cast<size_t>(seg) * kSubspaces * kClusters;
#pragma unroll
        for (int i = 0; i < kCbPer; ++i) cbr[i] = __ldg(cb + tid + i * kFT);
    }
    cta_wait(&ctl->arrive1, a.cps, a.status);

    // ---- 2. segment k-th bin b*.  Tokens above it are selected outright:
    // flagged (entry bit 15), listed for the attention and their code and
    // value rows sent to L2.  Tokens in b* are listed, re-scored together and
    // appended with their exact keys to the segment's candidates.
    const int nrows = (a.chunk + kFRow - 1) / kFRow;           // <= 64
    const uint32_t kSure = 0x80008000u, kWin = 0x40004000u;
    int bstar = kFBins;              // nothing selected when k == 0
    uint32_t above_bstar = 0, n_sure = 0;
    const char *vseg = static_cast<const char *>(a.V) + kv_seg * kHeadDim * EB;
    // value rows of the selected tokens: V itself, or its 2-bit rows (sinks
    // always read V)
    const char *vsel = VQ ? reinterpret_cast<const char *>(a.vq) + kv_seg * kVqRowBytes : vseg;
    uint32_t *pend = sh.hist;                                        // free: the local histogram is published
    // each warp's direct list of attended tokens (kFWarpList entries)
    int32_t *wlist = reinterpret_cast<int32_t *>(sh.hist) + 2 * kFPend + kFWarpList * warp;
    if (lane == 0) sh.wcnt[warp] = 0;
    if (k > 0) {
        const uint32_t *gh = a.ghist + static_cast<size_t>(seg) * kFBins;
        cta_find_bin<kFBins / kFT>([&](int i) { return __ldcg(gh + i); }, static_cast<uint32_t>(k), sh.wtot, sh.sc);
        bstar = static_cast<int>(sh.sc[0]);
        above_bstar = sh.sc[1];
        const uint32_t b2 = static_cast<uint32_t>(bstar + 1) * 0x10001u;
        // warp w scans rows w, w + 8, ... (at most 8) of 256 entries, 8 per
        // lane: it flags the tokens above b* and keeps, per lane, a 64-bit mask
        // of them (bit 8 r + j: entry j of the lane's r-th row) and of the
        // tokens in b*.  One pass over the masks then lists them: lane by
        // lane, row by row (a fixed order), positions from 7 ballots.
        unsigned long long gmask = 0ull, emask = 0ull;
#pragma unroll 1
        for (int r = 0, row = warp; row < nrows; ++r, row += kFW) {
            const int p0 = row * kFRow + 8 * lane;
            uint4 w = *reinterpret_cast<const uint4 *>(sh.bins + p0);
            const uint32_t gx = half_gt(w.x, b2), gy = half_gt(w.y, b2), gz = half_gt(w.z, b2), gw = half_gt(w.w, b2);
            const uint32_t ex = half_eq(w.x, b2), ey = half_eq(w.y, b2), ez = half_eq(w.z, b2), ew = half_eq(w.w, b2);
            if (gx | gy | gz | gw) {
                w.x |= sure_flags(gx);
                w.y |= sure_flags(gy);
                w.z |= sure_flags(gz);
                w.w |= sure_flags(gw);
                *reinterpret_cast<uint4 *>(sh.bins + p0) = w;
                gmask |= static_cast<unsigned long long>(mask8(gx, gy, gz, gw)) << (8 * r);
            }
            if (ex | ey | ez | ew) emask |= static_cast<unsigned long long>(mask8(ex, ey, ez, ew)) << (8 * r);
        }
        const uint32_t below = (1u << lane) - 1u;
        const uint32_t cnt = __popcll(gmask);
        uint32_t pos = 0, n_w = 0;
#pragma unroll
        for (int bit = 0; bit < 7; ++bit) {
            const uint32_t bb = __ballot_sync(0xffffffffu, (cnt >> bit) & 1u);
            pos += static_cast<uint32_t>(__popc(bb & below)) << bit;
            n_w += static_cast<uint32_t>(__popc(bb)) << bit;
        }
        for (unsigned long long mm = gmask; mm; mm &= mm - 1, ++pos) {
            const int bit = __ffsll(static_cast<long long>(mm)) - 1;
            const int t = t0 + (warp + kFW * (bit >> 3)) * kFRow + 8 * lane + (bit & 7);
            if (pos < static_cast<uint32_t>(kFWarpList)) wlist[pos] = t;
            prefetch_l2(crow + t);
            if (VQ) {                              // a 48-byte row may straddle two lines
                prefetch_l2(vsel + static_cast<size_t>(t) * kVqRowBytes);
                prefetch_l2(vsel + static_cast<size_t>(t) * kVqRowBytes + kVqRowBytes - 1);
            } else {
                prefetch_l2(vseg + static_cast<size_t>(t) * kHeadDim * EB);
                if (EB * kHeadDim > 128) prefetch_l2(vseg + static_cast<size_t>(t) * kHeadDim * EB + 128);
            }
        }
        for (unsigned long long mm = emask; mm; mm &= mm - 1) {
            const int bit = __ffsll(static_cast<long long>(mm)) - 1;
            const int p = (warp + kFW * (bit >> 3)) * kFRow + 8 * lane + (bit & 7);
            const uint32_t slot = atomicAdd(&sh.sc[8], 1u);
            if (slot < kFPend) pend[slot] = static_cast<uint32_t>(p);
            prefetch_l2(crow + t0 + p);            // re-read below
        }
        if (lane == 0) sh.wcnt[warp] = n_w;
        __syncthreads();
        n_sure = 0;
#pragma unroll
        for (int w2 = 0; w2 < kFW; ++w2) n_sure += sh.wcnt[w2];
        if (tid == 0) a.selcnt[static_cast<size_t>(seg) * a.cps + c] = static_cast<int32_t>(n_sure);
        const uint32_t npend = sh.sc[8];
        uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
        if (npend <= static_cast<uint32_t>(kFPend)) {
            // one slot reservation for the CTA, issued before the re-scoring
            int cbase = 0;
            if (tid == 0 && npend > 0) cbase = atomicAdd(&ctl->ncand, static_cast<int>(npend));
            // token t0 + p was scored by lane p mod 32 (the table's bank
            // rotation): warp e mod 8 takes pending token e in that lane
#pragma unroll 1
            for (uint32_t e = warp; e < npend; e += kFW) {
                const int p = static_cast<int>(pend[e]);
                if (lane == (p & 31))
                    pend[kFPend + e] = score_key(lut2_score(sh.u.tab.t2, __ldg(crow + t0 + p), lane, qmu));
            }
            if (tid == 0) sh.sc[9] = static_cast<uint32_t>(cbase);
            __syncthreads();
            const uint32_t base0 = sh.sc[9];
            for (uint32_t e = tid; e < npend; e += kFT)
                if (base0 + e < static_cast<uint32_t>(a.cand_cap))
                    cand[base0 + e] = make_uint2(pend[kFPend + e], static_cast<uint32_t>(t0) + pend[e]);
        } else {
            emit_bin_tokens(sh.bins, nrows, b2, sh.u.tab.t2, crow, t0, qmu, &ctl->ncand, cand, a.cand_cap);
        }
    }
    cta_arrive(&ctl->arrive2);

    // Attention.  Each warp keeps its own online softmax; the warps' states
    // merge once at the end.  The sinks and the tokens above b* need no
    // candidate ranking, so they are attended while the other CTAs finish
    // their candidates; the winners of b* follow after the wait.
    // The sinks t = c (mod cps): one warp per sink, lane l takes columns
    // 4l..4l+3 of its stored key and value.  The first sink's rows are
    // fetched before the LUTs are built.
    const int n_sinks = min(a.num_sinks, n_tok);
    const int my_sinks = (n_sinks > c) ? (n_sinks - c + a.cps - 1) / a.cps : 0;
    const char *kseg = static_cast<const char *>(a.K) + kv_seg * kHeadDim * EB;
    float4 sk_k = make_float4(0.f, 0.f, 0.f, 0.f), sk_v = sk_k;
    if (warp < my_sinks) {
        const size_t off = static_cast<size_t>(c + warp * a.cps) * kHeadDim * EB;
        sk_k = load4<DT>(kseg + off, 4 * lane);
        sk_v = load4<DT>(vseg + off, 4 * lane);
    }
    // per-head LUTs: q_h[4s:4s+4] . c[s][j]
#pragma unroll
    for (int i = 0; i < kCbPer; ++i) {
        const int r = tid + i * kFT, sidx = r >> 4;
        const float4 c4 = cbr[i];
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            float v = sh.qs[g][4 * sidx] * c4.x;
            v = fmaf(sh.qs[g][4 * sidx + 1], c4.y, v);
            v = fmaf(sh.qs[g][4 * sidx + 2], c4.z, v);
            v = fmaf(sh.qs[g][4 * sidx + 3], c4.w, v);
            sh.u.at.luth[r][g] = v;
        }
    }
    WarpSoftmax<GM> ws;
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        ws.m[g] = -INFINITY;
        ws.l[g] = 0.f;
        ws.o[g][0] = ws.o[g][1] = ws.o[g][2] = ws.o[g][3] = 0.f;
    }
#pragma unroll 1
    for (int i = warp; i < my_sinks; i += kFW) {
        if (i != warp) {
            const size_t off = static_cast<size_t>(c + i * a.cps) * kHeadDim * EB;
            sk_k = load4<DT>(kseg + off, 4 * lane);
            sk_v = load4<DT>(vseg + off, 4 * lane);
        }
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            float d = sh.qs[g][4 * lane] * sk_k.x;
            d = fmaf(sh.qs[g][4 * lane + 1], sk_k.y, d);
            d = fmaf(sh.qs[g][4 * lane + 2], sk_k.z, d);
            d = fmaf(sh.qs[g][4 * lane + 3], sk_k.w, d);
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o2);
            const float lgv = (g < group) ? d * a.scale : -INFINITY;
            const float mn = fmaxf(ws.m[g], lgv);
            const float alpha = (ws.m[g] == -INFINITY) ? 0.f : __expf(ws.m[g] - mn);
            const float pr = (lgv == -INFINITY) ? 0.f : __expf(lgv - mn);
            ws.l[g] = fmaf(ws.l[g], alpha, pr);
            ws.m[g] = mn;
            ws.o[g][0] = fmaf(pr, sk_v.x, ws.o[g][0] * alpha);
            ws.o[g][1] = fmaf(pr, sk_v.y, ws.o[g][1] * alpha);
            ws.o[g][2] = fmaf(pr, sk_v.z, ws.o[g][2] * alpha);
            ws.o[g][3] = fmaf(pr, sk_v.w, ws.o[g][3] * alpha);
        }
    }
    __syncthreads();
    uint32_t win_before = 0;           // this thread's share of winners with token < t0
    // Each warp attends its own direct list (deterministic order) unless some
    // warp's list overflowed; then the pass's tokens are staged from the
    // entry flags in windows of kFListCap and shared out 8 lanes apart.
    bool direct = true;
    for (int w2 = 0; w2 < kFW; ++w2) direct = direct && sh.wcnt[w2] <= static_cast<uint32_t>(kFWarpList);
    uint32_t n_list = n_sure, bit2 = kSure;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        int pass_v = pass;
        asm volatile("" : "+r"(pass_v));   // keeps the two passes in one copy of the code
        if (pass_v == 1) {
            if (k == 0) break;
            // ---- exact winners among the threshold-bin candidates (the same
            // answer in every CTA): a candidate wins when fewer than `need`
            // candidates come before it (key descending, token ascending).
            // The count and the first 2 kFT entries are read together; entries
            // past the count are ignored.
            cta_wait(&ctl->arrive2, a.cps, a.status);
            const uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
            const int nc_raw = __ldcg(&ctl->ncand);
            const uint2 zero2 = make_uint2(0u, 0u);
            const uint2 c0 = (tid < a.cand_cap) ? __ldcg(cand + tid) : zero2;
            const uint2 c1 = (tid + kFT < a.cand_cap) ? __ldcg(cand + tid + kFT) : zero2;
            const int ncand = min(nc_raw, a.cand_cap);
            const uint32_t need = static_cast<uint32_t>(k) - above_bstar;   // >= 1
            const bool ranked = ncand <= kFRankMax;
            for (int i = tid; i < kFMaxChunk / 32; i += kFT) sh.u.sel.winbits[i] = 0;
            if (ranked) {
                if (tid < ncand) sh.u.sel.ck[tid] = (static_cast<unsigned long long>(c0.x) << 32) | ~c0.y;
                if (tid + kFT < ncand) sh.u.sel.ck[tid + kFT] = (static_cast<unsigned long long>(c1.x) << 32) | ~c1.y;
            }
            __syncthreads();
            if (ranked) {
                for (int e = tid; e < ncand; e += kFT) {
                    const unsigned long long me = sh.u.sel.ck[e];
                    uint32_t rank = 0;
#pragma unroll 8
                    for (int f = 0; f < ncand; ++f) rank += sh.u.sel.ck[f] > me ? 1u : 0u;
                    if (rank < need) {
                        const int rel = static_cast<int>(~static_cast<uint32_t>(me)) - t0;
                        if (rel >= 0 && rel < a.chunk) atomicOr(&sh.u.sel.winbits[rel >> 5], 1u << (rel & 31));
                        else if (rel < 0) ++win_before;
                    }
                }
            } else {
                win_before += refine_by_radix(cand, ncand, need, t0, a.chunk,
                                              sh.u.sel.winbits, sh.hist, sh.wtot, sh.sc);
            }
            __syncthreads();
            // each warp lists the winners of its share of the chunk's bitmap,
            // in ascending token order
            {
                const int nwords = (a.chunk + 31) / 32;
                const int wpw = (nwords + kFW - 1) / kFW;        // <= 64
                uint32_t n_w = 0;
#pragma unroll 1
                for (int i0 = 0; i0 < wpw; i0 += 32) {
                    const int wd = warp * wpw + i0 + lane;
                    const uint32_t bits = (i0 + lane < wpw && wd < nwords) ? sh.u.sel.winbits[wd] : 0u;
                    const uint32_t cb = __popc(bits);
                    uint32_t incl = cb;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const uint32_t o2 = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off) incl += o2;
                    }
                    uint32_t pos = n_w + incl - cb;
                    n_w += __shfl_sync(0xffffffffu, incl, 31);
                    for (uint32_t mm = bits; mm; mm &= mm - 1, ++pos)
                        if (pos < static_cast<uint32_t>(kFWarpList)) wlist[pos] = t0 + 32 * wd + __ffs(mm) - 1;
                }
                if (lane == 0) sh.wcnt[warp] = n_w;
            }
            __syncthreads();
            direct = true;
            n_list = 0;
            for (int w2 = 0; w2 < kFW; ++w2) {
                direct = direct && sh.wcnt[w2] <= static_cast<uint32_t>(kFWarpList);
                n_list += sh.wcnt[w2];
            }
            bit2 = kWin;
            if (!direct || a.idx_out) {
                // flag the winners of this chunk (entry bit 14)
                const uint32_t b2 = static_cast<uint32_t>(bstar + 1) * 0x10001u;
#pragma unroll 1
                for (int row = warp; row < nrows; row += kFW) {
                    const int p0 = row * kFRow + 8 * lane;
                    uint4 w = *reinterpret_cast<const uint4 *>(sh.bins + p0);
                    const uint32_t wb = (sh.u.sel.winbits[p0 >> 5] >> (p0 & 31)) & 0xFFu;
                    // per 16-bit half: the entry is in b* and won
                    const uint32_t hx = half_eq(w.x, b2) & halves_of(wb, 0);
                    const uint32_t hy = half_eq(w.y, b2) & halves_of(wb, 1);
                    const uint32_t hz = half_eq(w.z, b2) & halves_of(wb, 2);
                    const uint32_t hw = half_eq(w.w, b2) & halves_of(wb, 3);
                    if (hx | hy | hz | hw) {
                        w.x |= win_flags(hx);
                        w.y |= win_flags(hy);
                        w.z |= win_flags(hz);
                        w.w |= win_flags(hw);
                        *reinterpret_cast<uint4 *>(sh.bins + p0) = w;
                    }
                }
                __syncthreads();
            }
        }
        const uint32_t n_windows = direct ? 1u : (n_list + kFListCap - 1) / kFListCap;
#pragma unroll 1
        for (uint32_t win = 0; win < n_windows; ++win) {
            const int32_t *lst = wlist;
            uint32_t nl = sh.wcnt[warp], lmul = 1, ladd = 0;
            if (!direct) {
                const uint32_t wbase = win * kFListCap;
                stage_flagged(sh.bins, nrows, bit2, wbase, t0, sh.rowcnt, sh.wtot, sh.u.at.list);
                lst = sh.u.at.list;
                nl = min(static_cast<uint32_t>(kFListCap), n_list - wbase);
                lmul = 8;
                ladd = static_cast<uint32_t>(warp);
            }
            // opaque to the optimizer: one copy of the batch loop serves both list kinds
            asm volatile("" : "+l"(lst), "+r"(nl), "+r"(lmul), "+r"(ladd));
            // batches of up to 32 entries: entry r0 + lmul lane + ladd
#pragma unroll 1
            for (uint32_t r0 = 0; r0 < nl; r0 += 32 * lmul) {
                const uint32_t e = r0 + lmul * lane + ladd;
                const bool valid = e < nl;
                const int nb = __popc(__ballot_sync(0xffffffffu, valid));   // the valid lanes are 0..nb-1
                if (nb == 0) break;
                const int t = valid ? lst[e] : 0;
                const uint4 row = valid ? __ldg(crow + t) : make_uint4(0u, 0u, 0u, 0u);
                int32_t *tok = sh.u.at.tok[warp];
                char *vb = sh.u.at.vbuf[warp];
                tok[lane] = t;
                __syncwarp();
                // the first value rows are in flight while the logits are formed;
                // then each half-buffer is refilled as soon as it is consumed
                // (one copy group per half, so waiting for "all but one group"
                // always means the half about to be read)
                constexpr int kVH = VStage<DT, VQ>::kHalf, kHB = kVH * VStage<DT, VQ>::kRowBytes;
                warp_stage_v<DT, VQ>(vb, tok, 0, min(nb, kVH), vsel, lane);
                cp_async_commit();
                warp_stage_v<DT, VQ>(vb + kHB, tok, kVH, max(0, min(nb - kVH, kVH)), vsel, lane);
                cp_async_commit();
                float lg[GM];
#pragma unroll
                for (int g = 0; g < GM; ++g) lg[g] = -INFINITY;
                if (valid) {
                    const uint32_t wd[4] = {row.x, row.y, row.z, row.w};
                    float acc[GM];
#pragma unroll
                    for (int g = 0; g < GM; ++g) acc[g] = 0.f;
#pragma unroll 4
                    for (int sidx = 0; sidx < kSubspaces; ++sidx) {
                        const int j = (wd[sidx >> 3] >> (4 * (sidx & 7))) & 15;
                        const float *lp = sh.u.at.luth[sidx * kClusters + j];
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
                    for (int g = 0; g < GM; ++g) lg[g] = (g < group) ? (acc[g] + sh.qmu_h[g]) * a.scale : -INFINITY;
                }
                warp_softmax_batch(ws, lg);
#pragma unroll 1
                for (int j0 = 0, half = 0; j0 < nb; j0 += kVH, half ^= 1) {
                    char *hb = vb + half * kHB;
                    cp_async_wait_one();
                    __syncwarp();
                    warp_fma_v<DT, GM, VQ>(ws, hb, lg, j0, min(kVH, nb - j0), lane);
                    __syncwarp();              // every lane is done with this half
                    warp_stage_v<DT, VQ>(hb, tok, j0 + 2 * kVH, max(0, min(nb - j0 - 2 * kVH, kVH)), vsel, lane);
                    cp_async_commit();
                }
                __syncwarp();                  // tok and vbuf are reused by the next batch
            }
            if (!direct) __syncthreads();
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
            uint32_t cnt = __popc(flagged8(sh.bins, row, lane, kSure | kWin));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
            if (lane == 0) sh.rowcnt[row] = cnt;
        }
        __syncthreads();
        rows_to_bases(sh.rowcnt, nrows, sh.wtot);
        int32_t *io = a.idx_out + static_cast<size_t>(seg) * a.kmax;
#pragma unroll 1
        for (int row = warp; row < nrows; row += kFW) {
            const uint32_t m = flagged8(sh.bins, row, lane, kSure | kWin);
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

    // merge the warps' softmax states into this CTA's partial (m, l, o);
    // red aliases the value-staging buffers, so every warp must be done first
    __syncthreads();
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            sh.wm[warp][g] = ws.m[g];
            sh.wl[warp][g] = ws.l[g];
        }
    }
#pragma unroll
    for (int g = 0; g < GM; ++g)
        *reinterpret_cast<float4 *>(&sh.u.at.red[warp][g][lane * 4]) =
            make_float4(ws.o[g][0], ws.o[g][1], ws.o[g][2], ws.o[g][3]);
    __syncthreads();
    {
        const size_t pb = (static_cast<size_t>(seg) * a.cps + c) * GM;
        for (int e = tid; e < GM * kHeadDim; e += kFT) {
            const int g = e / kHeadDim, d = e % kHeadDim;
            float mx = -INFINITY;
#pragma unroll
            for (int w = 0; w < kFW; ++w) mx = fmaxf(mx, sh.wm[w][g]);
            float sacc = 0.f, lsum = 0.f;
            if (mx != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kFW; ++w) {
                    const float mw = sh.wm[w][g];
                    const float f = (mw == -INFINITY) ? 0.f : __expf(mw - mx);
                    sacc = fmaf(f, sh.u.at.red[w][g][d], sacc);
                    lsum = fmaf(f, sh.wl[w][g], lsum);
                }
            }
            a.part_o[(pb + g) * kHeadDim + d] = sacc;
            if (d == 0) a.part_ml[pb + g] = make_float2(mx, lsum);
        }
    }

    // ---- last CTA of the segment: merge the partials, reset the coordination state
    const int old = cta_arrive(&ctl->arrive3);
    if (tid == 0) sh.last = (old == a.cps - 1);
    __syncthreads();
    if (!sh.last) return;
    __threadfence();
    {
        // this thread's output elements e = tid + kFT i; the first kFPre
        // partials of each are fetched together with the (m, l) pairs
        constexpr int kEl = GM * kHeadDim / kFT;       // 2 or 4
        constexpr int kFPre = kEl == 2 ? 16 : 8;
        const size_t seg_p = static_cast<size_t>(seg) * a.cps;
        float pre[kEl][kFPre];
#pragma unroll
        for (int i = 0; i < kEl; ++i) {
            const int e = tid + kFT * i, g = e / kHeadDim, d = e % kHeadDim;
#pragma unroll
            for (int cc = 0; cc < kFPre; ++cc)
                pre[i][cc] = (g < group && cc < a.cps) ? __ldcg(a.part_o + ((seg_p + cc) * GM + g) * kHeadDim + d) : 0.f;
        }
        float2 *mls = reinterpret_cast<float2 *>(&sh.u.at.red[0][0][0]);       // [cps][GM]
        float *wts = reinterpret_cast<float *>(mls + kFusedMaxCps * GM);       // [cps][GM]
        for (int e = tid; e < a.cps * GM; e += kFT) mls[e] = __ldcg(a.part_ml + seg_p * GM + e);
        __syncthreads();
        if (tid < GM) {
            float mx = -INFINITY;
            for (int cc = 0; cc < a.cps; ++cc) mx = fmaxf(mx, mls[cc * GM + tid].x);
            float l = 0.f;
            for (int cc = 0; cc < a.cps; ++cc) {
                const float2 ml = mls[cc * GM + tid];
                const float f = (ml.x == -INFINITY) ? 0.f : __expf(ml.x - mx);
                wts[cc * GM + tid] = f;
                l = fmaf(ml.y, f, l);
            }
            const float inv = (l > 0.f) ? __fdividef(1.f, l) : 0.f;
            for (int cc = 0; cc < a.cps; ++cc) wts[cc * GM + tid] *= inv;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kEl; ++i) {
            const int e = tid + kFT * i, g = e / kHeadDim, d = e % kHeadDim;
            if (g >= group) continue;
            float acc = 0.f;
#pragma unroll
            for (int cc = 0; cc < kFPre; ++cc) acc = fmaf(wts[min(cc, a.cps - 1) * GM + g], pre[i][cc], acc);
#pragma unroll 4
            for (int cc = kFPre; cc < a.cps; ++cc)
                acc = fmaf(wts[cc * GM + g], __ldcg(a.part_o + ((seg_p + cc) * GM + g) * kHeadDim + d), acc);
            const size_t orow = (static_cast<size_t>(b) * a.hq + static_cast<size_t>(h) * group + g) * kHeadDim + d;
            if (DT == SIKV_DTYPE_F32)
                static_cast<float *>(a.out)[orow] = acc;
            else
                static_cast<unsigned short *>(a.out)[orow] = static_cast<unsigned short>(f32_to_bf16_bits(acc));
        }
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

template <int DT, int GM, bool VQ>
sikv_status launch_fused_t(const FusedArgs &args, const FusedPlan &plan, cudaStream_t stream) {
    auto kern = decode_fused_kernel<DT, GM, VQ>;
    const size_t smem = sizeof(FusedSmem<GM>);   // limit raised by fused_plan on this device
    FusedArgs a = args;
    void *params[] = {&a};
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(plan.grid),
                                                      dim3(kFT), params, smem, stream);
    return e == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

// Per device: the kernel's dynamic shared-memory limit is raised once, and
// its occupancy (CTAs per SM) is computed once.  Values are idempotent, so
// concurrent first calls only repeat the same work and store the same value
// (relaxed atomics: no data race).
constexpr int kMaxDevices = 64;

template <int DT, int GM, bool VQ>
int occupancy_of() {
    static std::atomic<int> cached[kMaxDevices];    // 0: unknown, else occupancy + 1
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < kMaxDevices) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c - 1;
    }
    // the occupancy calculator honours the kernel's dynamic shared-memory
    // limit, which must be raised above the 48 KB default first
    auto kern = decode_fused_kernel<DT, GM, VQ>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FusedSmem<GM>)) !=
        cudaSuccess)
        return 0;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kFT, sizeof(FusedSmem<GM>)) != cudaSuccess)
        return 0;
    if (dev >= 0 && dev < kMaxDevices) cached[dev].store(blocks + 1, std::memory_order_relaxed);
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

FusedPlan fused_plan(const sikv_params &p, bool vq) {
    FusedPlan plan;
    const int group = p.num_q_heads / p.num_kv_heads;
    const int gm = group <= 4 ? 4 : 8;
    const int segs = p.batch * p.num_kv_heads;
    const int sms = device_sm_count();
    if (sms <= 0) return plan;
    int occ = 0;
    if (p.dtype == SIKV_DTYPE_BF16)
        occ = vq ? (gm == 4 ? occupancy_of<SIKV_DTYPE_BF16, 4, true>() : occupancy_of<SIKV_DTYPE_BF16, 8, true>())
                 : (gm == 4 ? occupancy_of<SIKV_DTYPE_BF16, 4, false>() : occupancy_of<SIKV_DTYPE_BF16, 8, false>());
    else
        occ = vq ? (gm == 4 ? occupancy_of<SIKV_DTYPE_F32, 4, true>() : occupancy_of<SIKV_DTYPE_F32, 8, true>())
                 : (gm == 4 ? occupancy_of<SIKV_DTYPE_F32, 4, false>() : occupancy_of<SIKV_DTYPE_F32, 8, false>());
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

int fused_sub_batch(const sikv_params &p, bool vq) {
    // the largest number of sequences per launch whose segments fit one
    // co-resident launch (0: none does, or the whole batch already does)
    for (int bs = p.batch - 1; bs >= 1; --bs) {
        sikv_params ps = p;
        ps.batch = bs;
        if (fused_plan(ps, vq).ok) return bs;
    }
    return 0;
}

sikv_status launch_decode_fused(const sikv_params &p, const FusedPlan &plan, const FusedLayout &L, const void *q,
                                const void *K, const void *V, const uint8_t *vq, const uint8_t *codes,
                                const float *codebook, const float *mu,
                                const int32_t *seq_lens, const int32_t *k_per_seq, void *out, int32_t *idx_out,
                                float *scores_out, char *ws, int32_t *status, cudaStream_t stream) {
    FusedArgs a;
    a.q = q;
    a.K = K;
    a.V = V;
    a.vq = vq;
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
    if (vq) {
        if (p.dtype == SIKV_DTYPE_BF16)
            return plan.gm == 4 ? launch_fused_t<SIKV_DTYPE_BF16, 4, true>(a, plan, stream)
                                : launch_fused_t<SIKV_DTYPE_BF16, 8, true>(a, plan, stream);
        return plan.gm == 4 ? launch_fused_t<SIKV_DTYPE_F32, 4, true>(a, plan, stream)
                            : launch_fused_t<SIKV_DTYPE_F32, 8, true>(a, plan, stream);
    }
    if (p.dtype == SIKV_DTYPE_BF16)
        return plan.gm == 4 ? launch_fused_t<SIKV_DTYPE_BF16, 4, false>(a, plan, stream)
                            : launch_fused_t<SIKV_DTYPE_BF16, 8, false>(a, plan, stream);
    return plan.gm == 4 ? launch_fused_t<SIKV_DTYPE_F32, 4, false>(a, plan, stream)
                        : launch_fused_t<SIKV_DTYPE_F32, 8, false>(a, plan, stream);
}

}  // namespace sikv
