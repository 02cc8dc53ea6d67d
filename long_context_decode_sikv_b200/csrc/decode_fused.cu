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
// launch).  A CTA keeps the scores of its chunk in registers (NPT per thread)
// and never writes them to memory unless asked to.  The CTAs of a segment
// agree on the selection through three counters in the workspace:
//   1. every CTA builds a 2048-bin histogram of its scores (bins linear in the
//      score between the bounds the LUT implies, so a higher bin means a
//      strictly higher score), finds its own local k-th bin b_c and adds its
//      counts for bins >= b_c into the segment histogram (the global k-th bin
//      b* is >= every b_c, so the lower bins are never needed);  arrive #1;
//   2. after all arrivals every CTA scans the segment histogram from the top
//      and finds b*; tokens in higher bins are selected outright, tokens in
//      b* are written to a candidate list;  arrive #2;
//   3. every CTA radix-selects, from the candidates, the exact k-th key T and
//      the lowest-index ties it needs (the same answer in every CTA), marks its
//      selected tokens, and attends over them (plus its share of the sinks)
//      with an online softmax; it writes (m, l, o) partials;  arrive #3 — the
//      last CTA to arrive merges the partials into the output and zeroes the
//      segment's coordination state for the next launch.
// Waits are bounded: a wait that runs out sets SIKV_DEVERR_TIMEOUT and the
// CTA carries on, so a kernel always ends.
#include "score_device.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kFT = 256;                 // threads per CTA
constexpr int kFW = kFT / 32;            // warps per CTA
constexpr int kFBins = 2048;             // histogram bins per segment
constexpr int kFTile = 256;              // list entries attended per pass
constexpr int kFCandSmem = 1024;         // candidates staged in shared memory
constexpr int kFUnroll = 8;              // code rows in flight per thread
constexpr int kFListCap = 2048;          // attended tokens staged per window
constexpr int kFGroups = 64 * kFW;       // (register slot, warp) groups, NPT <= 64
constexpr int kSpinLimit = 1 << 23;      // ~1 s of __nanosleep(128) polls

struct FusedArgs {
    const void *q, *K, *V;
    const uint8_t *codes;
    const float *codebook, *mu;
    const int32_t *seq_lens, *k_per_seq;
    void *out;
    int32_t *idx_out;
    float *scores_out;
    int hq, hkv, nmax, num_sinks, kmax, cps, chunk, cand_cap;
    float scale;
    uint32_t *ghist;      // [segs][kFBins]
    uint2 *cand;          // [segs][cand_cap] (key, token)
    FusedCtl *ctl;        // [segs]
    int32_t *selcnt;      // [segs][cps]
    float *part_o;        // [segs][cps][GM][D]
    float2 *part_ml;      // [segs][cps][GM]
    int32_t *status;
};

template <int GM>
struct FusedSmem {
    union {
        ScoreTables tab;                         // scoring phase
        struct {
            int32_t list[kFListCap];             // ordered tokens to attend (one window)
            uint32_t grp[kFGroups];              // per-(slot, warp) ordinal bases
            alignas(16) float logit[GM][kFTile];
            alignas(16) float red[kFW][GM][kHeadDim];
        } at;                                    // attention phase
    } u;
    alignas(16) float qs[GM][kHeadDim];
    alignas(16) float luth[kSubspaces * kClusters][GM];   // per-head LUT, [s*16+j][g]
    alignas(16) float qmu_h[GM];
    alignas(16) float run_m[GM];
    alignas(16) float run_l[GM];
    alignas(16) float tile_stat[kFW][GM];
    uint32_t hist[kFBins];
    uint32_t ckey[kFCandSmem];
    int32_t cidx[kFCandSmem];
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

// In a histogram of `nbins` bins scanned from the top bin down, finds the bin
// where the running count first reaches `need` (1 <= need <= total).  Each
// thread owns nbins/256 consecutive bins.  Writes (bin, count above) to
// out[0..1].  Ends synchronized.
template <typename Load>
__device__ __forceinline__ void cta_find_bin(Load load, int nbins, uint32_t need, uint32_t *wtot, uint32_t *out) {
    const int per = nbins / kFT;
    const int top = nbins - 1 - threadIdx.x * per;
    uint32_t loc = 0;
    for (int i = 0; i < per; ++i) loc += load(top - i);
    uint32_t total;
    uint32_t above = cta_excl_scan(loc, wtot, &total);
    if (above < need && need <= above + loc) {
        for (int i = 0; i < per; ++i) {
            const uint32_t h = load(top - i);
            if (above + h >= need) {
                out[0] = static_cast<uint32_t>(top - i);
                out[1] = above;
                break;
            }
            above += h;
        }
    }
    __syncthreads();
}

// Radix select over `n` elements (element e has key key(e) and passes
// keep(e)): returns the key of rank `need` counted from the largest and, in
// *need_left, how many elements equal to it are still needed.  Uses hist[0..255].
template <typename KeyF, typename KeepF>
__device__ __forceinline__ uint32_t cta_radix_select(KeyF key, KeepF keep, int n, uint32_t need, uint32_t *hist,
                                                     uint32_t *wtot, uint32_t *sc, uint32_t *need_left) {
    uint32_t prefix = 0, mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kFT) hist[i] = 0;
        __syncthreads();
        for (int e = threadIdx.x; e < n; e += kFT) {
            if (!keep(e)) continue;
            const uint32_t k = key(e);
            if (((k ^ prefix) & mask) == 0) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        cta_find_bin([&](int i) { return hist[i]; }, 256, need, wtot, sc);
        prefix |= sc[0] << shift;
        mask |= 255u << shift;
        need -= sc[1];
        __syncthreads();
    }
    *need_left = need;
    return prefix;
}

// Exact score of token t, recomputed by the lane that scored it (same table,
// same rotation, same order of additions: bit-identical).  Only tokens in the
// threshold bin need it, so it stays out of line.
__device__ __noinline__ float rescore(const float *t2, const uint4 *crow, int t, int lane, float qmu) {
    return lut2_score(t2, __ldg(crow + t), lane, qmu);
}

template <int DT, int GM, int NPT>
__global__ void __launch_bounds__(kFT, 2) decode_fused_kernel(FusedArgs a) {
    constexpr int EB = ElemBytes<DT>::value;
    extern __shared__ __align__(16) unsigned char fused_smem[];
    FusedSmem<GM> &sh = *reinterpret_cast<FusedSmem<GM> *>(fused_smem);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seg = blockIdx.x / a.cps, c = blockIdx.x % a.cps;
    const int b = seg / a.hkv, h = seg % a.hkv, group = a.hq / a.hkv;
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

    // ---- tables: byte-indexed scoring tables, per-head LUTs, bounds
    build_score_tables<DT>(sh.u.tab, a.q, a.codebook, a.mu, b, h, a.hq, group, seg);
    {
        const char *qrow = static_cast<const char *>(a.q) +
                           (static_cast<size_t>(b) * a.hq + static_cast<size_t>(h) * group) * kHeadDim * EB;
        for (int e = tid; e < GM * kHeadDim; e += kFT) {
            const int g = e / kHeadDim, d = e % kHeadDim;
            sh.qs[g][d] = g < group ? load1<DT>(qrow + static_cast<size_t>(g) * kHeadDim * EB, d) : 0.f;
        }
        for (int i = tid; i < kFBins; i += kFT) sh.hist[i] = 0;
    }
    __syncthreads();
    {
        const float4 *cb = reinterpret_cast<const float4 *>(a.codebook) + static_cast<size_t>(seg) * kSubspaces * kClusters;
        for (int e = tid; e < kSubspaces * kClusters * GM; e += kFT) {
            const int r = e / GM, g = e % GM, s = r >> 4;
            const float4 c4 = __ldg(cb + r);
            float v = sh.qs[g][4 * s] * c4.x;
            v = fmaf(sh.qs[g][4 * s + 1], c4.y, v);
            v = fmaf(sh.qs[g][4 * s + 2], c4.z, v);
            v = fmaf(sh.qs[g][4 * s + 3], c4.w, v);
            sh.luth[r][g] = v;
        }
        const float4 m4 = __ldg(reinterpret_cast<const float4 *>(a.mu + static_cast<size_t>(seg) * kHeadDim) + lane);
        for (int g = warp; g < GM; g += kFW) {
            double s = static_cast<double>(sh.qs[g][4 * lane]) * m4.x;
            s = fma(static_cast<double>(sh.qs[g][4 * lane + 1]), static_cast<double>(m4.y), s);
            s = fma(static_cast<double>(sh.qs[g][4 * lane + 2]), static_cast<double>(m4.z), s);
            s = fma(static_cast<double>(sh.qs[g][4 * lane + 3]), static_cast<double>(m4.w), s);
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
    }
    __syncthreads();
    const float bin_lo = sh.bin_lo, bin_inv = sh.bin_inv;
    const bool bin_flat = sh.bin_flat != 0;
    auto bin_of = [&](float s) -> int {
        if (bin_flat) return 0;
        const int v = __float2int_rz((s - bin_lo) * bin_inv);
        return min(max(v, 0), kFBins - 1);
    };

    // ---- scores of this chunk; each thread keeps only the histogram bin of
    // its tokens (16 bits each, bin + 1, 0 = no token), two per register.
    // Register slot i of (warp w, lane l) is token t0 + 256 i + 32 w + l.
    constexpr int NPK = NPT / 2;
    uint32_t binpk[NPK];
    const float qmu = sh.u.tab.qmu;
    const uint4 *crow = reinterpret_cast<const uint4 *>(a.codes) + static_cast<size_t>(seg) * a.nmax;
    const int tstart = max(t0, a.num_sinks);
    {
        float *so = a.scores_out ? a.scores_out + static_cast<size_t>(seg) * a.nmax : nullptr;
#pragma unroll
        for (int i = 0; i < NPK; ++i) binpk[i] = 0;
#pragma unroll
        for (int i0 = 0; i0 < NPT; i0 += kFUnroll) {
            uint4 rows[kFUnroll];
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u) {
                const int t = t0 + kFT * (i0 + u) + 32 * warp + lane;
                rows[u] = (t >= tstart && t < t1) ? __ldcs(crow + t) : make_uint4(0, 0, 0, 0);
            }
            // keep the next batch's loads below this point: kFUnroll rows in
            // flight per thread, not the whole unrolled chunk
            asm volatile("" ::: "memory");
#pragma unroll
            for (int u = 0; u < kFUnroll; ++u) {
                const int i = i0 + u;
                const int t = t0 + kFT * i + 32 * warp + lane;
                if (t >= tstart && t < t1) {
                    const float sv = lut2_score(sh.u.tab.t2, rows[u], lane, qmu);
                    const int bi = bin_of(sv);
                    atomicAdd(&sh.hist[bi], 1u);
                    binpk[i >> 1] |= static_cast<uint32_t>(bi + 1) << (16 * (i & 1));
                    if (so) so[t] = sv;
                } else if (so && t < t1) {
                    so[t] = -INFINITY;
                }
            }
        }
    }
    auto bin_at = [&](int i) -> int { return static_cast<int>((binpk[i >> 1] >> (16 * (i & 1))) & 0xFFFFu) - 1; };
    // exact score of register slot i (recomputed: same lane, same table, same bits)
    auto score_at = [&](int i) -> float {
        return rescore(sh.u.tab.t2, crow, t0 + kFT * i + 32 * warp + lane, lane, qmu);
    };
    __syncthreads();

    // ---- 1. local k-th bin, publish the bins at or above it
    {
        uint32_t total;
        {
            uint32_t loc = 0;
            for (int i = tid; i < kFBins; i += kFT) loc += sh.hist[i];
            cta_excl_scan(loc, sh.wtot, &total);
        }
        int bc = 0;
        if (k > 0 && total >= static_cast<uint32_t>(k)) {
            cta_find_bin([&](int i) { return sh.hist[i]; }, kFBins, static_cast<uint32_t>(k), sh.wtot, sh.sc);
            bc = static_cast<int>(sh.sc[0]);
        }
        if (k > 0) {
            uint32_t *gh = a.ghist + static_cast<size_t>(seg) * kFBins;
            for (int i = bc + tid; i < kFBins; i += kFT) {
                const uint32_t v = sh.hist[i];
                if (v) atomicAdd(gh + i, v);
            }
        }
    }
    cta_arrive(&ctl->arrive1);
    cta_wait(&ctl->arrive1, a.cps, a.status);

    // ---- 2. global k-th bin b*; select higher bins, list the tokens of b*
    int bstar = kFBins;              // nothing selected when k == 0
    uint32_t above_bstar = 0;
    if (k > 0) {
        const uint32_t *gh = a.ghist + static_cast<size_t>(seg) * kFBins;
        cta_find_bin([&](int i) { return __ldcg(gh + i); }, kFBins, static_cast<uint32_t>(k), sh.wtot, sh.sc);
        bstar = static_cast<int>(sh.sc[0]);
        above_bstar = sh.sc[1];
    }
    {
        uint32_t mine = 0;
        uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
#pragma unroll
        for (int i = 0; i < NPT; ++i) {
            const int t = t0 + kFT * i + 32 * warp + lane;
            const int bi = bin_at(i);
            if (bi < 0 || k == 0) continue;
            if (bi > bstar) {
                ++mine;
            } else if (bi == bstar) {
                const int slot = atomicAdd(&ctl->ncand, 1);
                if (slot < a.cand_cap) cand[slot] = make_uint2(score_key(score_at(i)), static_cast<uint32_t>(t));
            }
        }
        uint32_t tot;
        cta_excl_scan(mine, sh.wtot, &tot);
        if (tid == 0) a.selcnt[static_cast<size_t>(seg) * a.cps + c] = static_cast<int32_t>(tot);
    }
    cta_arrive(&ctl->arrive2);
    cta_wait(&ctl->arrive2, a.cps, a.status);

    // ---- 3. exact threshold among the candidates (same result in every CTA)
    uint32_t T = 0xFFFFFFFFu, tie_idx = 0;
    bool have_ties = false;
    if (k > 0) {
        const int ncand = min(__ldcg(&ctl->ncand), a.cand_cap);
        const uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
        const bool staged = ncand <= kFCandSmem;
        if (staged) {
            for (int e = tid; e < ncand; e += kFT) {
                const uint2 v = __ldcg(cand + e);
                sh.ckey[e] = v.x;
                sh.cidx[e] = static_cast<int32_t>(v.y);
            }
            __syncthreads();
        }
        auto ckey = [&](int e) -> uint32_t { return staged ? sh.ckey[e] : __ldcg(cand + e).x; };
        auto cidx = [&](int e) -> uint32_t {
            return staged ? static_cast<uint32_t>(sh.cidx[e]) : __ldcg(cand + e).y;
        };
        const uint32_t need = static_cast<uint32_t>(k) - above_bstar;   // >= 1
        uint32_t ties_needed;
        T = cta_radix_select(ckey, [&](int) { return true; }, ncand, need, sh.hist, sh.wtot, sh.sc, &ties_needed);
        // the ties_needed lowest token indices among keys equal to T
        uint32_t left;
        const uint32_t inv_idx = cta_radix_select([&](int e) { return ~cidx(e); },
                                                  [&](int e) { return ckey(e) == T; }, ncand, ties_needed,
                                                  sh.hist, sh.wtot, sh.sc, &left);
        tie_idx = ~inv_idx;          // ties with token index <= tie_idx are selected
        have_ties = true;
    }

    // ---- selection bits in registers (the exact keys of threshold-bin
    // tokens are recomputed, so the scoring tables must still be intact)
    uint32_t selmask = 0, selmask_hi = 0;      // bit i: register slot i selected
    {
#pragma unroll
        for (int i = 0; i < NPT; ++i) {
            const int bi = bin_at(i);
            bool sel = false;
            if (bi >= 0 && k > 0) {
                if (bi > bstar) {
                    sel = true;
                } else if (bi == bstar) {
                    const uint32_t key = score_key(score_at(i));
                    const uint32_t t = static_cast<uint32_t>(t0 + kFT * i + 32 * warp + lane);
                    sel = key > T || (have_ties && key == T && t <= tie_idx);
                }
            }
            if (sel) {
                if (i < 32) selmask |= 1u << i;
                else selmask_hi |= 1u << (i - 32);
            }
        }
    }
    auto sel_bit = [&](int i) -> bool { return i < 32 ? ((selmask >> i) & 1u) : ((selmask_hi >> (i - 32)) & 1u); };
    __syncthreads();                           // scoring tables dead from here on

    // ---- ordinals in ascending token order: group (i, w) holds tokens
    // t0 + 256 i + 32 w + [0, 32), ordered by i then w
    uint32_t *grp = sh.u.at.grp;
#pragma unroll
    for (int i = 0; i < NPT; ++i) {
        const uint32_t bal = __ballot_sync(0xffffffffu, sel_bit(i));
        if (lane == 0) grp[i * kFW + warp] = __popc(bal);
    }
    __syncthreads();
    uint32_t n_sel;
    {
        constexpr int per = (NPT * kFW + kFT - 1) / kFT;
        uint32_t v[per > 0 ? per : 1];
        uint32_t loc = 0;
#pragma unroll
        for (int j = 0; j < per; ++j) {
            const int gi = tid * per + j;
            v[j] = gi < NPT * kFW ? grp[gi] : 0u;
            loc += v[j];
        }
        uint32_t run = cta_excl_scan(loc, sh.wtot, &n_sel);
#pragma unroll
        for (int j = 0; j < per; ++j) {
            const int gi = tid * per + j;
            if (gi < NPT * kFW) grp[gi] = run;
            run += v[j];
        }
        __syncthreads();
    }

    // offset of this chunk's selection in idx_out: the selected tokens of the
    // earlier chunks (their higher-bin counts plus their winning candidates)
    uint32_t out_base = 0;
    if (a.idx_out && k > 0) {
        uint32_t before = 0;
        for (int cc = tid; cc < c; cc += kFT)
            before += static_cast<uint32_t>(__ldcg(a.selcnt + static_cast<size_t>(seg) * a.cps + cc));
        const int ncand = min(__ldcg(&ctl->ncand), a.cand_cap);
        const uint2 *cand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
        for (int e = tid; e < ncand; e += kFT) {
            const uint2 v = __ldcg(cand + e);
            const bool win = v.x > T || (have_ties && v.x == T && v.y <= tie_idx);
            if (win && static_cast<int>(v.y) < t0) ++before;
        }
        cta_excl_scan(before, sh.wtot, &out_base);
    }

    // ---- attention over this CTA's selected tokens and its share of the sinks
    const int n_sinks = min(a.num_sinks, n_tok);
    const int my_sinks = (n_sinks > c) ? (n_sinks - c + a.cps - 1) / a.cps : 0;   // sinks t = c (mod cps)
    const uint32_t n_list = n_sel + static_cast<uint32_t>(my_sinks);
    const size_t kv_seg = static_cast<size_t>(seg) * a.nmax;
    if (tid < GM) {
        sh.run_m[tid] = -INFINITY;
        sh.run_l[tid] = 0.f;
    }
    float o[GM][4];
#pragma unroll
    for (int g = 0; g < GM; ++g) o[g][0] = o[g][1] = o[g][2] = o[g][3] = 0.f;
    int32_t *io = a.idx_out ? a.idx_out + static_cast<size_t>(seg) * a.kmax : nullptr;
    for (uint32_t wbase = 0; wbase < n_list; wbase += kFListCap) {
        // stage the window [wbase, wbase + kFListCap) of the ordered list
        asm volatile("" ::: "memory");
        const uint32_t wn = min(static_cast<uint32_t>(kFListCap), n_list - wbase);
#pragma unroll
        for (int i = 0; i < NPT; ++i) {
            const uint32_t bal = __ballot_sync(0xffffffffu, sel_bit(i));
            if (sel_bit(i)) {
                const uint32_t ord = grp[i * kFW + warp] + __popc(bal & ((1u << lane) - 1u));
                const int t = t0 + kFT * i + 32 * warp + lane;
                if (ord >= wbase && ord < wbase + kFListCap) sh.u.at.list[ord - wbase] = t;
                if (io && wbase == 0 && out_base + ord < static_cast<uint32_t>(k)) io[out_base + ord] = t;
            }
        }
        for (uint32_t e = tid; e < wn; e += kFT) {
            const uint32_t ord = wbase + e;
            if (ord >= n_sel) sh.u.at.list[e] = -1 - static_cast<int32_t>(c + (ord - n_sel) * a.cps);   // a sink
        }
        __syncthreads();
        for (uint32_t tbase = 0; tbase < wn; tbase += kFTile) {
            const uint32_t tile_n = min(static_cast<uint32_t>(kFTile), wn - tbase);
            // logits, one list entry per thread
            {
                float lg[GM];
#pragma unroll
                for (int g = 0; g < GM; ++g) lg[g] = -INFINITY;
                if (static_cast<uint32_t>(tid) < tile_n) {
                    const int32_t ent = sh.u.at.list[tbase + tid];
                    if (ent >= 0) {
                        const uint4 row = __ldg(reinterpret_cast<const uint4 *>(a.codes) + kv_seg + ent);
                        const uint32_t w[4] = {row.x, row.y, row.z, row.w};
                        float acc[GM];
#pragma unroll
                        for (int g = 0; g < GM; ++g) acc[g] = 0.f;
#pragma unroll
                        for (int s = 0; s < kSubspaces; ++s) {
                            const int j = (w[s >> 3] >> (4 * (s & 7))) & 15;
                            const float *lp = sh.luth[s * kClusters + j];
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
                        const int t = -1 - ent;
                        const char *krow = static_cast<const char *>(a.K) + (kv_seg + t) * kHeadDim * EB;
                        float acc[GM];
#pragma unroll
                        for (int g = 0; g < GM; ++g) acc[g] = 0.f;
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
                alpha[g] = (sh.run_m[g] == -INFINITY) ? 0.f : expf(sh.run_m[g] - mx);
            }
            __syncthreads();
#pragma unroll
            for (int g = 0; g < GM; ++g) {
                const float lv = sh.u.at.logit[g][tid];
                const float pr = (lv == -INFINITY) ? 0.f : expf(lv - mnew[g]);
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
            for (uint32_t e = warp; e < tile_n; e += kFW) {
                const int32_t ent = sh.u.at.list[tbase + e];
                const int t = ent >= 0 ? ent : -1 - ent;
                const float4 v = load4<DT>(static_cast<const char *>(a.V) + (kv_seg + t) * kHeadDim * EB, lane * 4);
#pragma unroll
                for (int g = 0; g < GM; ++g) {
                    const float pr = sh.u.at.logit[g][e];
                    o[g][0] = fmaf(pr, v.x, o[g][0]);
                    o[g][1] = fmaf(pr, v.y, o[g][1]);
                    o[g][2] = fmaf(pr, v.z, o[g][2]);
                    o[g][3] = fmaf(pr, v.w, o[g][3]);
                }
            }
            __syncthreads();
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
                const float wgt = (ml.x == -INFINITY) ? 0.f : expf(ml.x - mx);
                l = fmaf(ml.y, wgt, l);
                acc = fmaf(__ldcg(a.part_o + pb * kHeadDim + d), wgt, acc);
            }
        }
        const float r = (l > 0.f) ? acc / l : 0.f;
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

template <int DT, int GM, int NPT>
sikv_status launch_fused_t(const sikv_params &p, const FusedArgs &args, const FusedPlan &plan, cudaStream_t stream) {
    auto kern = decode_fused_kernel<DT, GM, NPT>;
    const size_t smem = sizeof(FusedSmem<GM>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SIKV_ERR_CUDA;
    FusedArgs a = args;
    void *params[] = {&a};
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(plan.grid),
                                                      dim3(kFT), params, smem, stream);
    (void)p;
    return e == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

template <int DT, int GM>
sikv_status dispatch_npt(const sikv_params &p, const FusedArgs &args, const FusedPlan &plan, cudaStream_t stream) {
    switch (plan.npt) {
        case 8: return launch_fused_t<DT, GM, 8>(p, args, plan, stream);
        case 16: return launch_fused_t<DT, GM, 16>(p, args, plan, stream);
        case 32: return launch_fused_t<DT, GM, 32>(p, args, plan, stream);
        case 64: return launch_fused_t<DT, GM, 64>(p, args, plan, stream);
        default: return SIKV_ERR_UNSUPPORTED;
    }
}

template <int DT, int GM, int NPT>
int occupancy_of() {
    // the occupancy calculator honours the kernel's dynamic shared-memory
    // limit, which must be raised above the 48 KB default first
    auto kern = decode_fused_kernel<DT, GM, NPT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FusedSmem<GM>)) !=
        cudaSuccess)
        return 0;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kFT, sizeof(FusedSmem<GM>)) != cudaSuccess)
        return 0;
    return blocks;
}

template <int DT, int GM>
int occupancy_npt(int npt) {
    switch (npt) {
        case 8: return occupancy_of<DT, GM, 8>();
        case 16: return occupancy_of<DT, GM, 16>();
        case 32: return occupancy_of<DT, GM, 32>();
        case 64: return occupancy_of<DT, GM, 64>();
        default: return 0;
    }
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
    // two CTAs per SM is the design point; confirm with the occupancy calculator
    const int per_sm_guess = 2;
    int cps = (sms * per_sm_guess) / segs;
    const int min_chunk = 2048;
    cps = std::min(cps, (p.max_seq_len + min_chunk - 1) / min_chunk);
    cps = std::min(cps, kFusedMaxCps);
    if (cps < 1) return plan;                     // more segments than co-resident CTAs
    int chunk = (p.max_seq_len + cps - 1) / cps;
    chunk = (chunk + kFT - 1) / kFT * kFT;
    cps = (p.max_seq_len + chunk - 1) / chunk;
    const int npt_need = chunk / kFT;
    int npt = 8;
    while (npt < npt_need) npt *= 2;
    if (npt > 64) return plan;
    int occ = 0;
    if (p.dtype == SIKV_DTYPE_BF16)
        occ = gm == 4 ? occupancy_npt<SIKV_DTYPE_BF16, 4>(npt) : occupancy_npt<SIKV_DTYPE_BF16, 8>(npt);
    else
        occ = gm == 4 ? occupancy_npt<SIKV_DTYPE_F32, 4>(npt) : occupancy_npt<SIKV_DTYPE_F32, 8>(npt);
    if (occ < 1 || static_cast<long long>(segs) * cps > static_cast<long long>(occ) * sms) return plan;
    plan.ok = true;
    plan.cps = cps;
    plan.chunk = chunk;
    plan.npt = npt;
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
        return plan.gm == 4 ? dispatch_npt<SIKV_DTYPE_BF16, 4>(p, a, plan, stream)
                            : dispatch_npt<SIKV_DTYPE_BF16, 8>(p, a, plan, stream);
    return plan.gm == 4 ? dispatch_npt<SIKV_DTYPE_F32, 4>(p, a, plan, stream)
                        : dispatch_npt<SIKV_DTYPE_F32, 8>(p, a, plan, stream);
}

}  // namespace sikv
