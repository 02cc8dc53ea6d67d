// sikv_decode, single-launch form on thread-block clusters: scoring, exact
// top-k and fused sparse attention of a whole decode step, with the CTAs of
// each (sequence, KV head) segment forming one cluster.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 items 2-4: LUT-GEMV scores in the compressed domain,
// top-k on them, dequantization fused with sparse attention over the 64 sink
// tokens plus the selected tokens.
//
// Work split.  A segment is cut into C chunks (C = the cluster size, 1..16)
// of at most 32768 tokens, one CTA of 512 threads per chunk and one CTA per
// SM (the shared memory holds a whole chunk's bins and a batch of value rows
// for every warp).  The per-CTA work is the cooperative kernel's
// (decode_fused.cu): build the byte table, score the chunk's code rows into
// per-token bins and a local histogram, find the segment's threshold bin b*,
// select the tokens above it outright and re-rank the tokens in it on exact
// keys, attend (each pass's list split evenly over the warps, each batch's
// value rows requested at once).  The CTAs of a cluster agree through distributed shared
// memory and hardware cluster barriers instead of global-memory counters:
//   #1  (prologue)  the leader (rank 0) has zeroed its segment histogram;
//   #2  every CTA has added its counts of the bins at or above its own k-th
//       bin into the leader's histogram (remote atomic adds);  every CTA then
//       reads the leader's histogram and finds b*;
//   #3  every CTA has listed its tokens of bin b* with their exact keys in its
//       own shared memory (or, past a cap, in its region of the workspace);
//       every CTA reads all of them and ranks them (key descending, token
//       ascending) -- the same answer in every CTA -- while the sinks and the
//       tokens above b* have already been attended between arrive and wait;
//   #4  every CTA's (m, l, o) partial is in its shared memory; each CTA merges
//       its slice of the segment's output elements over all partials;
//   #5  nobody leaves while another CTA still reads its shared memory.
// Every CTA executes the same five arrive/wait pairs unconditionally, and a
// cluster's CTAs are co-scheduled by the hardware, so no wait depends on a CTA
// that has not started.  Nothing is left in the workspace between launches,
// and launches are independent of how many clusters fit on the device at
// once: extra clusters simply run in later waves.
#include <atomic>

#include "cluster_common.cuh"
#include "decode_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kMaxCluster = 16;          // CTAs per cluster (above 8: non-portable size)
constexpr int kCT = 512;                 // threads per CTA: one CTA per SM
constexpr int kCW = kCT / 32;            // warps per CTA
constexpr int kCMaxNpt = 64;             // token slots per thread at most
constexpr int kCMaxChunk = kCMaxNpt * kCT;                // tokens per CTA at most
constexpr int kCPend = 256;              // threshold-bin tokens a CTA keeps in shared memory
constexpr int kCHist = 2048;             // words of hist (the histogram's 1024 bins, then the lists)
constexpr int kCWarpList = (kCHist - 2 * kCPend) / kCW;   // tokens of each warp's direct list
constexpr int kCList = 2048;             // tokens of a pass list (in mhist)
constexpr int kCSmemBudget = 232448;     // 227 KB: the most one CTA may use

struct ClusterArgs {
    const void *q, *K, *V;
    const uint8_t *vq;    // 2-bit value rows of the selected tokens (VQ kernels only)
    const uint8_t *codes;
    const float *codebook, *mu;
    const int32_t *seq_lens, *k_per_seq;
    void *out;
    int32_t *idx_out;
    float *scores_out;
    int hq, hkv, nmax, num_sinks, kmax, csize, chunk, npt, cand_cap;
    float scale;
    uint2 *cand;          // [segs][cand_cap]: CTA r's overflow candidates from r * chunk on
    int32_t *status;
};

// Bytes of the attention extension `ax` (below): what the budget leaves.
template <int GM>
struct AxBytes {
    static constexpr int value = GM == 4 ? 73728 : 66560;
};

// Shared memory.  The union is reused in time: scoring tables, candidate
// ranking buffers, the warps' outputs at the end; during the attention passes
// the union and the extension `ax` hold the staged value rows, the per-head
// LUTs and the batch tokens (ClusterAttnLayout).
template <int GM>
struct ClusterSmem {
    union {
        ScoreTables tab;
        struct {
            // candidate (key, token) as one 64-bit value: key above the
            // inverted token, so a larger value ranks first (ties: lower token)
            unsigned long long ck[kFRankMax];
            uint32_t winbits[kCMaxChunk / 32];
        } sel;
        // the warps' outputs at the end; red[0] then holds the CTA's partial
        // o, read by the other CTAs of the cluster
        alignas(16) float red[kCW][GM][kHeadDim];
    } u;
    alignas(16) char ax[AxBytes<GM>::value];
    alignas(16) float qs[GM][kHeadDim];
    alignas(16) float mus[kHeadDim];
    alignas(16) float qmu_h[GM];
    alignas(16) float wm[kCW][GM];            // per-warp softmax state at the end
    alignas(16) float wl[kCW][GM];
    // the scoring histogram (kFBins words); from phase 2 on the threshold-bin
    // tokens (offsets in [0, kCPend), their keys in [kCPend, 2 kCPend), both
    // read by the other CTAs between barriers #3 and #4) and the warps'
    // direct lists of attended tokens in [2 kCPend, kCHist)
    uint32_t hist[kCHist];
    // leader: the segment histogram (kFBins words).  Every CTA: from phase 2
    // on the list a pass attends, the radix scratch of the tie-heavy refine,
    // after #4 the merge weights.
    uint32_t mhist[kCList];
    // one entry per token of the chunk, in token order (entry p: token t0 + p,
    // scored by thread p mod kCT): its bin + 1 (0: no token) in bits 0-13,
    // bit 15 set once the token is above the segment's threshold bin, bit 14
    // once it wins in the threshold bin.  Holds the codebook before scoring.
    alignas(16) uint16_t bins[kCMaxChunk];
    uint32_t rowcnt[kCMaxChunk / 256];        // selected tokens per row of 256, then their prefix
    uint32_t wtot[kCW + 1];
    uint32_t wcnt[kCW];                       // tokens in each warp's direct list
    uint32_t wpre[kCW + 1];                   // their prefix: where each starts in the pass's list
    uint32_t sc[16];
    // published to the cluster (read after barrier #3): candidates held, 1 if
    // they are in the workspace instead of pend, tokens selected above b*
    uint32_t pub[4];
    uint32_t bsd[2];                          // (b*, count above b*), written by the leader
    // gathered from the cluster after barrier #3: candidate prefix, overflow
    // flags, selected-above-b* counts of every CTA
    uint32_t cbase[kMaxCluster + 1], cover[kMaxCluster], cnsure[kMaxCluster];
    uint32_t rbase[kMaxCluster];              // cluster addresses of every CTA's partial o
    alignas(8) float2 pml[GM];                // this CTA's partial (m, l) per head
    float bin_lo, bin_inv;
    int bin_flat, pad;
};

static_assert(sizeof(ClusterSmem<4>) <= kCSmemBudget && sizeof(ClusterSmem<8>) <= kCSmemBudget,
              "one CTA per SM: 227 KB at most");

// The attention passes' layout.  A batch stages all its value rows at once
// (one round trip), kRows per warp (at most 32, one per lane): warp w's rows
// sit in the union (the byte table is dead by then) when they fit its first
// 64 KB, else in `ax`, followed by the per-head LUTs (q_h[4s:4s+4] . c[s][j],
// stored [s*16+j][g]); each warp's batch tokens sit in the union past 64 KB.
template <int DT, int GM, bool VQ>
struct ClusterAttnLayout {
    static constexpr int kRowBytes = VQ ? kVqRowBytes : kHeadDim * ElemBytes<DT>::value;
    static constexpr int kLuthBytes = kSubspaces * kClusters * GM * 4;
    static constexpr int kUnion = kT2Words * 4;                  // the union's first 64 KB
    static constexpr int fits(int rows) {
        return (kCW - kUnion / (rows * kRowBytes) > 0 ? kCW - kUnion / (rows * kRowBytes) : 0) * rows * kRowBytes +
                   kLuthBytes <= AxBytes<GM>::value;
    }
    static constexpr int pick(int rows) { return rows <= 1 || fits(rows) ? rows : pick(rows - 1); }
    static constexpr int kRows = pick(32);                               // rows per warp batch
    static constexpr int kInUnion = kUnion / (kRows * kRowBytes) < kCW ? kUnion / (kRows * kRowBytes) : kCW;
    static constexpr int kLuth = (kCW - kInUnion) * kRows * kRowBytes;  // offset of the LUTs in ax
    static constexpr int kTok = kUnion;                                 // offset of the batch tokens in the union
    static_assert(kRows >= 8, "a batch of at least 8 rows");
    static_assert(kLuth + kLuthBytes <= AxBytes<GM>::value, "staged rows and LUTs fit ax");
    static_assert(kTok + kCW * 32 * 4 <= static_cast<int>(sizeof(ScoreTables)), "batch tokens past the table");
};

// The threshold-bin candidates of a whole cluster, indexed 0..n-1 in rank
// order of their CTAs: candidate e belongs to CTA r with cbase[r] <= e <
// cbase[r + 1] and is (key, token) from that CTA's shared list (offsets at
// pend[j], keys at pend[kCPend + j]) or, when cover[r] is set, from its
// region of the workspace list.
struct ClusterCands {
    const uint32_t *cbase, *cover;
    uint32_t pend_local;     // shared-window address of this CTA's pend list
    int csize, chunk;
    const uint2 *gcand;      // the segment's workspace list
    __device__ __forceinline__ uint2 operator()(int e) const {
        int r = 0;
        while (r + 1 < csize && static_cast<int>(cbase[r + 1]) <= e) ++r;
        const int j = e - static_cast<int>(cbase[r]);
        if (cover[r]) return __ldcg(gcand + static_cast<size_t>(r) * chunk + j);
        // the same offset in CTA r's window: mapa of one rank per call
        uint32_t pb;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(pb) : "r"(pend_local), "r"(static_cast<uint32_t>(r)));
        const uint32_t p = dsmem_ld_u32(pb + 4u * static_cast<uint32_t>(j));
        const uint32_t key = dsmem_ld_u32(pb + 4u * static_cast<uint32_t>(kCPend + j));
        return make_uint2(key, static_cast<uint32_t>(r * chunk) + p);
    }
};

template <int DT, int GM, bool VQ>
__global__ void __launch_bounds__(kCT, 1) decode_cluster_kernel(ClusterArgs a) {
    constexpr int EB = ElemBytes<DT>::value;
    using AL = ClusterAttnLayout<DT, GM, VQ>;
    extern __shared__ __align__(16) unsigned char cluster_smem[];
    ClusterSmem<GM> &sh = *reinterpret_cast<ClusterSmem<GM> *>(cluster_smem);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = a.csize;
    const int c = static_cast<int>(cluster_ctarank());
    const int seg = blockIdx.x / C;
    const int b = seg / a.hkv, h = seg % a.hkv, group = a.hq / a.hkv;
    const int npt = a.npt;

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
    const char *vseg = static_cast<const char *>(a.V) + kv_seg * kHeadDim * EB;
    // value rows of the selected tokens: V itself, or its 2-bit rows (sinks
    // always read V)
    const char *vsel = VQ ? reinterpret_cast<const char *>(a.vq) + kv_seg * kVqRowBytes : vseg;

    // ---- tables.  Their inputs are requested first; while they travel, the
    // first code rows and this CTA's share of the sink rows go to L2.
    TableInputs<DT, kCT> tin;
    tin.load(a.q, a.codebook, a.mu, b, h, a.hq, group, seg);
#pragma unroll 1
    for (int i = 0; i < kFPrefetchRows && i < npt; ++i) {
        const int t = t0 + kCT * i + my;
        if (t >= tstart && t < t1) prefetch_l2(crow + t);
    }
    {
        const int n_sinks0 = min(a.num_sinks, n_tok);
        for (int sk = c + C * tid; sk < n_sinks0; sk += C * kCT) {
            prefetch_l2(static_cast<const char *>(a.K) + (kv_seg + sk) * kHeadDim * EB);
            prefetch_l2(static_cast<const char *>(a.V) + (kv_seg + sk) * kHeadDim * EB);
        }
    }
    float4 *cbs = reinterpret_cast<float4 *>(sh.bins);     // 8 KB, free until scoring
    for (int e = tid; e < GM * kHeadDim; e += kCT) sh.qs[e / kHeadDim][e % kHeadDim] = 0.f;
    for (int i = tid; i < kFBins; i += kCT) {
        sh.hist[i] = 0;
        sh.mhist[i] = 0;
    }
    if (tid < 4) sh.pub[tid] = 0;
    cluster_arrive_cta();                                    // #1: the leader's histogram is zero
    tin.store(&sh.qs[0][0], cbs, sh.mus, group);
    __syncthreads();
    build_score_tables<kCT>(sh.u.tab, &sh.qs[0][0], cbs, sh.mus, group);
    for (int g = warp; g < GM; g += kCW) {
        double s = static_cast<double>(sh.qs[g][4 * lane]) * sh.mus[4 * lane];
        s = fma(static_cast<double>(sh.qs[g][4 * lane + 1]), static_cast<double>(sh.mus[4 * lane + 1]), s);
        s = fma(static_cast<double>(sh.qs[g][4 * lane + 2]), static_cast<double>(sh.mus[4 * lane + 2]), s);
        s = fma(static_cast<double>(sh.qs[g][4 * lane + 3]), static_cast<double>(sh.mus[4 * lane + 3]), s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) sh.qmu_h[g] = static_cast<float>(s);
    }
    if (warp == kCW - 1) {
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
                if (i0 + u < npt) r[u] = __ldcs(crow + min(t0 + kCT * (i0 + u) + my, tmax));
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
                const int t = t0 + kCT * i + my;
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
                sh.bins[i * kCT + tid] = static_cast<uint16_t>(e);
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

    // ---- 1. local k-th bin; the counts at or above it go into the leader's
    // histogram (the segment's k-th bin b* is >= every CTA's local one)
    cluster_wait();                                          // #1
    const uint32_t mh_leader = dsmem_map(&sh.mhist[0], 0);
    if (k > 0) {
        if (tid == 0) {
            sh.sc[0] = 0;
            sh.sc[1] = 0;
            sh.sc[8] = 0;     // threshold-bin tokens listed
        }
        __syncthreads();
        cta_find_bin<kFBins / kCT, kCT>([&](int i) { return sh.hist[i]; }, static_cast<uint32_t>(k), sh.wtot, sh.sc);
        const int bc = static_cast<int>(sh.sc[0]);    // 0 when the chunk holds fewer than k tokens
        for (int i = bc + tid; i < kFBins; i += kCT) {
            const uint32_t v = sh.hist[i];
            if (v) dsmem_red_add(mh_leader + 4u * static_cast<uint32_t>(i), v);
        }
    }
    cluster_arrive_cta();                                    // #2
    // this thread's codebook rows for the per-head LUTs, fetched during the wait
    constexpr int kCbPer = kSubspaces * kClusters / kCT;
    float4 cbr[kCbPer];
    {
        const float4 *cb = reinterpret_cast<const float4 *>(a.codebook) + static_cast<size_t>(seg) * kSubspaces * kClusters;
#pragma unroll
        for (int i = 0; i < kCbPer; ++i) cbr[i] = __ldg(cb + tid + i * kCT);
    }
    // and this warp's first sink rows (the sinks t = c (mod C), one per warp)
    const int n_sinks = min(a.num_sinks, n_tok);
    const int my_sinks = (n_sinks > c) ? (n_sinks - c + C - 1) / C : 0;
    const char *kseg = static_cast<const char *>(a.K) + kv_seg * kHeadDim * EB;
    float4 sk_k = make_float4(0.f, 0.f, 0.f, 0.f), sk_v = sk_k;
    if (warp < my_sinks) {
        const size_t off = static_cast<size_t>(c + warp * C) * kHeadDim * EB;
        sk_k = load4<DT>(kseg + off, 4 * lane);
        sk_v = load4<DT>(vseg + off, 4 * lane);
    }
    cluster_wait();                                          // #2

    // ---- the leader finds the segment's k-th bin b* in its histogram and
    // hands (b*, count above b*) to every CTA of the cluster; meanwhile the
    // CTAs attend their share of the sinks (nothing there depends on b*)
    if (c == 0 && k > 0) {
        cta_find_bin<kFBins / kCT, kCT>([&](int i) { return sh.mhist[i]; }, static_cast<uint32_t>(k), sh.wtot, sh.sc);
        if (tid < C) {
            dsmem_st_u32(dsmem_map(&sh.bsd[0], static_cast<uint32_t>(tid)), sh.sc[0]);
            dsmem_st_u32(dsmem_map(&sh.bsd[1], static_cast<uint32_t>(tid)), sh.sc[1]);
        }
    }
    cluster_arrive_cta();                                    // #2b
    // Attention.  Each warp keeps its own online softmax; the warps' states
    // merge once at the end.  The sinks t = c (mod C) come first: one warp
    // per sink, lane l takes columns 4l..4l+3 of its stored key and value.
    WarpSoftmax<GM> ws;
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        ws.m[g] = -INFINITY;
        ws.l[g] = 0.f;
        ws.o[g][0] = ws.o[g][1] = ws.o[g][2] = ws.o[g][3] = 0.f;
    }
#pragma unroll 1
    for (int i = warp; i < my_sinks; i += kCW) {
        if (i != warp) {
            const size_t off = static_cast<size_t>(c + i * C) * kHeadDim * EB;
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
    cluster_wait();                                          // #2b

    // ---- 2. segment k-th bin b*, as the leader found it.  Tokens
    // above it are selected outright: flagged (entry bit 15), listed for the
    // attention and their code and value rows sent to L2.  Tokens in b* are
    // listed and re-scored together; their exact keys stay in this CTA's
    // shared memory for the other CTAs to read.
    const int nrows = (a.chunk + kFRow - 1) / kFRow;           // <= 64
    const uint32_t kSure = 0x80008000u, kWin = 0x40004000u;
    int bstar = kFBins;              // nothing selected when k == 0
    uint32_t above_bstar = 0;
    uint32_t *pend = sh.hist;                                        // free: the local histogram is published
    // each warp's direct list of attended tokens (kCWarpList entries)
    int32_t *wlist = reinterpret_cast<int32_t *>(sh.hist) + 2 * kCPend + kCWarpList * warp;
    if (lane == 0) sh.wcnt[warp] = 0;
    if (k > 0) {
        bstar = static_cast<int>(sh.bsd[0]);
        above_bstar = sh.bsd[1];
        const uint32_t b2 = static_cast<uint32_t>(bstar + 1) * 0x10001u;
        // warp w scans rows w, w + 8, ... (at most 8) of 256 entries, 8 per
        // lane: it flags the tokens above b* and keeps, per lane, a 64-bit mask
        // of them (bit 8 r + j: entry j of the lane's r-th row) and of the
        // tokens in b*.  One pass over the masks then lists them: lane by
        // lane, row by row (a fixed order), positions from 7 ballots.
        unsigned long long gmask = 0ull, emask = 0ull;
#pragma unroll 1
        for (int r = 0, row = warp; row < nrows; ++r, row += kCW) {
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
        // the threshold-bin tokens first: their code rows are re-read soon
        for (unsigned long long mm = emask; mm; mm &= mm - 1) {
            const int bit = __ffsll(static_cast<long long>(mm)) - 1;
            const int p = (warp + kCW * (bit >> 3)) * kFRow + 8 * lane + (bit & 7);
            const uint32_t slot = atomicAdd(&sh.sc[8], 1u);
            if (slot < kCPend) pend[slot] = static_cast<uint32_t>(p);
            prefetch_l2(crow + t0 + p);            // re-read below
            // its value row too: most of these tokens win
            if (VQ) {
                prefetch_l2(vsel + static_cast<size_t>(t0 + p) * kVqRowBytes);
                prefetch_l2(vsel + static_cast<size_t>(t0 + p) * kVqRowBytes + kVqRowBytes - 1);
            } else {
                prefetch_l2(vseg + static_cast<size_t>(t0 + p) * kHeadDim * EB);
                if (EB * kHeadDim > 128) prefetch_l2(vseg + static_cast<size_t>(t0 + p) * kHeadDim * EB + 128);
            }
        }
        for (unsigned long long mm = gmask; mm; mm &= mm - 1, ++pos) {
            const int bit = __ffsll(static_cast<long long>(mm)) - 1;
            const int t = t0 + (warp + kCW * (bit >> 3)) * kFRow + 8 * lane + (bit & 7);
            if (pos < static_cast<uint32_t>(kCWarpList)) wlist[pos] = t;
            prefetch_l2(crow + t);
            if (VQ) {                              // a 48-byte row may straddle two lines
                prefetch_l2(vsel + static_cast<size_t>(t) * kVqRowBytes);
                prefetch_l2(vsel + static_cast<size_t>(t) * kVqRowBytes + kVqRowBytes - 1);
            } else {
                prefetch_l2(vseg + static_cast<size_t>(t) * kHeadDim * EB);
                if (EB * kHeadDim > 128) prefetch_l2(vseg + static_cast<size_t>(t) * kHeadDim * EB + 128);
            }
        }
        if (lane == 0) sh.wcnt[warp] = n_w;
        __syncthreads();
        const uint32_t npend = sh.sc[8];
        if (tid == 0) {
            uint32_t n_sure = 0;
#pragma unroll
            for (int w2 = 0; w2 < kCW; ++w2) n_sure += sh.wcnt[w2];
            sh.pub[2] = n_sure;
        }
        if (npend <= static_cast<uint32_t>(kCPend)) {
            // token t0 + p was scored by lane p mod 32 (the table's bank
            // rotation): warp e mod 8 takes pending token e in that lane
#pragma unroll 1
            for (uint32_t e = warp; e < npend; e += kCW) {
                const int p = static_cast<int>(pend[e]);
                if (lane == (p & 31))
                    pend[kCPend + e] = score_key(lut2_score(sh.u.tab.t2, __ldg(crow + t0 + p), lane, qmu));
            }
            if (tid == 0) {
                sh.pub[0] = npend;
                sh.pub[1] = 0;
            }
        } else {
            // more than the shared list holds (flat or tie-heavy tables): every
            // token of bin b* with its exact key into this CTA's region of the
            // workspace list (one region of `chunk` entries per CTA)
            if (tid == 0) sh.sc[10] = 0;
            __syncthreads();
            uint2 *mine = a.cand + static_cast<size_t>(seg) * a.cand_cap + static_cast<size_t>(t0);
            emit_bin_tokens<kCT>(sh.bins, nrows, b2, sh.u.tab.t2, crow, t0, qmu, reinterpret_cast<int *>(&sh.sc[10]),
                            mine, max(0, min(a.chunk, a.cand_cap - t0)));
            __syncthreads();
            if (tid == 0) {
                sh.pub[0] = min(sh.sc[10], static_cast<uint32_t>(a.chunk));
                sh.pub[1] = 1;
            }
        }
    }
    cluster_arrive_cta();                                    // #3

    // Attention.  Each warp keeps its own online softmax; the warps' states
    // merge once at the end.  The sinks and the tokens above b* need no
    // candidate ranking, so they are attended while the other CTAs finish
    // their candidates; the winners of b* follow after the wait.
    char *ubase = reinterpret_cast<char *>(&sh.u);
    float (*luth)[GM] = reinterpret_cast<float (*)[GM]>(sh.ax + AL::kLuth);
    // the list a pass attends (its warps' direct lists concatenated, or a
    // window of kListCap tokens staged from the entry flags) lives in mhist,
    // unused by then
    constexpr uint32_t kListCap = kCList;
    int32_t *alist = reinterpret_cast<int32_t *>(sh.mhist);
    // per-head LUTs: q_h[4s:4s+4] . c[s][j]
#pragma unroll
    for (int i = 0; i < kCbPer; ++i) {
        const int r = tid + i * kCT, sidx = r >> 4;
        const float4 c4 = cbr[i];
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            float v = sh.qs[g][4 * sidx] * c4.x;
            v = fmaf(sh.qs[g][4 * sidx + 1], c4.y, v);
            v = fmaf(sh.qs[g][4 * sidx + 2], c4.z, v);
            v = fmaf(sh.qs[g][4 * sidx + 3], c4.w, v);
            luth[r][g] = v;
        }
    }
    __syncthreads();
    uint32_t win_before = 0;           // this thread's share of winners with token < t0
    // A pass attends its list split evenly over the warps: the warps' direct
    // lists concatenated in warp order, or, when some warp's list overflowed,
    // the tokens staged from the entry flags in windows of kListCap.
    bool direct = true;
    uint32_t n_list = 0;
    for (int w2 = 0; w2 < kCW; ++w2) {
        direct = direct && sh.wcnt[w2] <= static_cast<uint32_t>(kCWarpList);
        n_list += sh.wcnt[w2];
    }
    uint32_t bit2 = kSure;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        int pass_v = pass;
        asm volatile("" : "+r"(pass_v));   // keeps the two passes in one copy of the code
        if (pass_v == 1) {
            cluster_wait();                                  // #3 (every thread reaches pass 1)
            if (k == 0) break;
            // ---- exact winners among the threshold-bin candidates of the
            // whole cluster (the same answer in every CTA): a candidate wins
            // when fewer than `need` candidates come before it (key
            // descending, token ascending).
            if (tid < C) {
                sh.cbase[tid] = dsmem_ld_u32(dsmem_map(&sh.pub[0], tid));
                sh.cover[tid] = dsmem_ld_u32(dsmem_map(&sh.pub[1], tid));
                sh.cnsure[tid] = dsmem_ld_u32(dsmem_map(&sh.pub[2], tid));
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t run = 0, over = 0;
                for (int r = 0; r < C; ++r) {
                    const uint32_t t = sh.cbase[r];
                    sh.cbase[r] = run;
                    run += t;
                    over |= sh.cover[r];
                }
                sh.cbase[C] = run;
                sh.sc[11] = over;
            }
            __syncthreads();
            const int ncand = static_cast<int>(sh.cbase[C]);
            const bool any_over = sh.sc[11] != 0;
            const uint32_t need = static_cast<uint32_t>(k) - above_bstar;   // >= 1
            const uint2 *gcand = a.cand + static_cast<size_t>(seg) * a.cand_cap;
            // candidate e of the cluster as (key, token); a by-value functor,
            // so that the out-of-line refine takes it in registers
            const ClusterCands cand_at{sh.cbase, sh.cover, static_cast<uint32_t>(__cvta_generic_to_shared(pend)), C, a.chunk,
                                      gcand};
            const bool ranked = ncand <= kFRankMax && !any_over;
            for (int i = tid; i < kCMaxChunk / 32; i += kCT) sh.u.sel.winbits[i] = 0;
            if (ranked) {
                for (int e = tid; e < ncand; e += kCT) {
                    const uint2 v = cand_at(e);
                    sh.u.sel.ck[e] = (static_cast<unsigned long long>(v.x) << 32) | ~v.y;
                }
            }
            __syncthreads();
            if (ranked) {
                for (int e = tid; e < ncand; e += kCT) {
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
                // the radix scratch is this CTA's mhist: nobody reads it after #3
                win_before += refine_by_radix<kCT>(cand_at, ncand, need, t0, a.chunk, sh.u.sel.winbits, sh.mhist,
                                              sh.wtot, sh.sc);
            }
            __syncthreads();
            // each warp lists the winners of its share of the chunk's bitmap,
            // in ascending token order
            {
                const int nwords = (a.chunk + 31) / 32;
                const int wpw = (nwords + kCW - 1) / kCW;        // <= 64 (chunk <= 32768)
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
                        if (pos < static_cast<uint32_t>(kCWarpList)) wlist[pos] = t0 + 32 * wd + __ffs(mm) - 1;
                }
                if (lane == 0) sh.wcnt[warp] = n_w;
            }
            __syncthreads();
            direct = true;
            n_list = 0;
            for (int w2 = 0; w2 < kCW; ++w2) {
                direct = direct && sh.wcnt[w2] <= static_cast<uint32_t>(kCWarpList);
                n_list += sh.wcnt[w2];
            }
            bit2 = kWin;
            if (!direct || a.idx_out) {
                // flag the winners of this chunk (entry bit 14)
                const uint32_t b2 = static_cast<uint32_t>(bstar + 1) * 0x10001u;
#pragma unroll 1
                for (int row = warp; row < nrows; row += kCW) {
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
        const uint32_t n_windows = direct ? 1u : (n_list + kListCap - 1) / kListCap;
        // where each warp's direct list starts in the pass's list order
        if (tid == 0) {
            uint32_t run = 0;
            for (int w2 = 0; w2 < kCW; ++w2) {
                sh.wpre[w2] = run;
                run += sh.wcnt[w2];
            }
            sh.wpre[kCW] = run;
        }
        __syncthreads();
        // the direct lists concatenated into the pass list (alist), one
        // entry per lane and warp
        if (direct) {
            const int32_t *wl_all = reinterpret_cast<const int32_t *>(sh.hist) + 2 * kCPend;
            for (uint32_t i = lane; i < sh.wcnt[warp]; i += 32) alist[sh.wpre[warp] + i] = wl_all[kCWarpList * warp + i];
            __syncthreads();
        }
        char *vb = warp < AL::kInUnion ? ubase + warp * AL::kRows * AL::kRowBytes
                                       : sh.ax + (warp - AL::kInUnion) * AL::kRows * AL::kRowBytes;
        int32_t *tok = reinterpret_cast<int32_t *>(ubase + AL::kTok) + 32 * warp;
#pragma unroll 1
        for (uint32_t win = 0; win < n_windows; ++win) {
            uint32_t total = n_list;
            if (!direct) {
                const uint32_t wbase = win * kListCap;
                stage_flagged<kCT>(sh.bins, nrows, bit2, wbase, t0, sh.rowcnt, sh.wtot, alist, kListCap);
                total = min(kListCap, n_list - wbase);
            }
            // this warp's share: an even split of the window's list (a fixed
            // order, so every run accumulates the same terms in the same order)
            const uint32_t per = (total + kCW - 1) / kCW;
            const uint32_t lo = min(total, per * static_cast<uint32_t>(warp)), hi = min(total, lo + per);
            // batches of up to AL::kRows tokens, one per lane: all the batch's
            // value rows are requested at once while its logits are formed
#pragma unroll 1
            for (uint32_t b0 = lo; b0 < hi; b0 += AL::kRows) {
                const int nb = static_cast<int>(min(static_cast<uint32_t>(AL::kRows), hi - b0));
                const bool valid = lane < nb;
                int t = 0;
                if (valid) t = alist[b0 + static_cast<uint32_t>(lane)];
                tok[lane] = t;
                __syncwarp();
                warp_stage_v<DT, VQ>(vb, tok, 0, nb, vsel, lane);
                cp_async_commit();
                const uint4 row = valid ? __ldg(crow + t) : make_uint4(0u, 0u, 0u, 0u);
                float lg[GM];
#pragma unroll
                for (int g = 0; g < GM; ++g) lg[g] = -INFINITY;
                if (valid) {
                    float acc[GM];
#pragma unroll
                    for (int g = 0; g < GM; ++g) acc[g] = 0.f;
                    // code word wq holds subspaces 8 wq .. 8 wq + 7 (no
                    // run-time indexing of a register array)
#pragma unroll 2
                    for (int wq = 0; wq < 4; ++wq) {
                        const uint32_t word = wq == 0 ? row.x : (wq == 1 ? row.y : (wq == 2 ? row.z : row.w));
#pragma unroll
                        for (int k8 = 0; k8 < 8; ++k8) {
                            const int j = (word >> (4 * k8)) & 15;
                            const float *lp = luth[(8 * wq + k8) * kClusters + j];
#pragma unroll
                            for (int g = 0; g < GM; g += 4) {
                                const float4 v4 = *reinterpret_cast<const float4 *>(lp + g);
                                acc[g] += v4.x;
                                acc[g + 1] += v4.y;
                                acc[g + 2] += v4.z;
                                acc[g + 3] += v4.w;
                            }
                        }
                    }
#pragma unroll
                    for (int g = 0; g < GM; ++g) lg[g] = (g < group) ? (acc[g] + sh.qmu_h[g]) * a.scale : -INFINITY;
                }
                warp_softmax_batch(ws, lg);
                cp_async_wait_all();
                __syncwarp();
                warp_fma_v<DT, GM, VQ>(ws, vb, lg, 0, nb, lane);
                __syncwarp();                  // tok and the staged rows are reused by the next batch
            }
            if (!direct) __syncthreads();
        }
    }

    // selected tokens in ascending order into idx_out, after the selected
    // tokens of the earlier chunks (their counts above b* plus their winners)
    if (a.idx_out && k > 0) {
        uint32_t before = win_before;
        if (tid < c) before += sh.cnsure[tid];
        uint32_t out_base;
        cta_excl_scan<kCT>(before, sh.wtot, &out_base);
#pragma unroll 1
        for (int row = warp; row < nrows; row += kCW) {
            uint32_t cnt = __popc(flagged8(sh.bins, row, lane, kSure | kWin));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
            if (lane == 0) sh.rowcnt[row] = cnt;
        }
        __syncthreads();
        rows_to_bases<kCT>(sh.rowcnt, nrows, sh.wtot);
        int32_t *io = a.idx_out + static_cast<size_t>(seg) * a.kmax;
#pragma unroll 1
        for (int row = warp; row < nrows; row += kCW) {
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

    // merge the warps' softmax states into this CTA's partial (m, l, o):
    // o into red[0] (each thread reads and then writes only its own
    // elements), (m, l) into pml; red aliases the value-staging buffers, so
    // every warp must be done first
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
        *reinterpret_cast<float4 *>(&sh.u.red[warp][g][lane * 4]) =
            make_float4(ws.o[g][0], ws.o[g][1], ws.o[g][2], ws.o[g][3]);
    __syncthreads();
    for (int e = tid; e < GM * kHeadDim; e += kCT) {
        const int g = e / kHeadDim, d = e % kHeadDim;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kCW; ++w) mx = fmaxf(mx, sh.wm[w][g]);
        float sacc = 0.f, lsum = 0.f;
        if (mx != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kCW; ++w) {
                const float mw = sh.wm[w][g];
                const float f = (mw == -INFINITY) ? 0.f : __expf(mw - mx);
                sacc = fmaf(f, sh.u.red[w][g][d], sacc);
                lsum = fmaf(f, sh.wl[w][g], lsum);
            }
        }
        sh.u.red[0][g][d] = sacc;
        if (d == 0) sh.pml[g] = make_float2(mx, lsum);
    }
    if (tid < C) sh.rbase[tid] = dsmem_map(&sh.u.red[0][0][0], static_cast<uint32_t>(tid));
    cluster_arrive_cta();                                    // #4
    cluster_wait();

    // ---- output: this CTA merges its slice of the segment's group x 128
    // output elements over the C partials (fixed order r = 0..C-1)
    {
        float2 *mls = reinterpret_cast<float2 *>(sh.mhist);                   // [C][GM]
        float *wts = reinterpret_cast<float *>(mls + kMaxCluster * GM);       // [C][GM]
        for (int i = tid; i < C * GM; i += kCT)
            mls[i] = dsmem_ld_f2(dsmem_map(&sh.pml[i % GM], static_cast<uint32_t>(i / GM)));
        __syncthreads();
        if (tid < GM) {
            float mx = -INFINITY;
            for (int r = 0; r < C; ++r) mx = fmaxf(mx, mls[r * GM + tid].x);
            float l = 0.f;
            for (int r = 0; r < C; ++r) {
                const float2 ml = mls[r * GM + tid];
                const float f = (ml.x == -INFINITY) ? 0.f : __expf(ml.x - mx);
                wts[r * GM + tid] = f;
                l = fmaf(ml.y, f, l);
            }
            const float inv = (l > 0.f) ? __fdividef(1.f, l) : 0.f;
            for (int r = 0; r < C; ++r) wts[r * GM + tid] *= inv;
        }
        __syncthreads();
        const int nel = group * kHeadDim;
        const int per = (nel + C - 1) / C;
        const int e1 = min((c + 1) * per, nel);
        for (int e = c * per + tid; e < e1; e += kCT) {
            const int g = e / kHeadDim, d = e % kHeadDim;
            const uint32_t off = 4u * static_cast<uint32_t>(g * kHeadDim + d);
            float acc = 0.f;
            for (int r = 0; r < C; ++r) acc = fmaf(wts[r * GM + g], dsmem_ld_f32(sh.rbase[r] + off), acc);
            const size_t orow = (static_cast<size_t>(b) * a.hq + static_cast<size_t>(h) * group + g) * kHeadDim + d;
            if (DT == SIKV_DTYPE_F32)
                static_cast<float *>(a.out)[orow] = acc;
            else
                static_cast<unsigned short *>(a.out)[orow] = static_cast<unsigned short>(f32_to_bf16_bits(acc));
        }
    }
    if (a.idx_out && c == 0) {
        int32_t *io = a.idx_out + static_cast<size_t>(seg) * a.kmax;
        for (int i = k + tid; i < a.kmax; i += kCT) io[i] = -1;
    }
    cluster_arrive_relaxed();                                // #5: no CTA leaves while its partial is read
    cluster_wait();
}

// Per device and cluster size: how many clusters of the kernel fit on the
// device at once (0: the launch configuration is not possible).  The kernel's
// shared-memory limit and the non-portable cluster sizes are enabled on the
// first query on each device.  Values are idempotent; concurrent first calls
// store the same value.
constexpr int kMaxDevices = 64;

template <int DT, int GM, bool VQ>
int max_clusters_of(int csize) {
    static std::atomic<int> cached[kMaxDevices][kMaxCluster + 1];   // 0: unknown, else count + 1
    int dev = 0;
    if (csize < 1 || csize > kMaxCluster) return 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < kMaxDevices) {
        const int v = cached[dev][csize].load(std::memory_order_relaxed);
        if (v > 0) return v - 1;
    }
    auto kern = decode_cluster_kernel<DT, GM, VQ>;
    const size_t smem = sizeof(ClusterSmem<GM>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return 0;
    if (csize > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(csize));
    cfg.blockDim = dim3(kCT);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = static_cast<unsigned>(csize);
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (dev >= 0 && dev < kMaxDevices) cached[dev][csize].store(n + 1, std::memory_order_relaxed);
    return n;
}

int max_clusters(const sikv_params &p, bool vq, int gm, int csize) {
    if (p.dtype == SIKV_DTYPE_BF16)
        return vq ? (gm == 4 ? max_clusters_of<SIKV_DTYPE_BF16, 4, true>(csize)
                             : max_clusters_of<SIKV_DTYPE_BF16, 8, true>(csize))
                  : (gm == 4 ? max_clusters_of<SIKV_DTYPE_BF16, 4, false>(csize)
                             : max_clusters_of<SIKV_DTYPE_BF16, 8, false>(csize));
    return vq ? (gm == 4 ? max_clusters_of<SIKV_DTYPE_F32, 4, true>(csize) : max_clusters_of<SIKV_DTYPE_F32, 8, true>(csize))
              : (gm == 4 ? max_clusters_of<SIKV_DTYPE_F32, 4, false>(csize)
                         : max_clusters_of<SIKV_DTYPE_F32, 8, false>(csize));
}

template <int DT, int GM, bool VQ>
sikv_status launch_cluster_t(const ClusterArgs &args, const ClusterPlan &plan, cudaStream_t stream) {
    auto kern = decode_cluster_kernel<DT, GM, VQ>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(plan.grid));
    cfg.blockDim = dim3(kCT);
    cfg.dynamicSmemBytes = sizeof(ClusterSmem<GM>);   // limit raised by cluster_plan on this device
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = static_cast<unsigned>(plan.csize);
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args) == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace

ClusterPlan cluster_plan(const sikv_params &p, bool vq) {
    ClusterPlan plan;
    const int group = p.num_q_heads / p.num_kv_heads;
    const int gm = group <= 4 ? 4 : 8;
    const int segs = p.batch * p.num_kv_heads;
    const int nmax = p.max_seq_len;
    const int cmin = std::max(1, (nmax + kCMaxChunk - 1) / kCMaxChunk);
    if (cmin > kMaxCluster || segs < 1) return plan;
    constexpr int kMinChunk = 2048;
    auto chunk_of = [&](int cs) {
        const int ch = (nmax + cs - 1) / cs;
        return (ch + kCT - 1) / kCT * kCT;
    };
    // the largest cluster whose whole batch runs in one wave (and whose
    // chunks are not tiny); else the smallest possible cluster, whose waves
    // carry the most tokens per CTA
    int csize = 0;
    for (int cs = kMaxCluster; cs >= cmin; --cs) {
        if (cs > cmin && chunk_of(cs) < kMinChunk) continue;
        if ((nmax + chunk_of(cs) - 1) / chunk_of(cs) != cs) continue;   // every CTA holds tokens
        const int fit = max_clusters(p, vq, gm, cs);
        if (fit >= segs) {
            csize = cs;
            break;
        }
    }
    if (csize == 0) {
        if (max_clusters(p, vq, gm, cmin) < 1) return plan;
        csize = cmin;
    }
    const int chunk = chunk_of(csize);
    if (chunk > kCMaxChunk) return plan;
    plan.ok = true;
    plan.csize = csize;
    plan.chunk = chunk;
    plan.npt = chunk / kCT;
    plan.gm = gm;
    plan.grid = segs * csize;
    return plan;
}

sikv_status launch_decode_cluster(const sikv_params &p, const ClusterPlan &plan, const void *q, const void *K,
                                  const void *V, const uint8_t *vq, const uint8_t *codes, const float *codebook,
                                  const float *mu, const int32_t *seq_lens, const int32_t *k_per_seq, void *out,
                                  int32_t *idx_out, float *scores_out, uint2 *cand, size_t cand_cap, int32_t *status,
                                  cudaStream_t stream) {
    ClusterArgs a;
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
    a.csize = plan.csize;
    a.chunk = plan.chunk;
    a.npt = plan.npt;
    a.cand_cap = static_cast<int>(cand_cap);
    a.scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf(static_cast<float>(p.head_dim));
    a.cand = cand;
    a.status = status;
    const bool v = vq != nullptr;
    if (v) {
        if (p.dtype == SIKV_DTYPE_BF16)
            return plan.gm == 4 ? launch_cluster_t<SIKV_DTYPE_BF16, 4, true>(a, plan, stream)
                                : launch_cluster_t<SIKV_DTYPE_BF16, 8, true>(a, plan, stream);
        return plan.gm == 4 ? launch_cluster_t<SIKV_DTYPE_F32, 4, true>(a, plan, stream)
                            : launch_cluster_t<SIKV_DTYPE_F32, 8, true>(a, plan, stream);
    }
    if (p.dtype == SIKV_DTYPE_BF16)
        return plan.gm == 4 ? launch_cluster_t<SIKV_DTYPE_BF16, 4, false>(a, plan, stream)
                            : launch_cluster_t<SIKV_DTYPE_BF16, 8, false>(a, plan, stream);
    return plan.gm == 4 ? launch_cluster_t<SIKV_DTYPE_F32, 4, false>(a, plan, stream)
                        : launch_cluster_t<SIKV_DTYPE_F32, 8, false>(a, plan, stream);
}

}  // namespace sikv
