// Device helpers shared by the single-launch decode kernels (the
// cooperative one in decode_fused.cu and the cluster one in
// decode_cluster.cu): CTA-wide scans, histogram threshold search, radix
// select, the bin-entry masks of the per-token bins, the warp online softmax
// and the value-row staging of the attention passes.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 items 2-4.
#pragma once

#include "score_device.cuh"

namespace sikv {

namespace {

constexpr int kFT = 256;                 // threads per CTA
constexpr int kFW = kFT / 32;            // warps per CTA
constexpr int kFBins = 1024;             // histogram bins per segment
constexpr int kFListCap = 2048;          // attended tokens staged per window
constexpr int kFMaxNpt = 64;             // token slots per thread at most
constexpr int kFMaxChunk = kFMaxNpt * kFT;
constexpr int kFRankMax = 512;           // up to this many candidates: rank directly
constexpr int kFUnroll = 4;              // code rows in flight per thread
constexpr int kFPrefetchRows = 16;       // code rows per thread sent to L2 during the prologue
constexpr int kFPend = kFBins / 4;       // threshold-bin tokens of a CTA re-scored together
constexpr int kFDirect = kFBins / 2;     // attended tokens listed directly during the scans
constexpr int kFWarpList = kFDirect / kFW;   // of which each warp lists (and attends) at most this many
constexpr int kFVBytes = 4096;           // value rows staged per warp: 16 bf16 or 8 fp32 rows
constexpr int kFRow = 256;               // tokens per row scan of a warp (32 lanes x 8)

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Exclusive scan over the CTA (NT threads) of one value per thread; wtot
// holds NT / 32 + 1 words.
template <int NT = kFT>
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t *wtot, uint32_t *total) {
    constexpr int NW = NT / 32;
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
        for (int w = 0; w < NW; ++w) {
            const uint32_t t = wtot[w];
            wtot[w] = run;
            run += t;
        }
        wtot[NW] = run;
    }
    __syncthreads();
    const uint32_t r = wtot[warp] + incl - v;
    *total = wtot[NW];
    __syncthreads();
    return r;
}

// In a histogram of PER * NT bins scanned from the top bin down, finds the
// bin where the running count first reaches `need` (1 <= need <= total).
// Each thread loads its PER consecutive bins once.  Writes (bin, count above)
// to out[0..1]; out is left untouched when the total is below need.  Ends
// synchronized.
template <int PER, int NT = kFT, typename Load>
__device__ __forceinline__ void cta_find_bin(Load load, uint32_t need, uint32_t *wtot, uint32_t *out) {
    const int top = PER * NT - 1 - static_cast<int>(threadIdx.x) * PER;
    uint32_t h[PER];
    uint32_t loc = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        h[i] = load(top - i);
        loc += h[i];
    }
    uint32_t total;
    uint32_t above = cta_excl_scan<NT>(loc, wtot, &total);
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
template <int NT = kFT, typename KeyF, typename KeepF>
__device__ __noinline__ uint32_t cta_radix_select(KeyF key, KeepF keep, int n, uint32_t need, uint32_t *hist,
                                                  uint32_t *wtot, uint32_t *sc, uint32_t *need_left) {
    uint32_t prefix = 0, mask = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0;
        __syncthreads();
        for (int e = threadIdx.x; e < n; e += NT) {
            if (!keep(e)) continue;
            const uint32_t k = key(e);
            if (((k ^ prefix) & mask) == 0) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (NT == 256) {
            cta_find_bin<1, NT>([&](int i) { return hist[i]; }, need, wtot, sc);
        } else {
            // NT threads and 256 buckets: the upper threads hold empty buckets
            cta_find_bin<1, NT>([&](int i) { return i < 256 ? hist[i] : 0u; }, need, wtot, sc);
        }
        prefix |= sc[0] << shift;
        mask |= 255u << shift;
        need -= sc[1];
        __syncthreads();
    }
    *need_left = need;
    return prefix;
}

// bins[] holds one 16-bit entry per token of the chunk in token order (entry
// p is token t0 + p): bin + 1 in bits 0-13, flags in bits 14-15.  A lane
// scans 8 consecutive entries with one 16-byte load.  The tests below give,
// per 16-bit half of a word, a bit at position 0 (low half) or 16 (high half).
// half_ge: [entry >= thr] for thr2 = thr * 0x10001, thr <= 0x4000.  Per half
// v + 0x4000 - thr lies in [0, 0x7FFF] (v, thr < 0x4000 after masking the
// flags), so the halves never borrow from each other, and its bit 14 is
// [v >= thr].
__device__ __forceinline__ uint32_t half_ge(uint32_t w, uint32_t thr2) {
    return (((w & 0x3FFF3FFFu) + 0x40004000u - thr2) >> 14) & 0x00010001u;
}
__device__ __forceinline__ uint32_t half_gt(uint32_t w, uint32_t thr2) { return half_ge(w, thr2 + 0x10001u); }
__device__ __forceinline__ uint32_t half_eq(uint32_t w, uint32_t thr2) {
    return half_ge(w, thr2) & ~half_ge(w, thr2 + 0x10001u);
}
// The halves carrying any of the flag bits bit2 (bits 14 and / or 15 of each half).
__device__ __forceinline__ uint32_t half_flagged(uint32_t w, uint32_t bit2) {
    const uint32_t t = (w & bit2) >> 14;
    return (t | (t >> 1)) & 0x00010001u;
}
// The flag pattern (bit 15 or 14 of each half) of the halves marked in m.
__device__ __forceinline__ uint32_t sure_flags(uint32_t m) { return m << 15; }
__device__ __forceinline__ uint32_t win_flags(uint32_t m) { return m << 14; }
// 8-bit mask (bit j = entry j of the lane's 8) from the four words' half bits
__device__ __forceinline__ uint32_t mask8(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
    const uint32_t a = m0 | (m1 << 2) | (m2 << 4) | (m3 << 6);   // entry 2k at bit 2k, entry 2k+1 at bit 16 + 2k
    return (a | (a >> 15)) & 0xFFu;
}
// The half bits of word k (entries 2k, 2k+1) of an 8-bit per-entry mask.
__device__ __forceinline__ uint32_t halves_of(uint32_t m8, int k) {
    return ((m8 >> (2 * k)) & 1u) | (((m8 >> (2 * k + 1)) & 1u) << 16);
}

// Appends the tokens of bin b* (entries equal to b2 in both halves) to the
// segment's candidate list one by one with their exact keys, each re-scored
// by the lane that scored it (same table, same rotation, same order of
// additions, so bit-identical).  The fallback for a CTA whose threshold bin
// holds more tokens than the shared list takes; ties-heavy tables only.
template <int NT = kFT>
__device__ __noinline__ void emit_bin_tokens(const uint16_t *bins, int nrows, uint32_t b2, const float *t2,
                                             const uint4 *crow, int t0, float qmu, int *ncand, uint2 *cand, int cap) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
    for (int row = warp; row < nrows; row += NT / 32) {
        const uint4 w = *reinterpret_cast<const uint4 *>(bins + row * kFRow + 8 * lane);
        const uint32_t eq = mask8(half_eq(w.x, b2), half_eq(w.y, b2), half_eq(w.z, b2), half_eq(w.w, b2));
        // token t0 + p was scored by lane p mod 32 (the table's bank rotation)
        uint32_t todo = __ballot_sync(0xffffffffu, eq != 0);
        while (todo) {
            const int src = __ffs(todo) - 1;
            todo &= todo - 1;
            const uint32_t em = __shfl_sync(0xffffffffu, eq, src);
            for (uint32_t mm = em; mm; mm &= mm - 1) {
                const int p = row * kFRow + 8 * src + __ffs(mm) - 1;
                if (lane == (p & 31)) {
                    const float sv = lut2_score(t2, __ldg(crow + t0 + p), lane, qmu);
                    const int slot = atomicAdd(ncand, 1);
                    if (slot < cap) cand[slot] = make_uint2(score_key(sv), static_cast<uint32_t>(t0 + p));
                }
            }
        }
    }
}

// Turns sh.rowcnt-style per-row counts into exclusive prefix sums in place and
// returns the total.  Expects the counts to be visible; ends synchronized.
template <int NT = kFT>
__device__ __forceinline__ uint32_t rows_to_bases(uint32_t *rowcnt, int nrows, uint32_t *wtot) {
    uint32_t total;
    const int tid = threadIdx.x;
    const uint32_t v = tid < nrows ? rowcnt[tid] : 0u;
    const uint32_t run = cta_excl_scan<NT>(v, wtot, &total);
    if (tid < nrows) rowcnt[tid] = run;
    __syncthreads();
    return total;
}

// 8-bit mask of the entries of row `row` (8 per lane) that carry flag bit2.
__device__ __forceinline__ uint32_t flagged8(const uint16_t *bins, int row, int lane, uint32_t bit2) {
    const uint4 w = *reinterpret_cast<const uint4 *>(bins + row * kFRow + 8 * lane);
    return mask8(half_flagged(w.x, bit2), half_flagged(w.y, bit2), half_flagged(w.z, bit2), half_flagged(w.w, bit2));
}

// Fills list[0, wn) with the tokens of the entries flagged bit2 whose
// ordinals (ascending token order) lie in [wbase, wbase + wn).  The fallback
// when a pass holds more tokens than the direct list takes.  Ends synchronized.
// (Inlined: as a call it costs the kernel spills around the call site.)
template <int NT = kFT>
__device__ __forceinline__ void stage_flagged(const uint16_t *bins, int nrows, uint32_t bit2, uint32_t wbase, int t0,
                                           uint32_t *rowcnt, uint32_t *wtot, int32_t *list,
                                           uint32_t cap = kFListCap) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
    for (int row = warp; row < nrows; row += NT / 32) {
        uint32_t cnt = __popc(flagged8(bins, row, lane, bit2));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
        if (lane == 0) rowcnt[row] = cnt;
    }
    __syncthreads();
    rows_to_bases<NT>(rowcnt, nrows, wtot);
#pragma unroll 1
    for (int row = warp; row < nrows; row += NT / 32) {
        const uint32_t m = flagged8(bins, row, lane, bit2);
        uint32_t incl = __popc(m);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o2 = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o2;
        }
        uint32_t ord = rowcnt[row] + incl - __popc(m);
        for (uint32_t mm = m; mm; mm &= mm - 1, ++ord) {
            const int t = t0 + row * kFRow + 8 * lane + __ffs(mm) - 1;
            if (ord >= wbase && ord < wbase + cap) list[ord - wbase] = t;
        }
    }
    __syncthreads();
}

// Online-softmax state of one warp: running max m and sum l per head (equal
// in every lane) and the lane's four output columns (4 lane .. 4 lane + 3).
template <int GM>
struct WarpSoftmax {
    float m[GM], l[GM], o[GM][4];
};

// A batch of up to 32 entries, one per lane (logit -INFINITY: no entry).
// Folds the batch's maximum into m, rescales l and o, adds the batch's
// weights to l and turns lg into the lane's weight exp(lg - m).
template <int GM>
__device__ __forceinline__ void warp_softmax_batch(WarpSoftmax<GM> &s, float (&lg)[GM]) {
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        float mx = lg[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mn = fmaxf(s.m[g], mx);
        const float alpha = (s.m[g] == -INFINITY) ? 0.f : __expf(s.m[g] - mn);
        const float pr = (lg[g] == -INFINITY) ? 0.f : __expf(lg[g] - mn);
        float sum = pr;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        s.l[g] = fmaf(s.l[g], alpha, sum);
        s.m[g] = mn;
#pragma unroll
        for (int i = 0; i < 4; ++i) s.o[g][i] *= alpha;
        lg[g] = pr;
    }
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

// Closes the current group of this thread's cp.async copies.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Waits until at most one group of this thread's copies is still in flight.
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Waits until none of this thread's copies is in flight.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Value rows staged by a warp: two halves of its buffer, so that one half
// is consumed while the other is in flight.
template <int DT, bool VQ>
struct VStage {
    static constexpr int kRowBytes = VQ ? kVqRowBytes : kHeadDim * ElemBytes<DT>::value;
    static constexpr int kHalf = VQ ? 16 : kFVBytes / kRowBytes / 2;  // 16 (2-bit), 8 (bf16) or 4 (fp32) rows
};

// Starts copying the value rows of tokens tok[j0 .. j0 + n) into vb (row j
// at j * kRowBytes), 16 bytes per copy, all in flight at once.
template <int DT, bool VQ>
__device__ __forceinline__ void warp_stage_v(char *vb, const int32_t *tok, int j0, int n, const char *vseg,
                                             int lane) {
    constexpr int kRowBytes = VStage<DT, VQ>::kRowBytes, kChunks = kRowBytes / 16;
#pragma unroll 1
    for (int i = lane; i < n * kChunks; i += 32) {
        const int j = i / kChunks, cc = i % kChunks;
        cp_async16(vb + j * kRowBytes + 16 * cc,
                   vseg + static_cast<size_t>(tok[j0 + j]) * kRowBytes + 16 * cc);
    }
}

// o += sum over the staged rows j < n of pr_{j0+j} V[row j]; lane l takes
// columns 4l..4l+3 (a 2-bit row is read back as min + level * step).
template <int DT, int GM, bool VQ>
__device__ __forceinline__ void warp_fma_v(WarpSoftmax<GM> &s, const char *vb, const float (&pr)[GM], int j0, int n,
                                           int lane) {
    constexpr int kRowBytes = VStage<DT, VQ>::kRowBytes;
#pragma unroll 2
    for (int j = 0; j < n; ++j) {
        float4 vv;
        if (VQ) {
            vv = vq_decode4(reinterpret_cast<const uint8_t *>(vb + j * kRowBytes), lane);
        } else if (DT == SIKV_DTYPE_BF16) {
            const uint2 w = *reinterpret_cast<const uint2 *>(vb + j * kRowBytes + 8 * lane);
            vv = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
        } else {
            vv = *reinterpret_cast<const float4 *>(vb + j * kRowBytes + 16 * lane);
        }
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            const float w = __shfl_sync(0xffffffffu, pr[g], j0 + j);
            s.o[g][0] = fmaf(w, vv.x, s.o[g][0]);
            s.o[g][1] = fmaf(w, vv.y, s.o[g][1]);
            s.o[g][2] = fmaf(w, vv.z, s.o[g][2]);
            s.o[g][3] = fmaf(w, vv.w, s.o[g][3]);
        }
    }
}

// Winners among many candidates (more than the rank path takes): radix
// select of the need-th key and of the lowest tied token indices, then one
// marking pass.  Returns this thread's count of winners before the chunk.
// Kept out of line: it only runs for heavily tied or flat score tables.
template <int NT = kFT, typename CandF>
__device__ __noinline__ uint32_t refine_by_radix(CandF cand, int ncand, uint32_t need, int t0, int chunk,
                                                 uint32_t *winbits, uint32_t *hist, uint32_t *wtot, uint32_t *sc) {
    uint32_t ties_needed, left, before = 0;
    const uint32_t T = cta_radix_select<NT>([&](int e) { return cand(e).x; }, [&](int) { return true; }, ncand,
                                        need, hist, wtot, sc, &ties_needed);
    // the ties_needed lowest token indices among keys equal to T
    const uint32_t tie_idx = ~cta_radix_select<NT>([&](int e) { return ~cand(e).y; },
                                               [&](int e) { return cand(e).x == T; }, ncand, ties_needed,
                                               hist, wtot, sc, &left);
    for (int e = threadIdx.x; e < ncand; e += NT) {
        const uint2 v = cand(e);
        if (v.x > T || (v.x == T && v.y <= tie_idx)) {
            const int rel = static_cast<int>(v.y) - t0;
            if (rel >= 0 && rel < chunk) atomicOr(&winbits[rel >> 5], 1u << (rel & 31));
            else if (rel < 0) ++before;
        }
    }
    return before;
}

// The same over a candidate list in global memory.
template <int NT = kFT>
__device__ __noinline__ uint32_t refine_by_radix(const uint2 *cand, int ncand, uint32_t need, int t0, int chunk,
                                                 uint32_t *winbits, uint32_t *hist, uint32_t *wtot, uint32_t *sc) {
    uint32_t ties_needed, left, before = 0;
    const uint32_t T = cta_radix_select<NT>([&](int e) { return __ldcg(cand + e).x; }, [&](int) { return true; }, ncand,
                                        need, hist, wtot, sc, &ties_needed);
    // the ties_needed lowest token indices among keys equal to T
    const uint32_t tie_idx = ~cta_radix_select<NT>([&](int e) { return ~__ldcg(cand + e).y; },
                                               [&](int e) { return __ldcg(cand + e).x == T; }, ncand, ties_needed,
                                               hist, wtot, sc, &left);
    for (int e = threadIdx.x; e < ncand; e += NT) {
        const uint2 v = __ldcg(cand + e);
        if (v.x > T || (v.x == T && v.y <= tie_idx)) {
            const int rel = static_cast<int>(v.y) - t0;
            if (rel >= 0 && rel < chunk) atomicOr(&winbits[rel >> 5], 1u << (rel & 31));
            else if (rel < 0) ++before;
        }
    }
    return before;
}

}  // namespace

}  // namespace sikv
