// Prefill encoder: channel mean, sign-pattern codes and the one-pass codebook.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 1 (sign-based 1-bit VQ: channel-mean
// normalization, 4-dim sub-vectors -> 16 sign-pattern clusters, codebook
// without iterations) and item 3 (token-wise codes, 64 sink tokens).
//
// Four launches.  Each (sequence, KV head) segment is cut into token chunks,
// one CTA per chunk:
//   enc_mean_partial   K -> exact channel sums of each chunk (plain fp64 where
//                      that is exact, double-double otherwise)
//   enc_mean_final     the chunks' sums -> mu, the correctly rounded fp32 mean
//   enc_codes_partial  K, mu -> packed codes and each chunk's cluster sums
//                      and counts
//   enc_codebook_final the chunks' partials -> centroids and cluster sizes
// K is read twice (the mean must be known before any sign is taken).  The
// chunk length is chosen per shape and device so that the chunk CTAs fill
// whole waves of the GPU (encode_layout).  All sums run in a fixed order.
#include <cuda_bf16.h>

#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / 32;
constexpr int kEncUnroll = 4;      // rows in flight per thread, fp32 mean chunks
constexpr int kEncMaxChunk = 16384;  // encode_layout never makes a longer chunk
constexpr int kEncCtasPerSm = 3;     // both chunk kernels are built for 3 CTAs per SM

// Shared memory of one CTA: a codes chunk's per-thread cluster sums
// (bins[16][256] as fp32 pairs, counts[8][256]).
constexpr size_t kEncSmem = kClusters * kEncThreads * 16 + kClusters / 2 * kEncThreads * 4;

// ---------------------------------------------------------------------------
// Exact channel sums of bf16 keys.
//
// A bf16 value v with 2^-20 <= |v| < 2^17 has 8 significant bits and an
// exponent of at least -20, so it is an integer multiple of 2^-27.  A sum of
// at most 2^9 such values is below 2^26 in magnitude, so every partial sum is
// an integer multiple of 2^-27 below 2^53 * 2^-27: plain fp64 additions of
// them are exact.  Each lane adds its fast accumulators into its
// double-double slots after at most 264 values.  A load (two rows of a warp)
// in which any lane sees a value outside the window (zero, subnormal, tiny,
// huge, inf or nan) is added by two-sums into the lane's double-double
// accumulator instead.  The result is the exact sum either way.
// ---------------------------------------------------------------------------

// Window edges as 15-bit bf16 magnitudes (exponent and mantissa fields):
// 2^-20 has exponent field 107, 2^17 has 144.
constexpr uint32_t kWinLoBits = 107u << 7, kWinHiBits = 144u << 7;
constexpr int kMeanG = 8;          // 16-byte loads in flight per thread

__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// True when all eight bf16 values of w lie in the window.  A magnitude's
// bit pattern orders like the magnitude; nan and inf patterns lie above
// the window, zero and subnormals below it.
__device__ __forceinline__ bool in_window8(const uint4 &w) {
    const uint32_t a = w.x & 0x7FFF7FFFu, b = w.y & 0x7FFF7FFFu, c = w.z & 0x7FFF7FFFu, d = w.w & 0x7FFF7FFFu;
    const uint32_t lo = min_u16x2(min_u16x2(a, b), min_u16x2(c, d));
    const uint32_t hi = max_u16x2(max_u16x2(a, b), max_u16x2(c, d));
    const uint32_t lo1 = min(lo & 0xFFFFu, lo >> 16), hi1 = max(hi & 0xFFFFu, hi >> 16);
    return lo1 >= kWinLoBits && hi1 < kWinHiBits;
}

// Two-sum addition of one load's eight values into a lane's slots (channel
// 8 cg + i at slot[16 i]).  Out of line: the path is rare and its registers
// should not count against the fast loop's.
__device__ __noinline__ void slow_add8(dd *slot, uint4 w) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        dd_add_double(slot[16 * (2 * i)], static_cast<double>(bf16_lo(x[i])));
        dd_add_double(slot[16 * (2 * i + 1)], static_cast<double>(bf16_hi(x[i])));
    }
}

// Channel sums of rows [t0, t1) of a bf16 segment into part[D].  Lane l of a
// warp reads channels 8 (l & 15) .. 8 (l & 15) + 7 of row pair member l >> 4;
// a warp covers two consecutive rows per load, the CTA 16.  The loads run a
// group ahead: load u of the next group is issued as soon as load u of the
// current one has been added, so kMeanG loads stay in flight.  `red` holds
// one double-double slot per (warp, row half, channel), channel 8 cg + i at
// [i][cg] so that a warp's accesses fall in distinct banks.
__device__ __forceinline__ void mean_chunk_bf16(const uint4 *seg_rows, int t0, int t1, dd (*red)[2][8][16],
                                                double2 *part) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = lane >> 4, cg = lane & 15;
    const uint4 *rows = seg_rows + cg;
    dd *slot = &red[warp][half][0][cg];
#pragma unroll
    for (int i = 0; i < 8; ++i) slot[16 * i] = dd{0.0, 0.0};
    double fast[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) fast[i] = 0.0;

    constexpr int kStride = 2 * kEncWarps;            // rows per CTA load round
    constexpr int kGroup = kMeanG * kStride;          // rows per CTA group
    const int my = 2 * warp + half;
    auto row = [&](int t) { return __ldg(rows + static_cast<size_t>(t) * (kHeadDim / 8)); };
    int tb = t0;
    uint4 w[kMeanG];
    if (tb + kGroup <= t1) {
#pragma unroll
        for (int u = 0; u < kMeanG; ++u) w[u] = row(tb + u * kStride + my);
    }
    int since_flush = 0;
    for (; tb + kGroup <= t1; tb += kGroup) {
        if (++since_flush > 32) {                     // at most 32 * kMeanG values per fast accumulator
            since_flush = 1;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                dd_add_double(slot[16 * i], fast[i]);
                fast[i] = 0.0;
            }
        }
        const bool next = tb + 2 * kGroup <= t1;      // uniform over the CTA
#pragma unroll
        for (int u = 0; u < kMeanG; ++u) {
            const uint4 x = w[u];
            if (next) w[u] = row(tb + kGroup + u * kStride + my);
            if (__all_sync(0xffffffffu, in_window8(x))) {
                const uint32_t v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    fast[2 * i] += static_cast<double>(bf16_lo(v[i]));
                    fast[2 * i + 1] += static_cast<double>(bf16_hi(v[i]));
                }
            } else {
                slow_add8(slot, x);
            }
        }
    }
    // the ragged end, one CTA round (16 rows) at a time
    for (; tb < t1; tb += kStride) {
        const int t = tb + my;
        const bool have = t < t1;
        const uint4 x = have ? row(t) : make_uint4(0u, 0u, 0u, 0u);
        if (__all_sync(0xffffffffu, !have || in_window8(x))) {
            if (have) {
                const uint32_t v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    fast[2 * i] += static_cast<double>(bf16_lo(v[i]));
                    fast[2 * i + 1] += static_cast<double>(bf16_hi(v[i]));
                }
            }
        } else if (have) {
            slow_add8(slot, x);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) dd_add_double(slot[16 * i], fast[i]);
    __syncthreads();
    if (tid < kHeadDim) {
        const int i = tid & 7, g = tid >> 3;
        dd s = red[0][0][i][g];
        s = dd_add(s, red[0][1][i][g]);
#pragma unroll
        for (int w2 = 1; w2 < kEncWarps; ++w2) {
            s = dd_add(s, red[w2][0][i][g]);
            s = dd_add(s, red[w2][1][i][g]);
        }
        part[tid] = make_double2(s.hi, s.lo);
    }
}

// fp32 keys: every element through a double-double two-sum; `red` is
// [8 warps][D] double-double.
__device__ __forceinline__ void mean_chunk_f32(const float *seg_rows, int t0, int t1, dd (*red)[kHeadDim],
                                               double2 *part) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4 *rows = reinterpret_cast<const float4 *>(seg_rows) + lane;
    dd acc[4] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
    int t = t0 + warp;
    for (; t + (kEncUnroll - 1) * kEncWarps < t1; t += kEncUnroll * kEncWarps) {
        float4 v[kEncUnroll];
#pragma unroll
        for (int u = 0; u < kEncUnroll; ++u) v[u] = __ldg(rows + static_cast<size_t>(t + u * kEncWarps) * 32);
#pragma unroll
        for (int u = 0; u < kEncUnroll; ++u) {
            dd_add_double(acc[0], v[u].x);
            dd_add_double(acc[1], v[u].y);
            dd_add_double(acc[2], v[u].z);
            dd_add_double(acc[3], v[u].w);
        }
    }
    for (; t < t1; t += kEncWarps) {
        const float4 v = __ldg(rows + static_cast<size_t>(t) * 32);
        dd_add_double(acc[0], v.x);
        dd_add_double(acc[1], v.y);
        dd_add_double(acc[2], v.z);
        dd_add_double(acc[3], v.w);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane * 4 + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < kHeadDim) {
        dd s = red[0][threadIdx.x];
#pragma unroll
        for (int w = 1; w < kEncWarps; ++w) s = dd_add(s, red[w][threadIdx.x]);
        part[threadIdx.x] = make_double2(s.hi, s.lo);
    }
}

// Four consecutive channels of a key row as loaded (8 bytes of bf16, 16 of
// fp32).
template <int DT>
struct KeyQuad;
template <>
struct KeyQuad<SIKV_DTYPE_BF16> {
    using raw = uint2;
    static constexpr int kRows = 8;      // rows per load buffer (two buffers in flight)
};
template <>
struct KeyQuad<SIKV_DTYPE_F32> {
    using raw = uint4;
    static constexpr int kRows = 4;
};

__device__ __forceinline__ unsigned long long pair_bits(float lo, float hi) {
    return static_cast<unsigned long long>(__float_as_uint(lo)) |
           (static_cast<unsigned long long>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ unsigned long long sub_f32x2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long add_f32x2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The smallest bf16 value >= m, as bits.  For a bf16 key v, v >= m exactly
// when v >= this ceiling, so the sign decisions can be taken on bf16 pairs.
__device__ __forceinline__ uint32_t bf16_ceil_bits(float m) {
    const uint32_t u = __float_as_uint(m);
    if ((u & 0xFFFFu) == 0u) return u >> 16;                 // representable (zeros and infinities too)
    return (u >> 16) + ((u >> 31) ? 0u : 1u);                 // negative: truncation rounds up
}

// Per token and lane: the 4-bit sign pattern j of (k - mu) over channels
// 4 lane .. 4 lane + 3 (bit i for channel 4 lane + i, k >= mu), and the four
// differences k - mu in fp32, as two lane pairs.
template <int DT>
struct SignCoder;
template <>
struct SignCoder<SIKV_DTYPE_BF16> {
    unsigned long long m01, m23;      // mu pairs
    __nv_bfloat162 c01, c23;          // bf16 ceilings of mu
    __device__ explicit SignCoder(float4 m) : m01(pair_bits(m.x, m.y)), m23(pair_bits(m.z, m.w)) {
        const uint32_t a = bf16_ceil_bits(m.x) | (bf16_ceil_bits(m.y) << 16);
        const uint32_t b = bf16_ceil_bits(m.z) | (bf16_ceil_bits(m.w) << 16);
        c01 = *reinterpret_cast<const __nv_bfloat162 *>(&a);
        c23 = *reinterpret_cast<const __nv_bfloat162 *>(&b);
    }
    __device__ int code(uint2 w) const {
        const uint32_t g01 = __hge2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&w.x), c01);
        const uint32_t g23 = __hge2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&w.y), c23);
        const uint32_t t = (g01 & 0x00020001u) | (g23 & 0x00080004u);
        return static_cast<int>((t | (t >> 16)) & 15u);
    }
    __device__ void diff(uint2 w, unsigned long long &d01, unsigned long long &d23) const {
        d01 = sub_f32x2(pair_bits(bf16_lo(w.x), bf16_hi(w.x)), m01);
        d23 = sub_f32x2(pair_bits(bf16_lo(w.y), bf16_hi(w.y)), m23);
    }
};
template <>
struct SignCoder<SIKV_DTYPE_F32> {
    float4 m;
    __device__ explicit SignCoder(float4 m_) : m(m_) {}
    __device__ int code(uint4 w) const {
        return (__uint_as_float(w.x) >= m.x ? 1 : 0) | (__uint_as_float(w.y) >= m.y ? 2 : 0) |
               (__uint_as_float(w.z) >= m.z ? 4 : 0) | (__uint_as_float(w.w) >= m.w ? 8 : 0);
    }
    __device__ void diff(uint4 w, unsigned long long &d01, unsigned long long &d23) const {
        d01 = sub_f32x2(pair_bits(__uint_as_float(w.x), __uint_as_float(w.y)), pair_bits(m.x, m.y));
        d23 = sub_f32x2(pair_bits(__uint_as_float(w.z), __uint_as_float(w.w)), pair_bits(m.z, m.w));
    }
};

// Codes of rows [t0, t1) of a segment and the chunk's cluster sums.  Thread
// (warp w, lane s) owns subspace s: channels 4s..4s+3 of every row the warp
// visits.  Its cluster sums live in shared memory, private to the thread:
// bins[j][thread] (two fp32 pairs) and cnt[j / 2][thread] (two 16-bit counts
// per word: a thread sees at most kEncMaxChunk / 8 = 2048 rows), laid out so
// that a warp's accesses hit distinct banks whatever the codes are.  Row
// loads are double-buffered: the next buffer of rows is requested before the
// current one is consumed.  The counts are added with shared-memory
// reductions, which need no read-back.  cbp / cnp:
// the chunk's [P][16] partials.
template <int DT>
__device__ __forceinline__ void codes_chunk(const void *seg_K, uint8_t *seg_codes, const float *seg_mu, int t0,
                                            int t1, int num_sinks, float4 *smem, double *cbp, int32_t *cnp) {
    using Q = KeyQuad<DT>;
    using R = typename Q::raw;
    constexpr int U = Q::kRows;
    ulonglong2 *bins = reinterpret_cast<ulonglong2 *>(smem);                           // [16][256]
    uint32_t *cnt = reinterpret_cast<uint32_t *>(smem + kClusters * kEncThreads);       // [8][256]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const R *rows = static_cast<const R *>(seg_K) + lane;
    uint8_t *crow = seg_codes + (lane >> 1);
    const SignCoder<DT> sc(__ldcg(reinterpret_cast<const float4 *>(seg_mu) + lane));

#pragma unroll
    for (int j = 0; j < kClusters; ++j) bins[j * kEncThreads + tid] = make_ulonglong2(0ull, 0ull);
#pragma unroll
    for (int j = 0; j < kClusters / 2; ++j) cnt[j * kEncThreads + tid] = 0u;
    __syncthreads();

    auto put_code = [&](int t, int j) {
        const int jn = __shfl_down_sync(0xffffffffu, j, 1);
        if (!(lane & 1)) crow[static_cast<size_t>(t) * kCodeBytes] = static_cast<uint8_t>(j | (jn << 4));
    };
    auto consume = [&](int t, R w) {
        const int j = sc.code(w);
        put_code(t, j);
        unsigned long long d01, d23;
        sc.diff(w, d01, d23);
        ulonglong2 *bp = bins + j * kEncThreads + tid;
        ulonglong2 a = *bp;
        a.x = add_f32x2(a.x, d01);
        a.y = add_f32x2(a.y, d23);
        *bp = a;
        atomicAdd(cnt + (j >> 1) * kEncThreads + tid, 1u << ((j & 1) * 16));
    };
    auto load = [&](R (&buf)[U], int tb) {
#pragma unroll
        for (int u = 0; u < U; ++u) buf[u] = __ldg(rows + static_cast<size_t>(tb + u * kEncWarps) * kSubspaces);
    };
    auto consume_all = [&](const R (&buf)[U], int tb) {
#pragma unroll
        for (int u = 0; u < U; ++u) consume(tb + u * kEncWarps, buf[u]);
    };

    // sink rows: codes only
    const int ts = max(t0, min(num_sinks, t1));
    for (int t = t0 + warp; t < ts; t += kEncWarps) put_code(t, sc.code(__ldg(rows + static_cast<size_t>(t) * kSubspaces)));
    // this warp's rows: ts + warp + 8 i
    constexpr int kSpan = U * kEncWarps;
    R a[U], b[U];
    int tb = ts + warp;
    bool have_a = tb + (U - 1) * kEncWarps < t1;
    if (have_a) load(a, tb);
    while (have_a) {
        const int tn = tb + kSpan;
        const bool have_b = tn + (U - 1) * kEncWarps < t1;
        if (have_b) load(b, tn);
        consume_all(a, tb);
        tb = tn;
        if (!have_b) break;
        const int tm = tb + kSpan;
        have_a = tm + (U - 1) * kEncWarps < t1;
        if (have_a) load(a, tm);
        consume_all(b, tb);
        tb = tm;
    }
    for (int t = tb; t < t1; t += kEncWarps) consume(t, __ldg(rows + static_cast<size_t>(t) * kSubspaces));
    __syncthreads();

    // Reduce the 8 warps' bins of each (subspace, cluster) in a fixed order.
    for (int pr = tid; pr < kSubspaces * kClusters; pr += kEncThreads) {
        const int j = pr >> 5, s = pr & 31;
        double sx = 0.0, sy = 0.0, sz = 0.0, sw = 0.0;
        uint32_t n = 0;
#pragma unroll
        for (int w = 0; w < kEncWarps; ++w) {
            const float4 a4 = smem[j * kEncThreads + w * 32 + s];
            sx += a4.x;
            sy += a4.y;
            sz += a4.z;
            sw += a4.w;
            n += (cnt[(j >> 1) * kEncThreads + w * 32 + s] >> ((j & 1) * 16)) & 0xFFFFu;
        }
        const int o = s * kClusters + j;
        reinterpret_cast<double4 *>(cbp)[o] = make_double4(sx, sy, sz, sw);
        cnp[o] = static_cast<int32_t>(n);
    }
}

// mu of each segment from its chunks' exact sums: a fixed-order
// double-double sum over the chunks that hold tokens, one correctly rounded
// division.
__global__ void __launch_bounds__(kHeadDim)
enc_mean_final(const double2 *__restrict__ part, const int32_t *__restrict__ seq_lens, int hkv, int nmax,
               int num_sinks, int chunk, int nchunks, float *__restrict__ mu, int32_t *status) {
    const int seg = blockIdx.x, ch = threadIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int n = max(n_tok - num_sinks, 0);
    float m = 0.0f;
    if (n > 0) {
        const int used = min((n_tok + chunk - 1) / chunk, nchunks);
        dd s = {0.0, 0.0};
        for (int c = 0; c < used; ++c) {
            const double2 p = part[(static_cast<size_t>(seg) * nchunks + c) * kHeadDim + ch];
            s = dd_add(s, dd{p.x, p.y});
        }
        m = dd_div_to_float_rn(s, static_cast<double>(n));
    }
    mu[static_cast<size_t>(seg) * kHeadDim + ch] = m;
}

// Channel sums of chunk blockIdx.x of segment blockIdx.y (rows past the
// sinks only).
template <int DT>
__global__ void __launch_bounds__(kEncThreads, kEncCtasPerSm)
enc_mean_partial(const void *__restrict__ K, const int32_t *__restrict__ seq_lens, int hkv, int nmax,
                 int num_sinks, int chunk, int nchunks, double2 *__restrict__ part, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    __shared__ dd red[DT == SIKV_DTYPE_BF16 ? kEncWarps * 2 * kHeadDim : kEncWarps * kHeadDim];
    const int seg = blockIdx.y, c = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int t0 = max(c * chunk, num_sinks), t1 = min((c + 1) * chunk, n_tok);
    const char *segK = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    double2 *out = part + (static_cast<size_t>(seg) * nchunks + c) * kHeadDim;
    if (DT == SIKV_DTYPE_BF16)
        mean_chunk_bf16(reinterpret_cast<const uint4 *>(segK), t0, t1, reinterpret_cast<dd(*)[2][8][16]>(red), out);
    else
        mean_chunk_f32(reinterpret_cast<const float *>(segK), t0, t1, reinterpret_cast<dd(*)[kHeadDim]>(red), out);
}

// Codes and cluster partials of chunk blockIdx.x of segment blockIdx.y.
template <int DT>
__global__ void __launch_bounds__(kEncThreads, kEncCtasPerSm)
enc_codes_partial(const void *__restrict__ K, const int32_t *__restrict__ seq_lens, const float *__restrict__ mu,
                  int hkv, int nmax, int num_sinks, int chunk, int nchunks, uint8_t *__restrict__ codes,
                  double *__restrict__ cb_part, int32_t *__restrict__ cnt_part, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    extern __shared__ float4 enc_smem[];
    const int seg = blockIdx.y, c = blockIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int t0 = c * chunk, t1 = min((c + 1) * chunk, n_tok);
    const size_t seg_rows = static_cast<size_t>(seg) * nmax;
    const size_t pc = (static_cast<size_t>(seg) * nchunks + c) * kSubspaces * kClusters;
    codes_chunk<DT>(static_cast<const char *>(K) + seg_rows * kHeadDim * EB, codes + seg_rows * kCodeBytes,
                    mu + static_cast<size_t>(seg) * kHeadDim, t0, t1, num_sinks, enc_smem, cb_part + 4 * pc,
                    cnt_part + pc);
}

// Centroids and counts of each segment from its chunks' partials, summed over
// the chunks in order; thread pr = s * 16 + j.
__global__ void __launch_bounds__(kSubspaces * kClusters)
enc_codebook_final(const double *__restrict__ cb_part, const int32_t *__restrict__ cnt_part,
                   const int32_t *__restrict__ seq_lens, int hkv, int nmax, int chunk, int nchunks,
                   float *__restrict__ codebook, int32_t *__restrict__ counts, int32_t *status) {
    const int seg = blockIdx.x, pr = threadIdx.x;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const int used = min((n_tok + chunk - 1) / chunk, nchunks);
    double sx = 0.0, sy = 0.0, sz = 0.0, sw = 0.0;
    long long n = 0;
    for (int c = 0; c < used; ++c) {
        const size_t o = (static_cast<size_t>(seg) * nchunks + c) * kSubspaces * kClusters + pr;
        const double4 a = reinterpret_cast<const double4 *>(cb_part)[o];
        sx += a.x;
        sy += a.y;
        sz += a.z;
        sw += a.w;
        n += cnt_part[o];
    }
    float4 cv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n > 0) {
        const double dn = static_cast<double>(n);
        cv = make_float4(__double2float_rn(sx / dn), __double2float_rn(sy / dn), __double2float_rn(sz / dn),
                         __double2float_rn(sw / dn));
    }
    reinterpret_cast<float4 *>(codebook)[static_cast<size_t>(seg) * kSubspaces * kClusters + pr] = cv;
    if (counts) counts[static_cast<size_t>(seg) * kSubspaces * kClusters + pr] = static_cast<int32_t>(n);
}

static_assert(kClusters * kEncThreads * sizeof(ulonglong2) + kClusters / 2 * kEncThreads * sizeof(uint32_t) <= kEncSmem,
              "cluster sums and counts fit the codes kernel's shared memory");

}  // namespace

// Chunk length: a multiple of 256 tokens, at most kEncMaxChunk, chosen so
// that the chunk CTAs fill whole waves of the device (kEncCtasPerSm CTAs on
// each of `num_sms` SMs).  The estimate of a launch's time is its number of
// waves times the rows of one chunk plus a fixed cost of 512 rows per CTA;
// the cheapest chunk wins, the longer one on a tie.  Without a device
// (num_sms == 0) the chunk is Nmax / 16, clamped to [256, 4096].
EncodeLayout encode_layout(const sikv_params &p, int num_sms) {
    EncodeLayout L;
    const int nmax = std::max(p.max_seq_len, 1);
    const long long segs = static_cast<long long>(p.batch) * p.num_kv_heads;
    int chunk = 0;
    if (num_sms > 0 && segs > 0) {
        const long long slots = static_cast<long long>(kEncCtasPerSm) * num_sms;
        long long best = -1;
        for (int n = 1; n <= (nmax + 255) / 256; ++n) {
            const int ch = ((nmax + n - 1) / n + 255) / 256 * 256;
            if (ch > kEncMaxChunk) continue;
            const long long nn = (nmax + ch - 1) / ch;
            const long long cost = (segs * nn + slots - 1) / slots * (ch + 512);
            if (best < 0 || cost < best) {
                best = cost;
                chunk = ch;
            }
        }
    }
    if (chunk == 0) {
        chunk = (nmax + 15) / 16;
        chunk = (chunk + 255) / 256 * 256;
        chunk = chunk < 256 ? 256 : (chunk > 4096 ? 4096 : chunk);
    }
    L.chunk = chunk;
    L.nchunks = (nmax + chunk - 1) / chunk;
    size_t off = kHeaderBytes;
    L.mean_part = off;
    off = align_up(off + static_cast<size_t>(segs) * L.nchunks * kHeadDim * sizeof(double2), 256);
    L.cb_part = off;
    off = align_up(off + static_cast<size_t>(segs) * L.nchunks * kSubspaces * kClusters * 4 * sizeof(double), 256);
    L.cnt_part = off;
    off = align_up(off + static_cast<size_t>(segs) * L.nchunks * kSubspaces * kClusters * sizeof(int32_t), 256);
    L.total = off;
    return L;
}

sikv_status launch_encode(const sikv_params &p, const EncodeLayout &L, const void *K, const int32_t *seq_lens,
                          float *mu, uint8_t *codes, float *codebook, int32_t *counts, char *ws,
                          cudaStream_t stream) {
    if (L.chunk > kEncMaxChunk || L.chunk < 1) return SIKV_ERR_UNSUPPORTED;
    const int segs = p.batch * p.num_kv_heads;
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    double2 *mean_part = reinterpret_cast<double2 *>(ws + L.mean_part);
    double *cb_part = reinterpret_cast<double *>(ws + L.cb_part);
    int32_t *cnt_part = reinterpret_cast<int32_t *>(ws + L.cnt_part);
    const dim3 grid(L.nchunks, segs);
    const int hkv = p.num_kv_heads, nmax = p.max_seq_len, S = p.num_sinks;
    if (p.dtype == SIKV_DTYPE_BF16) {
        enc_mean_partial<SIKV_DTYPE_BF16><<<grid, kEncThreads, 0, stream>>>(K, seq_lens, hkv, nmax, S, L.chunk,
                                                                             L.nchunks, mean_part, status);
    } else {
        enc_mean_partial<SIKV_DTYPE_F32><<<grid, kEncThreads, 0, stream>>>(K, seq_lens, hkv, nmax, S, L.chunk,
                                                                            L.nchunks, mean_part, status);
    }
    enc_mean_final<<<segs, kHeadDim, 0, stream>>>(mean_part, seq_lens, hkv, nmax, S, L.chunk, L.nchunks, mu, status);
    auto kern = p.dtype == SIKV_DTYPE_BF16 ? enc_codes_partial<SIKV_DTYPE_BF16> : enc_codes_partial<SIKV_DTYPE_F32>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kEncSmem)) !=
        cudaSuccess)
        return SIKV_ERR_CUDA;
    kern<<<grid, kEncThreads, kEncSmem, stream>>>(K, seq_lens, mu, hkv, nmax, S, L.chunk, L.nchunks, codes, cb_part,
                                                  cnt_part, status);
    enc_codebook_final<<<segs, kSubspaces * kClusters, 0, stream>>>(cb_part, cnt_part, seq_lens, hkv, nmax, L.chunk,
                                                                     L.nchunks, codebook, counts, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
