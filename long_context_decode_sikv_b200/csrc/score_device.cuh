// LUT-GEMV scoring in the compressed domain, device side.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 2: the query is split into 4-dim sub-queries,
// each is dotted with the 16 centroids of its subspace to form a lookup
// table, and a token's score is the sum of the entries its codes select.
//
// B200 layout of the table.  Two subspaces share a code byte, so the 32
// per-subspace tables are merged into 16 byte-indexed tables
//   T2[m][b] = LUT[2m][b & 15] + LUT[2m+1][b >> 4],   m = byte position,
// which halves the lookups to 16 per token.  A warp scores 32 consecutive
// tokens, one per lane; at step i lane l reads byte (l + i) mod 16 of its
// code row (the row is rotated in registers by l mod 16 bytes first) and looks
// it up in shared word  b * 64 + l + i,  which holds T2[(l + i) mod 16][b].
// Word l + i sits in bank (l + i) mod 32, distinct for the 32 lanes whatever
// the code bytes are, so every lookup is one conflict-free wavefront.  The
// byte address (b << 8) | 4l comes out of a single byte-permute, and 4i is a
// constant offset: one PRMT + one LDS + one FADD per lookup.  The sum order
// (two chains over steps 0-7 and 8-15, then q_bar.mu) is fixed by t mod 16, so
// a token's fp32 score does not depend on which kernel or CTA computes it.
#pragma once

#include "sikv_common.cuh"

namespace sikv {

constexpr int kT2RowWords = 64;                    // words per byte value (48 used)
constexpr int kT2Words = 256 * kT2RowWords;        // 64 KB

struct ScoreTables {
    float t2[kT2Words];                // byte-indexed merged tables
    float qbar[kHeadDim];              // summed group query
    float lutT[kClusters * kSubspaces];// LUT[s][j] stored j-major: lutT[j * 32 + s]
    float qmu;                         // q_bar . mu
    float pad[3];
};

constexpr int kTableThreads = 256;      // CTA size of every kernel that builds the tables

// One thread's share (of NT threads) of the inputs of the tables of segment
// (b, h): the group's query rows (as fp32), the segment's codebook (512
// float4) and its channel means (128).  load() issues every global load at once; store()
// writes them to shared memory (qs: group x 128, cbs, mus), so that other
// work can be issued in between.
template <int DT, int NT = kTableThreads>
struct TableInputs {
    static constexpr int kQ = kMaxGroup * kHeadDim / NT;             // 4 (256 threads) or 2 (512)
    static constexpr int kCb = kSubspaces * kClusters / NT;          // 2 or 1
    float qv[kQ];
    float4 cv[kCb];
    float mv;

    __device__ __forceinline__ void load(const void *__restrict__ q, const float *__restrict__ codebook,
                                         const float *__restrict__ mu, int b, int h, int hq, int group, int seg) {
        constexpr int EB = ElemBytes<DT>::value;
        const int tid = threadIdx.x;
        const char *qrow = static_cast<const char *>(q) +
                           (static_cast<size_t>(b) * hq + static_cast<size_t>(h) * group) * kHeadDim * EB;
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
            const int e = tid + NT * i;
            qv[i] = (e < group * kHeadDim) ? load1<DT>(qrow, e) : 0.f;
        }
        const float4 *cb = reinterpret_cast<const float4 *>(codebook) + static_cast<size_t>(seg) * kSubspaces * kClusters;
#pragma unroll
        for (int i = 0; i < kCb; ++i) cv[i] = __ldg(cb + tid + NT * i);
        mv = (tid < kHeadDim) ? __ldg(mu + static_cast<size_t>(seg) * kHeadDim + tid) : 0.f;
    }

    __device__ __forceinline__ void store(float *qs, float4 *cbs, float *mus, int group) const {
        const int tid = threadIdx.x;
#pragma unroll
        for (int i = 0; i < kQ; ++i) {
            const int e = tid + NT * i;
            if (e < group * kHeadDim) qs[e] = qv[i];
        }
#pragma unroll
        for (int i = 0; i < kCb; ++i) cbs[tid + NT * i] = cv[i];
        if (tid < kHeadDim) mus[tid] = mv;
    }
};

// Builds q_bar, LUT, q_bar.mu and T2 from staged inputs with the whole CTA.
// Expects the staged inputs to be visible (a __syncthreads() after staging);
// ends with a __syncthreads().
template <int NT = kTableThreads>
__device__ __forceinline__ void build_score_tables(ScoreTables &sh, const float *qs, const float4 *cbs,
                                                   const float *mus, int group) {
    constexpr int nt = NT;
    const int tid = threadIdx.x;
    for (int c = tid; c < kHeadDim; c += nt) {
        float acc = qs[c];
        for (int g = 1; g < group; ++g) acc += qs[g * kHeadDim + c];
        sh.qbar[c] = acc;
    }
    __syncthreads();
    for (int e = tid; e < kSubspaces * kClusters; e += nt) {
        const int j = e >> 5, s = e & 31;
        const float4 c4 = cbs[s * kClusters + j];
        float v = sh.qbar[4 * s] * c4.x;
        v = fmaf(sh.qbar[4 * s + 1], c4.y, v);
        v = fmaf(sh.qbar[4 * s + 2], c4.z, v);
        v = fmaf(sh.qbar[4 * s + 3], c4.w, v);
        sh.lutT[e] = v;
    }
    if (tid < 32) {
        double a = static_cast<double>(sh.qbar[4 * tid]) * mus[4 * tid];
        a = fma(static_cast<double>(sh.qbar[4 * tid + 1]), static_cast<double>(mus[4 * tid + 1]), a);
        a = fma(static_cast<double>(sh.qbar[4 * tid + 2]), static_cast<double>(mus[4 * tid + 2]), a);
        a = fma(static_cast<double>(sh.qbar[4 * tid + 3]), static_cast<double>(mus[4 * tid + 3]), a);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (tid == 0) sh.qmu = static_cast<float>(a);
    }
    __syncthreads();
    // One byte value per warp and iteration: lane (m, copy) with m = lane & 15
    // reads lutT[j * 32 + 2m (+1)] (distinct banks, pairs broadcast) and stores
    // word m + 16 copy (32 distinct banks), then lanes 0..15 store word m + 32.
    {
        const int lane = tid & 31, m = lane & 15, copy = lane >> 4;
#pragma unroll 2
        for (int byte = tid >> 5; byte < 256; byte += nt >> 5) {
            const float v = sh.lutT[(byte & 15) * kSubspaces + 2 * m] + sh.lutT[(byte >> 4) * kSubspaces + 2 * m + 1];
            float *row = sh.t2 + byte * kT2RowWords;
            row[m + 16 * copy] = v;
            if (copy == 0) row[m + 32] = v;
        }
    }
    __syncthreads();
}

// Score of the token whose 16-byte code row is `row`, computed by `lane`
// (the token index must be congruent to lane modulo 16).
__device__ __forceinline__ float lut2_score(const float *__restrict__ t2, uint4 row, int lane,
                                            float qmu) {
    const int r = lane & 15;
    uint32_t a0 = row.x, a1 = row.y, a2 = row.z, a3 = row.w;
    if (r & 4) {
        const uint32_t t = a0;
        a0 = a1;
        a1 = a2;
        a2 = a3;
        a3 = t;
    }
    if (r & 8) {
        uint32_t t = a0;
        a0 = a2;
        a2 = t;
        t = a1;
        a1 = a3;
        a3 = t;
    }
    const uint32_t rb = static_cast<uint32_t>(r & 3);
    const uint32_t sel = rb * 0x1111u + 0x3210u;
    const uint32_t w0 = __byte_perm(a0, a1, sel), w1 = __byte_perm(a1, a2, sel);
    const uint32_t w2 = __byte_perm(a2, a3, sel), w3 = __byte_perm(a3, a0, sel);
    const uint32_t base = 4u * static_cast<uint32_t>(lane);
    const char *tb = reinterpret_cast<const char *>(t2);
#define SIKV_LK(W, I) (*reinterpret_cast<const float *>(tb + __byte_perm((W), base, 0x6504u | (((I) & 3u) << 4)) + 4 * (I)))
    // two independent chains (steps 0-7 and 8-15) halve the add latency
    float a = SIKV_LK(w0, 0), c = SIKV_LK(w2, 8);
    a += SIKV_LK(w0, 1);
    c += SIKV_LK(w2, 9);
    a += SIKV_LK(w0, 2);
    c += SIKV_LK(w2, 10);
    a += SIKV_LK(w0, 3);
    c += SIKV_LK(w2, 11);
    a += SIKV_LK(w1, 4);
    c += SIKV_LK(w3, 12);
    a += SIKV_LK(w1, 5);
    c += SIKV_LK(w3, 13);
    a += SIKV_LK(w1, 6);
    c += SIKV_LK(w3, 14);
    a += SIKV_LK(w1, 7);
    c += SIKV_LK(w3, 15);
#undef SIKV_LK
    return (a + c) + qmu;
}

// Scores of two tokens computed by `lane` with their instructions interleaved
// (four independent addition chains).  Each result is bit-identical to
// lut2_score on the same row: same rotation, same order of additions.
__device__ __forceinline__ float2 lut2_score2(const float *__restrict__ t2, uint4 ra, uint4 rb, int lane, float qmu) {
    const int r = lane & 15;
    uint32_t a0 = ra.x, a1 = ra.y, a2 = ra.z, a3 = ra.w;
    uint32_t b0 = rb.x, b1 = rb.y, b2 = rb.z, b3 = rb.w;
    if (r & 4) {
        uint32_t t = a0;
        a0 = a1;
        a1 = a2;
        a2 = a3;
        a3 = t;
        t = b0;
        b0 = b1;
        b1 = b2;
        b2 = b3;
        b3 = t;
    }
    if (r & 8) {
        uint32_t t = a0;
        a0 = a2;
        a2 = t;
        t = a1;
        a1 = a3;
        a3 = t;
        t = b0;
        b0 = b2;
        b2 = t;
        t = b1;
        b1 = b3;
        b3 = t;
    }
    const uint32_t rb3 = static_cast<uint32_t>(r & 3);
    const uint32_t sel = rb3 * 0x1111u + 0x3210u;
    const uint32_t x0 = __byte_perm(a0, a1, sel), x1 = __byte_perm(a1, a2, sel);
    const uint32_t x2 = __byte_perm(a2, a3, sel), x3 = __byte_perm(a3, a0, sel);
    const uint32_t y0 = __byte_perm(b0, b1, sel), y1 = __byte_perm(b1, b2, sel);
    const uint32_t y2 = __byte_perm(b2, b3, sel), y3 = __byte_perm(b3, b0, sel);
    const uint32_t base = 4u * static_cast<uint32_t>(lane);
    const char *tb = reinterpret_cast<const char *>(t2);
#define SIKV_LK(W, I) (*reinterpret_cast<const float *>(tb + __byte_perm((W), base, 0x6504u | (((I) & 3u) << 4)) + 4 * (I)))
    float pa = SIKV_LK(x0, 0), qa = SIKV_LK(x2, 8), pb = SIKV_LK(y0, 0), qb = SIKV_LK(y2, 8);
    pa += SIKV_LK(x0, 1);
    qa += SIKV_LK(x2, 9);
    pb += SIKV_LK(y0, 1);
    qb += SIKV_LK(y2, 9);
    pa += SIKV_LK(x0, 2);
    qa += SIKV_LK(x2, 10);
    pb += SIKV_LK(y0, 2);
    qb += SIKV_LK(y2, 10);
    pa += SIKV_LK(x0, 3);
    qa += SIKV_LK(x2, 11);
    pb += SIKV_LK(y0, 3);
    qb += SIKV_LK(y2, 11);
    pa += SIKV_LK(x1, 4);
    qa += SIKV_LK(x3, 12);
    pb += SIKV_LK(y1, 4);
    qb += SIKV_LK(y3, 12);
    pa += SIKV_LK(x1, 5);
    qa += SIKV_LK(x3, 13);
    pb += SIKV_LK(y1, 5);
    qb += SIKV_LK(y3, 13);
    pa += SIKV_LK(x1, 6);
    qa += SIKV_LK(x3, 14);
    pb += SIKV_LK(y1, 6);
    qb += SIKV_LK(y3, 14);
    pa += SIKV_LK(x1, 7);
    qa += SIKV_LK(x3, 15);
    pb += SIKV_LK(y1, 7);
    qb += SIKV_LK(y3, 15);
#undef SIKV_LK
    return make_float2((pa + qa) + qmu, (pb + qb) + qmu);
}

}  // namespace sikv
