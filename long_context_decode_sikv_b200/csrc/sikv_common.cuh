// Shared device helpers of libsikv (sm_100a).
//
// Method: "Self-Indexing KVCache: Predicting Sparse Attention from Compressed
// Keys" (gist.science summary of paper 2603.14224), technical summary §2.1.
#pragma once

#include <cuda_fp16.h>

#include <cuda_runtime.h>
#include <stdint.h>

#include "sikv.h"

namespace sikv {

constexpr int kHeadDim = 128;      // D: the only supported head dimension
constexpr int kSubDim = 4;         // §2.1 item 1: 4-dim sub-vectors
constexpr int kSubspaces = 32;     // P = D / 4
constexpr int kClusters = 16;      // 2^4 sign patterns per sub-vector
constexpr int kCodeBytes = 16;     // D / 8: two 4-bit codes per byte
constexpr int kMaxGroup = 8;       // query heads per KV head handled by the kernels
constexpr size_t kHeaderBytes = 256;

// Workspace header at offset 0 of every workspace.
struct WsHeader {
    int32_t status;       // sticky SIKV_DEVERR_* bits
    int32_t pad[63];
};

__device__ __forceinline__ void flag_error(int32_t *status, int32_t bits) {
    atomicOr(status, bits);
}

// Reads a KV sequence length and validates it; -1 when invalid.
__device__ __forceinline__ int load_seq_len(const int32_t *seq_lens, int b, int nmax,
                                            int32_t *status) {
    int n = __ldg(seq_lens + b);
    if (n < 0 || n > nmax) {
        flag_error(status, SIKV_DEVERR_SEQ_LEN);
        return -1;
    }
    return n;
}

// Reads k_b and validates it against kmax and the number of scored tokens.
__device__ __forceinline__ int load_topk(const int32_t *k_per_seq, int b, int kmax, int scored,
                                         int32_t *status) {
    int k = __ldg(k_per_seq + b);
    if (k < 0 || k > kmax || k > scored) {
        flag_error(status, SIKV_DEVERR_TOPK);
        return -1;
    }
    return k;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round-to-nearest-even fp32 -> bf16 bits (inputs are finite).
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

// Four consecutive elements of a dtype row as floats.  `row` points at the
// row start; `c` is the first element index (a multiple of 4).
template <int DT>
__device__ __forceinline__ float4 load4(const void *row, int c);

template <>
__device__ __forceinline__ float4 load4<SIKV_DTYPE_F32>(const void *row, int c) {
    return __ldg(reinterpret_cast<const float4 *>(row) + (c >> 2));
}

template <>
__device__ __forceinline__ float4 load4<SIKV_DTYPE_BF16>(const void *row, int c) {
    uint2 w = __ldg(reinterpret_cast<const uint2 *>(row) + (c >> 2));
    return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}

template <int DT>
__device__ __forceinline__ float load1(const void *row, int c);

template <>
__device__ __forceinline__ float load1<SIKV_DTYPE_F32>(const void *row, int c) {
    return __ldg(reinterpret_cast<const float *>(row) + c);
}

template <>
__device__ __forceinline__ float load1<SIKV_DTYPE_BF16>(const void *row, int c) {
    unsigned short h = __ldg(reinterpret_cast<const unsigned short *>(row) + c);
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

template <int DT>
struct ElemBytes;
template <>
struct ElemBytes<SIKV_DTYPE_F32> { static constexpr int value = 4; };
template <>
struct ElemBytes<SIKV_DTYPE_BF16> { static constexpr int value = 2; };

// Order-preserving map of a finite fp32 score to uint32 (larger score ->
// larger key); -0.0 is mapped like +0.0 so that the two compare equal.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// double-double helpers (error-free transformations)
// ---------------------------------------------------------------------------

struct dd {
    double hi, lo;
};

__device__ __forceinline__ dd two_sum(double a, double b) {
    double s = a + b;
    double bb = s - a;
    double err = (a - (s - bb)) + (b - bb);
    return {s, err};
}

__device__ __forceinline__ dd fast_two_sum(double a, double b) {   // |a| >= |b| or a == 0
    double s = a + b;
    return {s, b - (s - a)};
}

__device__ __forceinline__ void dd_add_double(dd &acc, double x) {
    dd t = two_sum(acc.hi, x);
    acc.hi = t.hi;
    acc.lo += t.lo;
}

__device__ __forceinline__ dd dd_add(dd a, dd b) {
    dd s = two_sum(a.hi, b.hi);
    double e = s.lo + (a.lo + b.lo);
    return fast_two_sum(s.hi, e);
}

// Correctly rounded fp32 value of the normalized pair hi + lo
// (|lo| <= ulp(hi) / 2).  Only an hi exactly halfway between two fp32
// neighbours needs lo to pick the side.
__device__ __forceinline__ float dd_to_float_rn(double hi, double lo) {
    float f = __double2float_rn(hi);
    double fd = static_cast<double>(f);
    double diff = hi - fd;                         // exact
    if (diff == 0.0 || lo == 0.0) return f;
    float f2 = nextafterf(f, diff > 0.0 ? INFINITY : -INFINITY);
    double half = (static_cast<double>(f2) - fd) * 0.5;   // exact, signed like diff
    if (diff == half && ((lo > 0.0) == (diff > 0.0))) return f2;
    return f;
}

// Correctly rounded fp32 of (hi + lo) / n for an exact pair and n >= 1.
__device__ __forceinline__ float dd_div_to_float_rn(dd s, double n) {
    double qh = s.hi / n;
    double r = fma(-qh, n, s.hi);                  // exact remainder
    double ql = (r + s.lo) / n;
    dd q = fast_two_sum(qh, ql);
    return dd_to_float_rn(q.hi, q.lo);
}

// ---------------------------------------------------------------------------
// 2-bit value rows: 32 bytes of levels (dimension d in bits 2 (d mod 4) of
// byte d / 4), then the (min, step) fp16 pairs of the four 32-channel groups
// ---------------------------------------------------------------------------

constexpr int kVqRowBytes = 48;
constexpr int kVqGroup = 32;

// Dimensions 4 lane .. 4 lane + 3 of a quantized row: min + level * step.
__device__ __forceinline__ float4 vq_decode4(const uint8_t *row, int lane) {
    const uint32_t lv = row[lane];
    const uint32_t ms = *reinterpret_cast<const uint32_t *>(row + 32 + 4 * (lane >> 3));
    const float m = __half2float(__ushort_as_half(static_cast<unsigned short>(ms & 0xFFFFu)));
    const float st = __half2float(__ushort_as_half(static_cast<unsigned short>(ms >> 16)));
    return make_float4(fmaf(static_cast<float>(lv & 3u), st, m), fmaf(static_cast<float>((lv >> 2) & 3u), st, m),
                       fmaf(static_cast<float>((lv >> 4) & 3u), st, m), fmaf(static_cast<float>(lv >> 6), st, m));
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace sikv
