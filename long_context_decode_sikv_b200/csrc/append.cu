// sikv_append_codes: decode-time append of sign codes.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §2.1 item 1 (sign-based 1-bit VQ after channel-mean
// normalization) and item 3 (token-wise format).  The pages describe the
// encoding of the prefill keys only; a key that arrives during decode is
// coded the same way against the prefill mean, which stays frozen, and the
// codebook is left as it is.
//
// One warp per token: lane l reads dimensions 4l..4l+3 of the key (one
// 8- or 16-byte load), forms the 4-bit code of subspace l, and the 8 lanes of
// each group of 8 OR their nibbles into one 32-bit word of the 16-byte row.
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kAppendThreads = 256;
constexpr int kAppendWarps = kAppendThreads / 32;

template <int DT>
__global__ void __launch_bounds__(kAppendThreads)
append_codes_kernel(const void *__restrict__ K, const int32_t *__restrict__ start, const int32_t *__restrict__ count,
                    const float *__restrict__ mu, uint8_t *__restrict__ codes, int hkv, int nmax,
                    int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    const int seg = blockIdx.x, b = seg / hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = __ldg(start + b), n = __ldg(count + b);
    if (t0 < 0 || n < 0 || t0 > nmax || n > nmax - t0) {
        if (threadIdx.x == 0 && seg % hkv == 0) flag_error(status, SIKV_DEVERR_APPEND);
        return;
    }
    const float4 m4 = __ldg(reinterpret_cast<const float4 *>(mu + static_cast<size_t>(seg) * kHeadDim) + lane);
    const char *krows = static_cast<const char *>(K) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    uint4 *crows = reinterpret_cast<uint4 *>(codes) + static_cast<size_t>(seg) * nmax;
#pragma unroll 1
    for (int t = t0 + warp; t < t0 + n; t += kAppendWarps) {
        const float4 k4 = load4<DT>(krows + static_cast<size_t>(t) * kHeadDim * EB, 4 * lane);
        const uint32_t code = (k4.x >= m4.x ? 1u : 0u) | (k4.y >= m4.y ? 2u : 0u) | (k4.z >= m4.z ? 4u : 0u) |
                              (k4.w >= m4.w ? 8u : 0u);
        // subspace l is nibble (l mod 8) of word l / 8 (even subspace low)
        uint32_t word = code << (4 * (lane & 7));
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, off);
        const uint32_t w0 = __shfl_sync(0xffffffffu, word, 0), w1 = __shfl_sync(0xffffffffu, word, 8);
        const uint32_t w2 = __shfl_sync(0xffffffffu, word, 16), w3 = __shfl_sync(0xffffffffu, word, 24);
        if (lane == 0) crows[t] = make_uint4(w0, w1, w2, w3);
    }
}

}  // namespace

sikv_status launch_append(const sikv_params &p, const void *K, const int32_t *start, const int32_t *count,
                          const float *mu, uint8_t *codes, int32_t *status, cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    if (p.dtype == SIKV_DTYPE_BF16)
        append_codes_kernel<SIKV_DTYPE_BF16><<<segs, kAppendThreads, 0, stream>>>(K, start, count, mu, codes,
                                                                                  p.num_kv_heads, p.max_seq_len, status);
    else
        append_codes_kernel<SIKV_DTYPE_F32><<<segs, kAppendThreads, 0, stream>>>(K, start, count, mu, codes,
                                                                                 p.num_kv_heads, p.max_seq_len, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
