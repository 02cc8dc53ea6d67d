// sikv_quantize_values: 2-bit value rows for the selected tokens.
//
// "Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys",
// technical summary §3 and §4: accuracy is kept with 2-bit quantization and
// the memory saving matches 2-bit KIVI; the scheme is not given.  This is
// KIVI's per-token value quantization: each token's row is cut into 4 groups
// of 32 channels, a group keeps its minimum m and step s = (max - min) / 3 in
// fp16, and each value keeps the level
//     q = clamp(rint(fl32(fl32(v - m16) / s16)), 0, 3)   (0 when s16 = 0)
// that reads back as m16 + q s16.  Row layout: 32 bytes of levels (dimension
// d in bits 2 (d mod 4) of byte d / 4), then (m16, s16) of groups 0..3.
//
// One warp per token: lane l holds dimensions 4l..4l+3 (group l / 8); the
// group's minimum and maximum come from three xor-shuffles among its 8 lanes,
// and lanes 0..11 each store one 4-byte word of the 48-byte row.
#include "sikv_common.cuh"
#include "sikv_internal.h"

namespace sikv {

namespace {

constexpr int kQvThreads = 256;
constexpr int kQvWarps = kQvThreads / 32;
constexpr int kQvTokensPerWarp = 16;

template <int DT>
__global__ void __launch_bounds__(kQvThreads)
quantize_values_kernel(const void *__restrict__ V, const int32_t *__restrict__ seq_lens, uint8_t *__restrict__ vq,
                       int hkv, int nmax, int32_t *status) {
    constexpr int EB = ElemBytes<DT>::value;
    const int seg = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_tok = load_seq_len(seq_lens, seg / hkv, nmax, status);
    if (n_tok < 0) return;
    const char *vrows = static_cast<const char *>(V) + static_cast<size_t>(seg) * nmax * kHeadDim * EB;
    uint32_t *qrows = reinterpret_cast<uint32_t *>(vq + static_cast<size_t>(seg) * nmax * kVqRowBytes);
    const int tbeg = (blockIdx.x * kQvWarps + warp) * kQvTokensPerWarp;
#pragma unroll 1
    for (int t = tbeg; t < min(tbeg + kQvTokensPerWarp, n_tok); ++t) {
        const float4 v = load4<DT>(vrows + static_cast<size_t>(t) * kHeadDim * EB, 4 * lane);
        float lo = fminf(fminf(v.x, v.y), fminf(v.z, v.w)), hi = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        const __half m16 = __float2half_rn(lo), s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 3.0f));
        const float m = __half2float(m16), st = __half2float(s16);
        uint32_t byte = 0;
        if (st > 0.f) {
            const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float r = rintf(__fdiv_rn(__fsub_rn(e[i], m), st));
                byte |= static_cast<uint32_t>(fminf(fmaxf(r, 0.f), 3.f)) << (2 * i);
            }
        }
        // word w < 8: bytes 4w..4w+3 (lanes 4w..4w+3); word 8 + g: (m16, s16) of group g (lane 8g)
        const int src = 4 * (lane & 7);
        const uint32_t b0 = __shfl_sync(0xffffffffu, byte, src), b1 = __shfl_sync(0xffffffffu, byte, src + 1);
        const uint32_t b2 = __shfl_sync(0xffffffffu, byte, src + 2), b3 = __shfl_sync(0xffffffffu, byte, src + 3);
        const uint32_t prm = static_cast<uint32_t>(__half_as_ushort(m16)) |
                             (static_cast<uint32_t>(__half_as_ushort(s16)) << 16);
        const uint32_t pg = __shfl_sync(0xffffffffu, prm, 8 * (lane & 3));
        if (lane < 8) qrows[static_cast<size_t>(t) * (kVqRowBytes / 4) + lane] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        else if (lane < 12) qrows[static_cast<size_t>(t) * (kVqRowBytes / 4) + lane] = pg;
    }
}

}  // namespace

sikv_status launch_quantize_values(const sikv_params &p, const void *V, const int32_t *seq_lens, uint8_t *vq,
                                   int32_t *status, cudaStream_t stream) {
    const int segs = p.batch * p.num_kv_heads;
    const dim3 grid((p.max_seq_len + kQvWarps * kQvTokensPerWarp - 1) / (kQvWarps * kQvTokensPerWarp), segs);
    if (p.dtype == SIKV_DTYPE_BF16)
        quantize_values_kernel<SIKV_DTYPE_BF16><<<grid, kQvThreads, 0, stream>>>(V, seq_lens, vq, p.num_kv_heads,
                                                                                p.max_seq_len, status);
    else
        quantize_values_kernel<SIKV_DTYPE_F32><<<grid, kQvThreads, 0, stream>>>(V, seq_lens, vq, p.num_kv_heads,
                                                                               p.max_seq_len, status);
    return cudaGetLastError() == cudaSuccess ? SIKV_OK : SIKV_ERR_CUDA;
}

}  // namespace sikv
