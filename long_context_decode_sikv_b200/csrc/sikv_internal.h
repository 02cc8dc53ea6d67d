// Internal declarations of libsikv: workspace layouts and kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include "sikv.h"

namespace sikv {

struct EncodeLayout {
    int chunk = 0;          // tokens per CTA
    int nchunks = 0;        // chunks covering [0, Nmax)
    size_t mean_part = 0;   // double2 [segs][nchunks][D]
    size_t cb_part = 0;     // double4 [segs][nchunks][P][16]
    size_t cnt_part = 0;    // int32   [segs][nchunks][P][16]
    size_t total = 0;
};

struct TopkLayout {
    size_t total = 0;
};

struct AttnLayout {
    int split = 0;          // list positions per CTA
    int nsplit = 0;         // splits covering S + kmax positions
    size_t part_o = 0;      // float [segs][nsplit][G][D]
    size_t part_ml = 0;     // float2 [segs][nsplit][G]
    size_t total = 0;
};

struct DecodeLayout {
    size_t scores = 0;      // float [segs][Nmax]
    size_t idx = 0;         // int32 [segs][kmax]
    size_t attn = 0;        // base offset of an AttnLayout region
    AttnLayout a;
    size_t fused = 0;       // base offset of the fused kernel's coordination region
    size_t total = 0;
};

EncodeLayout encode_layout(const sikv_params &p, int num_sms);
TopkLayout topk_layout(const sikv_params &p);
AttnLayout attn_layout(const sikv_params &p, size_t base);
DecodeLayout decode_layout(const sikv_params &p);

sikv_status launch_encode(const sikv_params &p, const EncodeLayout &L, const void *K, const int32_t *seq_lens,
                          float *mu, uint8_t *codes, float *codebook, int32_t *counts, char *ws,
                          cudaStream_t stream);

// Dense comparison baselines (dense.cu).
struct DenseAttnLayout {
    int chunk = 0, nchunks = 0;
    size_t part_o = 0, part_ml = 0, total = 0;
};
DenseAttnLayout dense_attn_layout(const sikv_params &p, size_t base);
sikv_status launch_dense_score(const sikv_params &p, const void *q, const void *K, const int32_t *seq_lens,
                               float *scores, int32_t *status, cudaStream_t stream);
sikv_status launch_dense_attn(const sikv_params &p, const void *q, const void *K, const void *V,
                              const int32_t *seq_lens, void *out, char *ws, size_t base, int32_t *status,
                              cudaStream_t stream);

// K-means codebook baseline (kmeans.cu).
struct KmeansLayout {
    int chunk = 0, nchunks = 0;           // tokens per CTA, CTAs per segment
    size_t part_sum = 0, part_cnt = 0, total = 0;
};
KmeansLayout kmeans_layout(const sikv_params &p, int num_sms);
sikv_status launch_kmeans(const sikv_params &p, const KmeansLayout &L, const void *K, const int32_t *seq_lens,
                          const float *mu, const int32_t *init_idx, int iters, uint8_t *codes, float *codebook,
                          int32_t *counts, char *ws, cudaStream_t stream);

// 2-bit value rows (values.cu)
sikv_status launch_quantize_values(const sikv_params &p, const void *V, const int32_t *seq_lens, uint8_t *vq,
                                   int32_t *status, cudaStream_t stream);

sikv_status launch_append(const sikv_params &p, const void *K, const int32_t *start, const int32_t *count,
                          const float *mu, uint8_t *codes, int32_t *status, cudaStream_t stream);
sikv_status launch_score(const sikv_params &p, const void *q, const uint8_t *codes,
                         const float *codebook, const float *mu, const int32_t *seq_lens,
                         float *scores, int32_t *status, cudaStream_t stream);

sikv_status launch_topk(const sikv_params &p, const float *scores, const int32_t *seq_lens,
                        const int32_t *k_per_seq, int32_t *idx, int32_t *status,
                        cudaStream_t stream);

sikv_status launch_sparse_attn(const sikv_params &p, const void *q, const void *K, const void *V,
                               const uint8_t *vq,
                               const uint8_t *codes, const float *codebook, const float *mu,
                               const int32_t *idx, const int32_t *k_per_seq,
                               const int32_t *seq_lens, void *out, char *ws, size_t attn_base,
                               int32_t *status, cudaStream_t stream);

// Fused single-launch decode (decode_fused.cu).
constexpr int kFusedMaxCps = 64;          // CTAs per segment, upper bound for the workspace

struct FusedCtl {                          // per-segment counters, zero between launches
    int arrive1, arrive2, arrive3, ncand;
    int pad[4];
};

struct FusedLayout {
    size_t ghist = 0, ctl = 0, cand = 0, selcnt = 0, part_o = 0, part_ml = 0, total = 0;
};

struct FusedPlan {
    bool ok = false;
    int cps = 0, chunk = 0, npt = 0, gm = 0, grid = 0;
};

FusedLayout fused_layout(const sikv_params &p, size_t base);
// vq: the kernel that reads 2-bit value rows for the selected tokens
FusedPlan fused_plan(const sikv_params &p, bool vq = false);
int fused_sub_batch(const sikv_params &p, bool vq = false);   // sequences per launch when the batch must be split; 0: no split
// L: the coordination layout in ws; every launch that shares ws must use the
// same layout, because each launch leaves only its own segments' state zeroed
sikv_status launch_decode_fused(const sikv_params &p, const FusedPlan &plan, const FusedLayout &L, const void *q,
                                const void *K, const void *V, const uint8_t *vq, const uint8_t *codes,
                                const float *codebook, const float *mu,
                                const int32_t *seq_lens, const int32_t *k_per_seq, void *out, int32_t *idx_out,
                                float *scores_out, char *ws, int32_t *status, cudaStream_t stream);

// Cluster single-launch decode (decode_cluster.cu).
struct ClusterPlan {
    bool ok = false;
    int csize = 0, chunk = 0, npt = 0, gm = 0, grid = 0;
};
// vq: the kernel that reads 2-bit value rows for the selected tokens
ClusterPlan cluster_plan(const sikv_params &p, bool vq = false);
size_t fused_cand_cap(const sikv_params &p);
// cand: the workspace candidate list ([segs][cand_cap] pairs, cand_cap >=
// max_seq_len), used only by CTAs whose threshold bin overflows shared memory
sikv_status launch_decode_cluster(const sikv_params &p, const ClusterPlan &plan, const void *q, const void *K,
                                  const void *V, const uint8_t *vq, const uint8_t *codes, const float *codebook,
                                  const float *mu, const int32_t *seq_lens, const int32_t *k_per_seq, void *out,
                                  int32_t *idx_out, float *scores_out, uint2 *cand, size_t cand_cap, int32_t *status,
                                  cudaStream_t stream);

int device_sm_count();

}  // namespace sikv
